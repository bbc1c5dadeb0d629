// launch.h -- host-side launchers of the BlockFFN kernels (internal to the
// library; the public interface is include/blockffn.h).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace bffn {

cudaError_t launch_route(const void* x, const void* W_r, const float* b_r, const float* gamma,
                         float eps, int T, int d_h, int E, bool bf16, float* gates,
                         cudaStream_t s);

cudaError_t launch_chunk_union(const float* gates, int T, int E, int n, int32_t* counts,
                               int32_t* idx, uint32_t* tmask, cudaStream_t s);

cudaError_t launch_chunk_union_plan(const float* gates, int T, int E, int n, int32_t* counts,
                                    int32_t* idx, uint32_t* tmask, int32_t* offsets,
                                    int32_t* pair_ce, void* y, int d_h, int y_elem_bytes,
                                    cudaStream_t s);

cudaError_t launch_forward_f32(const float* x, const float* gates, const float* W_in,
                               const float* W_out, const int32_t* counts, const int32_t* offsets,
                               const int32_t* pair_ce, const uint32_t* tmask, float* hbuf,
                               int T, int d_h, int E, int d_e, int n, float* y, int num_sms,
                               cudaStream_t s);

// Arguments of the tensor-core union-expert forward (bf16).
struct TcArgs {
    const float* gates;       // [T, E]
    const int32_t* counts;    // [C]       (plan tables; unused when fuse_union)
    const int32_t* offsets;   // [C + 1]
    const int32_t* pair_ce;   // [P]       (chunk << 8) | expert
    const uint32_t* tmask;    // [C, E]
    __nv_bfloat16* hbuf;      // [C*E*N, d_e] gated activations of every pair
    float* partA;             // [grid][2][N*128] split-K partial sums (expert-in GEMM)
    float* partB;             // [grid][2][N*128] split-expert partial sums (expert-out GEMM)
    uint32_t* cntA;           // [C*E*MT] arrival counters
    uint32_t* cntB;           // [C*RT]
    uint32_t* flags;          // [C*E*MT] "gated activation ready" stamps
    Ctl* ctl;
    __nv_bfloat16* y;         // [T, d_h]
    int T, d_h, E, d_e, n, N, C;
    int KB;    // d_h / 64: k-blocks of one expert-in unit
    int MT;    // d_e / 128: 128-row tiles of one expert's W_in
    int RT;    // d_h / 128: 128-row tiles of y
    int KBe;   // d_e / 64: k-blocks of one expert in the expert-out GEMM
    int fuse_union;   // 1 when C == 1: each block forms the union itself from gates
    int skip_flag_unit;   // test support: never publish this A unit's flag (-1: off)
    unsigned long long wait_ns;
};

// maps: x, W_in, W_out, hbuf (2-D, bf16, 128-byte swizzle, boxes {64,N},{64,128},{64,128},{64,N})
cudaError_t launch_forward_tc(const TcArgs& a, const CUtensorMap* maps, int grid, cudaStream_t s);
size_t forward_tc_smem_bytes();

}  // namespace bffn
