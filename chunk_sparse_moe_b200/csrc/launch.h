// launch.h -- host-side launchers of the BlockFFN kernels (internal to the
// library; the public interface is include/blockffn.h).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace bffn {

// bf16 matrix [rows, cols] as a 3-D TMA tensor {64, row, column block}; a box
// {64, box_rows, nkb} lands as nkb consecutive [box_rows x 128 B] 128-byte-
// swizzled tiles (defined in abi.cu)
bool make_map_kblocks(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows,
                      uint32_t nkb);

cudaError_t launch_route(const void* x, const void* W_r, const float* b_r, const float* gamma,
                         float eps, int T, int d_h, int E, bool bf16, float* gates,
                         cudaStream_t s);

cudaError_t launch_residual_layernorm(const void* y, const void* x, const float* ln_gamma, const float* ln_beta,
                                      float eps, int T, int d_h, bool bf16, void* out, cudaStream_t s);

cudaError_t launch_chunk_union(const float* gates, int T, int E, int n, int32_t* counts,
                               int32_t* idx, uint32_t* tmask, cudaStream_t s);

// compute_union: tables from the gates; otherwise the caller's tables are checked
// (a mismatch records an error in ctl and the forward computes nothing)
cudaError_t launch_chunk_union_plan(const float* gates, int T, int E, int n, int32_t* counts,
                                    int32_t* idx, uint32_t* tmask, bool compute_union, Ctl* ctl,
                                    int32_t* offsets, int32_t* pair_ce, void* y, int d_h,
                                    int y_elem_bytes, cudaStream_t s);

// group tables of the multi-chunk forward (see union.cu)
cudaError_t launch_group_plan(const float* gates, int T, int E, int n, int32_t* counts, int32_t* idx,
                              uint32_t* tmask, bool compute_union, Ctl* ctl, int NG, int NGr,
                              int32_t* gcounts, int32_t* goffsets, int32_t* gpair, __nv_bfloat16* y,
                              int d_h, cudaStream_t s);

// b_in [E, d_e] and b_out [E, d_h] fp32 expert biases, or nullptr
cudaError_t launch_forward_f32(const float* x, const float* gates, const float* W_in,
                               const float* W_out, const float* b_in, const float* b_out,
                               const int32_t* counts, const int32_t* offsets,
                               const int32_t* pair_ce, const uint32_t* tmask, const Ctl* ctl,
                               float* hbuf, int T, int d_h, int E, int d_e, int n, float* y,
                               int num_sms, cudaStream_t s);

// ybias[t, :] = sum over the union of t's chunk (ascending) of the gate-masked
// fc2 biases, bit_t ? g[t,e] b_out[e,:] : 0, fp32 [T, d_h] (expert_bias.cu)
cudaError_t launch_expert_bias_sum(const float* gates, const int32_t* counts, const int32_t* idx,
                                   const uint32_t* tmask, const Ctl* ctl, const float* b_out, int T,
                                   int d_h, int E, int n, float* ybias, cudaStream_t s);

// Arguments of the multi-chunk group forward (forward_group.cu).
struct GrArgs {
    const float* gates;       // [T, E]
    const uint32_t* tmask;    // [C, E] chunk token masks
    const int32_t* gcounts;   // [NGr] size of each group's expert set
    const int32_t* goffsets;  // [NGr + 1]
    const int32_t* gpair;     // [P] (group << 8) | expert, by group, experts ascending
    __nv_bfloat16* hbuf;      // [P][N][d_e] gated activations h'
    float* partB;             // [grid][2][N*128] split-expert partial sums (expert-out)
    uint32_t* readyA;         // [2][cnt_a_len] expert-in units whose h' is written
    uint32_t* cntB;           // [2][cnt_b_len] blocks that published an expert-out partial
    long long cnt_a_len;      // NGr*E*MT
    long long cnt_b_len;      // NGr*RT
    Ctl* ctl;
    __nv_bfloat16* y;         // [T, d_h]
    const float* b_in;        // [E, d_e] fc1 biases, or nullptr
    const float* ybias;       // [T, d_h] per-token fc2 bias sums (expert_bias.cu), or nullptr
    int T, d_h, E, d_e, n;
    int N;     // tokens per MMA: 128 or 256
    int NT;    // tokens per group: (N / n) * n
    int NGr;   // groups
    int KB, MT, RT, KBe;
    int skip_flag_unit;       // test support: unit whose h' is never announced ready (-1: off)
    unsigned long long wait_ns;
    unsigned long long shape_key;
    unsigned long long* trace;   // optional [grid][64] globaltimer stamps (nullptr: off)
};
// maps: x [T, d_h] (box {64, N}), W_in [E*d_e, d_h] and W_out [E*d_h, d_e] (box
// {64, 128}), h' [P*N, d_e] (box {64, N}): 2-D, bf16, 128-byte swizzle; the
// expert-out partial tiles as fp32 lines of 512 floats (box {128, N/4}, no swizzle)
cudaError_t launch_forward_group(const GrArgs& a, const CUtensorMap* maps, int grid, cudaStream_t s);

// Arguments of the single-chunk forward (see forward_decode.cu): expert-in
// units are (union expert, 128-row tile of W_in) split along K over a pair of
// blocks (a cluster of 2); expert-out row tiles are split over blocks and
// reduced in two passes.
struct DcArgs {
    const float* gates;       // [T, E], T <= n
    // the caller's union tables of the chunk (counts [1], idx [E], tmask [E]), or
    // all nullptr: the kernel forms the union from the gates
    const int32_t* counts_in;
    const int32_t* idx_in;
    const uint32_t* tmask_in;
    __nv_bfloat16* y;         // [T, d_h]
    __nv_bfloat16* hbuf;      // [E slots][N][d_e] gated activations h'
    uint32_t* readyA;         // [2][E] halves of an expert slot written, by launch parity
    Ctl* ctl;
    const float* b_in;        // [E, d_e] fc1 biases, or nullptr
    const float* b_out;       // [E, d_h] fc2 biases, or nullptr
    int T, d_h, E, d_e, n, N;
    int KB;    // d_h / 64
    int RT;    // d_h / 128
    int skip_unit;            // test support: expert-in half never counted in (-1: off)
    unsigned long long wait_ns;
    unsigned long long* trace;   // optional [grid][64] globaltimer stamps
    unsigned long long shape_key;   // the workspace layout this launch expects (Ctl::shape_key)
};
// maps: x [T, d_h] (box N rows), W_in [E*d_e, d_h] and W_out [E*d_h, d_e] (box 128
// rows), h' [E*N, d_e] (box N rows): 3-D {64, rows, column block} boxes of two
// 64-wide column blocks, 128-byte swizzle; y [T, d_h] (box 32 wide x N rows, no
// swizzle, for stores)
cudaError_t launch_forward_decode(const DcArgs& a, const CUtensorMap* maps, int grid, cudaStream_t s);
size_t forward_decode_smem_bytes();
// clusters of 4 blocks that can be resident at once (the launch uses 4 x this
// many blocks), -1 on error
int decode_max_clusters();

}  // namespace bffn
