// union.cu -- chunk union of active experts.
//
// Pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device
// Deployment", Core Concept and Architecture Overview: the acceleration kernel
// processes n consecutive tokens at once and computes only the union of the
// experts any of them activates.
//
// One warp per chunk.  Lane l owns experts l, l+32, ...; it reads its expert's
// gate for every token of the chunk (for each token the warp reads a coalesced
// 128-byte row segment; all loads are in flight together) and ORs the tokens'
// active bits into a 32-bit token mask.  A ballot over
// the lanes' "any token active" bits then compacts the active experts of each
// 32-expert group in ascending order (prefix popcount of the ballot).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"

namespace bffn {

__device__ __forceinline__ void union_one_chunk(const float* __restrict__ gates, int T, int E,
                                                int n, int c, int lane,
                                                int32_t* __restrict__ counts,
                                                int32_t* __restrict__ idx,
                                                uint32_t* __restrict__ tmask) {
    int base = 0;
    const int t0 = c * n;
    const int nt = min(n, T - t0);
    for (int g0 = 0; g0 < E; g0 += 32) {
        const int e = g0 + lane;
        // all n loads of the lane are issued before the first use
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j)
            v[j] = (e < E && j < nt) ? __ldg(gates + (size_t)(t0 + j) * E + e) : 0.f;
        uint32_t bits = 0u;
#pragma unroll
        for (int j = 0; j < 32; ++j) bits |= (v[j] != 0.0f ? 1u : 0u) << j;
        if (e < E) tmask[(size_t)c * E + e] = bits;
        const uint32_t bal = __ballot_sync(0xffffffffu, bits != 0u);
        if (bits != 0u) idx[(size_t)c * E + base + __popc(bal & ((1u << lane) - 1u))] = e;
        base += __popc(bal);
    }
    for (int s = base + lane; s < E; s += 32) idx[(size_t)c * E + s] = -1;
    if (lane == 0) counts[c] = base;
}

// Public union: many blocks, warp per chunk.
__global__ void __launch_bounds__(256) chunk_union_kernel(const float* __restrict__ gates, int T,
                                                          int E, int n, int C,
                                                          int32_t* __restrict__ counts,
                                                          int32_t* __restrict__ idx,
                                                          uint32_t* __restrict__ tmask) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp < C) union_one_chunk(gates, T, E, n, warp, lane, counts, idx, tmask);
}

// Forward-internal union: one block of 1024 threads over all chunks, followed
// by the exclusive scan of the counts (offsets) and the pair table
// pair_ce[p] = (chunk << 8) | expert, p = offsets[c] + slot, in chunk order.
// Rows of y that belong to chunks with no active expert are zeroed here (no
// later kernel writes them).
__global__ void __launch_bounds__(1024) chunk_union_plan_kernel(
    const float* __restrict__ gates, int T, int E, int n, int C, int32_t* __restrict__ counts,
    int32_t* __restrict__ idx, uint32_t* __restrict__ tmask, int32_t* __restrict__ offsets,
    int32_t* __restrict__ pair_ce, void* __restrict__ y, int d_h, int y_elem_bytes) {
    __shared__ int32_t warp_sums[32];
    __shared__ int32_t carry;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    for (int c = warp; c < C; c += nwarps) union_one_chunk(gates, T, E, n, c, lane, counts, idx, tmask);
    __syncthreads();

    // exclusive scan of counts[0..C) in tiles of blockDim
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < C; base += blockDim.x) {
        const int c = base + threadIdx.x;
        const int v = c < C ? counts[c] : 0;
        int incl = v;
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        if (lane == 31) warp_sums[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int w = lane < nwarps ? warp_sums[lane] : 0;
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += u;
            }
            warp_sums[lane] = w;  // inclusive over warps
        }
        __syncthreads();
        const int excl = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + incl - v;
        if (c < C) offsets[c] = excl;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = excl + v;
        __syncthreads();
    }
    if (threadIdx.x == 0) offsets[C] = carry;
    __syncthreads();

    // pair table and zero rows of empty chunks
    for (int c = warp; c < C; c += nwarps) {
        const int cnt = counts[c];
        const int off = offsets[c];
        for (int s = lane; s < cnt; s += 32) pair_ce[off + s] = (c << 8) | idx[(size_t)c * E + s];
        if (cnt == 0 && y != nullptr) {
            const int t0 = c * n, nt = min(n, T - t0);
            const size_t bytes = (size_t)nt * d_h * y_elem_bytes;
            uint4* dst = reinterpret_cast<uint4*>(static_cast<char*>(y) + (size_t)t0 * d_h * y_elem_bytes);
            for (size_t i = lane; i < bytes / 16; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
            char* tail = reinterpret_cast<char*>(dst) + (bytes / 16) * 16;
            for (size_t i = lane; i < bytes % 16; i += 32) tail[i] = 0;
        }
    }
}

cudaError_t launch_chunk_union(const float* gates, int T, int E, int n, int32_t* counts,
                               int32_t* idx, uint32_t* tmask, cudaStream_t s) {
    const int C = (T + n - 1) / n;
    if (C == 0) return cudaSuccess;
    const int warps_per_block = 8;
    const int blocks = (C + warps_per_block - 1) / warps_per_block;
    chunk_union_kernel<<<blocks, warps_per_block * 32, 0, s>>>(gates, T, E, n, C, counts, idx,
                                                               tmask);
    return cudaGetLastError();
}

cudaError_t launch_chunk_union_plan(const float* gates, int T, int E, int n, int32_t* counts,
                                    int32_t* idx, uint32_t* tmask, int32_t* offsets,
                                    int32_t* pair_ce, void* y, int d_h, int y_elem_bytes,
                                    cudaStream_t s) {
    const int C = (T + n - 1) / n;
    if (C == 0) return cudaSuccess;
    chunk_union_plan_kernel<<<1, 1024, 0, s>>>(gates, T, E, n, C, counts, idx, tmask, offsets,
                                               pair_ce, y, d_h, y_elem_bytes);
    return cudaGetLastError();
}

}  // namespace bffn
