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

// Exclusive scan of in[0..count) into out[0..count], out[count] = the total,
// by one whole block (blockDim.x a multiple of 32, at most 1024).
__device__ void block_exclusive_scan(const int32_t* in, int count, int32_t* out) {
    __shared__ int32_t warp_sums[32];
    __shared__ int32_t carry;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < count; base += blockDim.x) {
        const int c = base + threadIdx.x;
        const int v = c < count ? in[c] : 0;
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
        if (c < count) out[c] = excl;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = excl + v;
        __syncthreads();
    }
    if (threadIdx.x == 0) out[count] = carry;
    __syncthreads();
}

// Caller-supplied union tables of chunk c: counts[c] and idx[c, :] must be what
// the token masks tmask[c, :] give (the experts with a nonzero mask, ascending,
// then -1).  A mismatch records BLOCKFFN_ERR_INVALID_ARG (detail kUnionTables)
// in the workspace; the forward then computes nothing.
__device__ __forceinline__ void check_one_chunk(int E, int c, int lane, const int32_t* counts,
                                                const int32_t* idx, const uint32_t* tmask, Ctl* ctl) {
    int base = 0;
    bool bad = false;
    for (int g0 = 0; g0 < E; g0 += 32) {
        const int e = g0 + lane;
        const bool on = e < E && tmask[(size_t)c * E + e] != 0u;
        const uint32_t bal = __ballot_sync(0xffffffffu, on);
        if (on && idx[(size_t)c * E + base + __popc(bal & ((1u << lane) - 1u))] != e) bad = true;
        base += __popc(bal);
    }
    for (int s = base + lane; s < E; s += 32)
        if (idx[(size_t)c * E + s] != -1) bad = true;
    if (lane == 0 && counts[c] != base) bad = true;
    if (__any_sync(0xffffffffu, bad) && lane == 0) record_error(ctl, kErrInvalidArg, kUnionTables);
}

// After the table phase (a block-wide barrier first): true when the workspace
// holds an error -- the caller's tables were refused just now, or an earlier
// launch failed -- in which case the forward computes nothing.
__device__ __forceinline__ bool plan_refused(const Ctl* ctl) {
    __shared__ int s_refused;
    __syncthreads();
    if (threadIdx.x == 0) s_refused = __ldcg(&ctl->status) != 0;
    __syncthreads();
    return s_refused != 0;
}

// Forward-internal union: one block of 1024 threads over all chunks (or a check
// of the caller's tables), followed by the exclusive scan of the counts
// (offsets) and the pair table pair_ce[p] = (chunk << 8) | expert, p =
// offsets[c] + slot, in chunk order.  Rows of y that belong to chunks with no
// active expert are zeroed here (no later kernel writes them).
__global__ void __launch_bounds__(1024) chunk_union_plan_kernel(
    const float* __restrict__ gates, int T, int E, int n, int C, int32_t* counts,
    int32_t* idx, uint32_t* tmask, int compute_union, Ctl* ctl, int32_t* __restrict__ offsets,
    int32_t* __restrict__ pair_ce, void* __restrict__ y, int d_h, int y_elem_bytes) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    if (compute_union) {
        for (int c = warp; c < C; c += nwarps) union_one_chunk(gates, T, E, n, c, lane, counts, idx, tmask);
    } else {
        for (int c = warp; c < C; c += nwarps) check_one_chunk(E, c, lane, counts, idx, tmask, ctl);
    }
    if (plan_refused(ctl)) return;   // refused tables or an earlier error: compute nothing
    block_exclusive_scan(counts, C, offsets);

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
                                    int32_t* idx, uint32_t* tmask, bool compute_union, Ctl* ctl,
                                    int32_t* offsets, int32_t* pair_ce, void* y, int d_h,
                                    int y_elem_bytes, cudaStream_t s) {
    const int C = (T + n - 1) / n;
    if (C == 0) return cudaSuccess;
    chunk_union_plan_kernel<<<1, 1024, 0, s>>>(gates, T, E, n, C, counts, idx, tmask,
                                               compute_union ? 1 : 0, ctl, offsets, pair_ce, y, d_h,
                                               y_elem_bytes);
    return cudaGetLastError();
}

// Group tables of the multi-chunk forward (forward_group.cu), one launch.  Groups
// are NG consecutive chunks; a group's expert set is the union of its chunks'
// unions, ascending: e is in it when some chunk of the group has a nonzero
// token mask for e.
//   1. every warp takes one chunk: its tables from the gates (union_one_chunk),
//      or the caller's tables checked against their token masks;
//   2. the last block to finish (a counter in the control block, reset by that
//      block for the next launch) builds the group tables: gcounts[g], their
//      exclusive scan goffsets, gpair[goffsets[g] + s] = (g << 8) | (s-th expert
//      of the set), and zeroes the rows of y of a group whose set is empty (no
//      later kernel writes them).
// Launched as a programmatic dependent of the previous kernel (the router, when
// the gates come from it): it waits for that kernel before reading the gates,
// and lets the group kernel, its own dependent, be scheduled at once.
__device__ __forceinline__ bool group_has(const uint32_t* tmask, int E, int C, int NG, int g, int e) {
    bool any = false;
    if (e < E) {
        const int c1 = min(C, (g + 1) * NG);
        for (int c = g * NG; c < c1; ++c) any = any || __ldcg(tmask + (size_t)c * E + e) != 0u;
    }
    return any;
}

constexpr int kGpThreads = 256;

__global__ void __launch_bounds__(kGpThreads) group_union_plan_kernel(
    const float* __restrict__ gates, int T, int E, int n, int C, int32_t* counts, int32_t* idx, uint32_t* tmask,
    int compute_union, Ctl* ctl, int NG, int NGr, int32_t* __restrict__ gcounts, int32_t* __restrict__ goffsets,
    int32_t* __restrict__ gpair, __nv_bfloat16* __restrict__ y, int d_h) {
    __shared__ int s_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    griddep_wait();
    if (threadIdx.x == 0) griddep_launch_dependents();
    const int c = blockIdx.x * nwarps + warp;
    if (c < C) {
        if (compute_union) union_one_chunk(gates, T, E, n, c, lane, counts, idx, tmask);
        else check_one_chunk(E, c, lane, counts, idx, tmask, ctl);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        fence_acq_rel_gpu();   // this block's tables before its count
        s_last = atomicAdd(&ctl->plan_done, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (!s_last) return;
    fence_acq_rel_gpu();       // every block's tables after the count that saw them all
    if (threadIdx.x == 0) ctl->plan_done = 0u;
    if (plan_refused(ctl)) return;   // refused tables or an earlier error: compute nothing
    for (int g = warp; g < NGr; g += nwarps) {
        int base = 0;
        for (int g0 = 0; g0 < E; g0 += 32)
            base += __popc(__ballot_sync(0xffffffffu, group_has(tmask, E, C, NG, g, g0 + lane)));
        if (lane == 0) gcounts[g] = base;
    }
    __syncthreads();
    block_exclusive_scan(gcounts, NGr, goffsets);
    const int NT = NG * n;
    for (int g = warp; g < NGr; g += nwarps) {
        int base = goffsets[g];
        for (int g0 = 0; g0 < E; g0 += 32) {
            const int e = g0 + lane;
            const bool on = group_has(tmask, E, C, NG, g, e);
            const uint32_t bal = __ballot_sync(0xffffffffu, on);
            if (on) gpair[base + __popc(bal & ((1u << lane) - 1u))] = (g << 8) | e;
            base += __popc(bal);
        }
        if (gcounts[g] == 0) {
            const int t0 = g * NT, nt = min(NT, T - t0);
            uint4* dst = reinterpret_cast<uint4*>(y + (size_t)t0 * d_h);   // d_h % 128 == 0
            const size_t n16 = (size_t)nt * d_h / 8;
            for (size_t i = lane; i < n16; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
        }
    }
}

cudaError_t launch_group_plan(const float* gates, int T, int E, int n, int32_t* counts, int32_t* idx,
                              uint32_t* tmask, bool compute_union, Ctl* ctl, int NG, int NGr,
                              int32_t* gcounts, int32_t* goffsets, int32_t* gpair, __nv_bfloat16* y,
                              int d_h, cudaStream_t s) {
    const int C = (T + n - 1) / n;
    if (C == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((C + kGpThreads / 32 - 1) / (kGpThreads / 32));
    cfg.blockDim = dim3(kGpThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, group_union_plan_kernel, gates, T, E, n, C, counts, idx, tmask,
                              compute_union ? 1 : 0, ctl, NG, NGr, gcounts, goffsets, gpair, y, d_h);
}

}  // namespace bffn
