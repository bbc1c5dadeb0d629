// expert_bias.cu -- the fc2-bias part of the multi-chunk bf16 forward.
//
// Pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device
// Deployment", Router Architecture Setup (each expert's fc2 is an nn.Linear,
// bias on by default) and Full BlockFFN Layer with Combined Losses (the gate
// multiplies the whole expert output, so the bias too).
//
// With fc2 biases the layer output gains, per token,
//   ybias[t, i] = sum over the union of t's chunk, ascending, of
//                 (bit_t(tmask[c, e]) ? g[t, e] : 0) * b_out[e, i]
// (the same select as the expert terms: a token adds a bias only for the experts
// it activates).  This kernel writes ybias in fp32 and the group kernel adds it
// to the expert sum before y is rounded.  One block per (chunk, 256 columns): a
// thread owns a column and the chunk's <= 32 tokens; the chunk's masked gates of
// 32 union experts at a time are staged in shared memory.  The work is
// C * d_h * |U_c| * n FMAs of fp32 (bandwidth: b_out rows of the union, L2-hot,
// and ybias once), small next to the expert GEMMs.
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace bffn {

constexpr int kEbThreads = 256;

__global__ void __launch_bounds__(kEbThreads) expert_bias_sum_kernel(
    const float* __restrict__ gates, const int32_t* __restrict__ counts, const int32_t* __restrict__ idx,
    const uint32_t* __restrict__ tmask, const Ctl* ctl, const float* __restrict__ b_out, int T, int d_h,
    int E, int n, int C, float* __restrict__ ybias) {
    // the forward after this kernel may set itself up meanwhile; it waits for
    // this kernel's completion before reading ybias
    griddep_launch_dependents();
    if (__ldcg(&ctl->status) != 0) return;   // refused tables (or an earlier error): nothing runs
    __shared__ float sgm[32][32];   // [union slot][token]: bit ? gate : 0
    __shared__ int se[32];
    const int ncb = (d_h + kEbThreads - 1) / kEbThreads;
    for (long long blk = blockIdx.x; blk < (long long)C * ncb; blk += gridDim.x) {
        const int c = (int)(blk / ncb);
        const int col = (int)(blk % ncb) * kEbThreads + threadIdx.x;
        const int t0 = c * n, nt = min(n, T - t0);
        const int cnt = counts[c];
        float acc[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = 0.f;
        for (int s0 = 0; s0 < cnt; s0 += 32) {
            __syncthreads();   // the previous batch is read
            for (int k = threadIdx.x; k < 32 * 32; k += kEbThreads) {
                const int sl = k >> 5, j = k & 31;
                float v = 0.f;
                if (s0 + sl < cnt && j < nt) {
                    const int e = idx[(size_t)c * E + s0 + sl];
                    if ((tmask[(size_t)c * E + e] >> j) & 1u) v = gates[(size_t)(t0 + j) * E + e];
                    if (j == 0) se[sl] = e;
                }
                sgm[sl][j] = v;
            }
            __syncthreads();
            if (col < d_h) {
                const int ns = min(32, cnt - s0);
                for (int sl = 0; sl < ns; ++sl) {
                    const float b = __ldg(b_out + (size_t)se[sl] * d_h + col);
#pragma unroll
                    for (int j = 0; j < 32; ++j) acc[j] = fmaf(sgm[sl][j], b, acc[j]);
                }
            }
        }
        if (col < d_h) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (j < nt) ybias[(size_t)(t0 + j) * d_h + col] = acc[j];
        }
    }
}

cudaError_t launch_expert_bias_sum(const float* gates, const int32_t* counts, const int32_t* idx,
                                   const uint32_t* tmask, const Ctl* ctl, const float* b_out, int T,
                                   int d_h, int E, int n, float* ybias, cudaStream_t s) {
    const int C = (T + n - 1) / n;
    if (C == 0) return cudaSuccess;
    const long long blocks = (long long)C * ((d_h + kEbThreads - 1) / kEbThreads);
    const int grid = (int)(blocks < 4096 ? blocks : 4096);
    expert_bias_sum_kernel<<<grid, kEbThreads, 0, s>>>(gates, counts, idx, tmask, ctl, b_out, T, d_h, E, n, C,
                                                       ybias);
    return cudaGetLastError();
}

}  // namespace bffn
