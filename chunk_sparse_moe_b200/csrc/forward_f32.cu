// forward_f32.cu -- fp32 union-expert forward on CUDA cores (FFMA).
//
// Pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device
// Deployment", Core Concept (union of the experts activated across n tokens,
// unneeded activations masked after computing) and Architecture Overview
// (non-gated Swish experts).
//
// The fp32 workload needs a relative L2 error of 1e-5, which TF32 tensor cores
// cannot give, so this path stays on FFMA.  Two kernels:
//   A: one block per (chunk, union expert) pair: h'[p, j, :] =
//      bit_j ? g[t,e] * Swish(W_in_e x_t) : 0 for the chunk's tokens.  A masked
//      token's activation is exactly zero whether or not it is computed, so the
//      block skips the dot products of masked tokens.
//   B: y[t, i] = sum over the chunk's union experts, ascending, of
//      W_out_e[i, :] . h'[p, j, :], one thread per output element, a fixed order.
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"

namespace bffn {

__global__ void __launch_bounds__(256) expert_in_f32_kernel(
    const float* __restrict__ x, const float* __restrict__ gates, const float* __restrict__ W_in,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ pair_ce,
    const uint32_t* __restrict__ tmask, int T, int d_h, int E, int d_e, int n, int C,
    float* __restrict__ hbuf) {
    const int P = offsets[C];
    for (int p = blockIdx.x; p < P; p += gridDim.x) {
        const int ce = pair_ce[p];
        const int c = ce >> 8, e = ce & 255;
        const uint32_t bits = tmask[(size_t)c * E + e];
        for (int o = threadIdx.x; o < n * d_e; o += blockDim.x) {
            const int j = o / d_e, row = o % d_e;
            const int t = c * n + j;
            float out = 0.f;
            if (t < T && ((bits >> j) & 1u)) {
                const float* w = W_in + ((size_t)e * d_e + row) * d_h;
                const float* xt = x + (size_t)t * d_h;
                float z = 0.f;
                for (int k = 0; k < d_h; ++k) z = fmaf(__ldg(w + k), __ldg(xt + k), z);
                const float sw = z / (1.0f + expf(-z));
                out = gates[(size_t)t * E + e] * sw;
            }
            hbuf[((size_t)p * n + j) * d_e + row] = out;
        }
    }
}

__global__ void __launch_bounds__(128) expert_out_f32_kernel(
    const float* __restrict__ W_out, const int32_t* __restrict__ counts,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ pair_ce,
    const float* __restrict__ hbuf, int T, int d_h, int d_e, int n, float* __restrict__ y) {
    const int c = blockIdx.y;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= d_h) return;
    const int cnt = counts[c], off = offsets[c];
    const int t0 = c * n, nt = min(n, T - t0);
    for (int j = 0; j < nt; ++j) {
        float acc = 0.f;
        for (int s = 0; s < cnt; ++s) {
            const int e = pair_ce[off + s] & 255;
            const float* w = W_out + ((size_t)e * d_h + i) * d_e;
            const float* h = hbuf + ((size_t)(off + s) * n + j) * d_e;
            for (int q = 0; q < d_e; ++q) acc = fmaf(__ldg(w + q), h[q], acc);
        }
        y[(size_t)(t0 + j) * d_h + i] = acc;
    }
}

cudaError_t launch_forward_f32(const float* x, const float* gates, const float* W_in,
                               const float* W_out, const int32_t* counts, const int32_t* offsets,
                               const int32_t* pair_ce, const uint32_t* tmask, float* hbuf,
                               int T, int d_h, int E, int d_e, int n, float* y, int num_sms,
                               cudaStream_t s) {
    const int C = (T + n - 1) / n;
    if (C == 0) return cudaSuccess;
    const long long pmax = (long long)C * E;
    const int gridA = (int)(pmax < 8LL * num_sms ? pmax : 8LL * num_sms);
    expert_in_f32_kernel<<<gridA, 256, 0, s>>>(x, gates, W_in, offsets, pair_ce, tmask, T, d_h,
                                               E, d_e, n, C, hbuf);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    dim3 gridB((d_h + 127) / 128, C);
    expert_out_f32_kernel<<<gridB, 128, 0, s>>>(W_out, counts, offsets, pair_ce, hbuf, T, d_h,
                                                d_e, n, y);
    return cudaGetLastError();
}

}  // namespace bffn
