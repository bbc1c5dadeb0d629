// forward_f32.cu -- fp32 union-expert forward on CUDA cores (FFMA).
//
// Pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device
// Deployment", Core Concept (union of the experts activated across n tokens,
// unneeded activations masked after computing) and Architecture Overview
// (non-gated Swish experts).
//
// The fp32 workload needs a relative L2 error of 1e-5, which TF32 tensor cores
// cannot give, so this path stays on FFMA.  Two kernels, both staging coalesced
// 64 x 64 tiles of the weights and of the chunk's activations in shared memory;
// a lane owns one token of the chunk and a warp eight output rows:
//   A: one block per (chunk, union expert) pair at a time:
//        h[j, r]  = sum_k W_in_e[r, k] x[t_j, k] + b_in[e, r]  for every token j of the chunk
//        h'[j, r] = bit_j ? g[t_j, e] * Swish(h[j, r]) : 0
//      Every token of the chunk is computed and the mask applied afterwards (a
//      select, so a masked token gives exactly 0), as the method states.
//   B: one block per (64 rows of y, chunk):
//        y[t_j, i] = sum over the chunk's union experts, ascending, of
//                    sum_q W_out_e[i, q] h'[p, j, q]
//                  + sum over the same experts of (bit_j ? g[t_j, e] b_out[e, i] : 0)
//      each output's sums running sequentially over (expert, q), then over the
//      experts' biases: a fixed order.  The biases (Router Architecture Setup:
//      the experts' nn.Linear layers) are optional.
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"

namespace bffn {

constexpr int kF32Tile = 64;       // rows and k per staged tile
constexpr int kF32Threads = 256;   // 8 warps x 8 rows

__global__ void __launch_bounds__(kF32Threads) expert_in_f32_kernel(
    const float* __restrict__ x, const float* __restrict__ gates, const float* __restrict__ W_in,
    const float* __restrict__ b_in, const int32_t* __restrict__ offsets, const int32_t* __restrict__ pair_ce,
    const uint32_t* __restrict__ tmask, const Ctl* ctl, int T, int d_h, int E, int d_e, int n, int C,
    float* __restrict__ hbuf) {
    if (__ldcg(&ctl->status) != 0) return;   // the union tables were refused (or an earlier error)
    __shared__ float sw[kF32Tile][kF32Tile + 1];   // [row][k]
    __shared__ float sx[32][kF32Tile + 1];         // [token][k]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = offsets[C];
    for (int p = blockIdx.x; p < P; p += gridDim.x) {
        const int ce = pair_ce[p];
        const int c = ce >> 8, e = ce & 255;
        const uint32_t bits = tmask[(size_t)c * E + e];
        const int t = c * n + lane;                       // this lane's token
        const bool live = lane < n && t < T;              // a token of the chunk
        const float g = live ? gates[(size_t)t * E + e] : 0.f;
        for (int r0 = 0; r0 < d_e; r0 += kF32Tile) {
            float acc[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) acc[u] = 0.f;
            for (int k0 = 0; k0 < d_h; k0 += kF32Tile) {
                __syncthreads();
                for (int i = threadIdx.x; i < kF32Tile * kF32Tile; i += kF32Threads) {
                    const int r = i / kF32Tile, k = i % kF32Tile;
                    sw[r][k] = (r0 + r < d_e && k0 + k < d_h)
                                   ? __ldg(W_in + ((size_t)e * d_e + r0 + r) * d_h + k0 + k) : 0.f;
                }
                for (int i = threadIdx.x; i < 32 * kF32Tile; i += kF32Threads) {
                    const int j = i / kF32Tile, k = i % kF32Tile;
                    const int tj = c * n + j;
                    sx[j][k] = (j < n && tj < T && k0 + k < d_h) ? __ldg(x + (size_t)tj * d_h + k0 + k) : 0.f;
                }
                __syncthreads();
#pragma unroll 4
                for (int k = 0; k < kF32Tile; ++k) {
                    const float xv = sx[lane][k];
#pragma unroll
                    for (int u = 0; u < 8; ++u) acc[u] = fmaf(sw[warp * 8 + u][k], xv, acc[u]);
                }
            }
            if (lane < n) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int r = r0 + warp * 8 + u;
                    if (r >= d_e) break;
                    const float z = b_in != nullptr ? acc[u] + __ldg(b_in + (size_t)e * d_e + r) : acc[u];
                    const float act = g * (z / (1.0f + expf(-z)));
                    hbuf[((size_t)p * n + lane) * d_e + r] = (live && ((bits >> lane) & 1u)) ? act : 0.f;
                }
            }
        }
    }
}

__global__ void __launch_bounds__(kF32Threads) expert_out_f32_kernel(
    const float* __restrict__ W_out, const float* __restrict__ b_out, const float* __restrict__ gates,
    const uint32_t* __restrict__ tmask, const int32_t* __restrict__ counts,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ pair_ce,
    const float* __restrict__ hbuf, const Ctl* ctl, int T, int d_h, int E, int d_e, int n,
    float* __restrict__ y) {
    if (__ldcg(&ctl->status) != 0) return;
    __shared__ float sw[kF32Tile][kF32Tile + 1];   // [row i][q]
    __shared__ float sh[32][kF32Tile + 1];         // [token][q]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.y;
    const int i0 = blockIdx.x * kF32Tile;
    const int cnt = counts[c], off = offsets[c];
    const int t0 = c * n, nt = min(n, T - t0);
    float acc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) acc[u] = 0.f;
    for (int s = 0; s < cnt; ++s) {
        const int e = pair_ce[off + s] & 255;
        const float* hp = hbuf + (size_t)(off + s) * n * d_e;
        for (int q0 = 0; q0 < d_e; q0 += kF32Tile) {
            __syncthreads();
            for (int i = threadIdx.x; i < kF32Tile * kF32Tile; i += kF32Threads) {
                const int r = i / kF32Tile, q = i % kF32Tile;
                sw[r][q] = (i0 + r < d_h && q0 + q < d_e)
                               ? __ldg(W_out + ((size_t)e * d_h + i0 + r) * d_e + q0 + q) : 0.f;
            }
            for (int i = threadIdx.x; i < 32 * kF32Tile; i += kF32Threads) {
                const int j = i / kF32Tile, q = i % kF32Tile;
                sh[j][q] = (j < nt && q0 + q < d_e) ? hp[(size_t)j * d_e + q0 + q] : 0.f;
            }
            __syncthreads();
#pragma unroll 4
            for (int q = 0; q < kF32Tile; ++q) {
                const float hv = sh[lane][q];
#pragma unroll
                for (int u = 0; u < 8; ++u) acc[u] = fmaf(sw[warp * 8 + u][q], hv, acc[u]);
            }
        }
    }
    if (b_out != nullptr) {
        // the gated fc2 biases of the experts this lane's token activates
        for (int s = 0; s < cnt; ++s) {
            const int e = pair_ce[off + s] & 255;
            const bool keep = lane < nt && ((tmask[(size_t)c * E + e] >> lane) & 1u);
            const float g = keep ? gates[(size_t)(t0 + lane) * E + e] : 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + warp * 8 + u;
                if (i < d_h) acc[u] = fmaf(g, __ldg(b_out + (size_t)e * d_h + i), acc[u]);
            }
        }
    }
    if (lane < nt) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + warp * 8 + u;
            if (i < d_h) y[(size_t)(t0 + lane) * d_h + i] = acc[u];
        }
    }
}

cudaError_t launch_forward_f32(const float* x, const float* gates, const float* W_in,
                               const float* W_out, const float* b_in, const float* b_out,
                               const int32_t* counts, const int32_t* offsets,
                               const int32_t* pair_ce, const uint32_t* tmask, const Ctl* ctl,
                               float* hbuf, int T, int d_h, int E, int d_e, int n, float* y,
                               int num_sms, cudaStream_t s) {
    const int C = (T + n - 1) / n;
    if (C == 0) return cudaSuccess;
    if (C > 65535) return cudaErrorInvalidValue;
    const long long pmax = (long long)C * E;
    const int gridA = (int)(pmax < 8LL * num_sms ? pmax : 8LL * num_sms);
    expert_in_f32_kernel<<<gridA, kF32Threads, 0, s>>>(x, gates, W_in, b_in, offsets, pair_ce, tmask, ctl, T,
                                                       d_h, E, d_e, n, C, hbuf);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    dim3 gridB((d_h + kF32Tile - 1) / kF32Tile, C);
    expert_out_f32_kernel<<<gridB, kF32Threads, 0, s>>>(W_out, b_out, gates, tmask, counts, offsets, pair_ce,
                                                        hbuf, ctl, T, d_h, E, d_e, n, y);
    return cudaGetLastError();
}

}  // namespace bffn
