// route.cu -- the router g = RMSNorm(ReLU(W_r x + b_r)) over the expert axis.
//
// Pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device
// Deployment", Architecture Overview (Router Module: linear transformation,
// ReLU, RMSNorm) and Router Architecture Setup (nn.Linear(hidden, E) without
// bias, nn.RMSNorm(E)); "BlockFFN: Towards End-Side Acceleration-Friendly
// Mixture-of-Experts with Chunk-Level Activation Sparsity", Abstract.
//
// A block handles kTok tokens.  Each warp computes whole logits (one token, one
// expert): lanes stride over d_h with 16-byte vector loads, accumulate in fp32
// and reduce with a fixed butterfly, so the result does not depend on timing.
// The block's logits stay in shared memory; one warp per token then applies
// ReLU, the mean of squares over E and the scale, and writes the gates row.
// The router reads x once (its bytes dominate: d_h*T elements against E*d_h of
// W_r, which stays in L2).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"

namespace bffn {

constexpr int kRouteTok = 8;
constexpr int kRouteThreads = 256;

__device__ __forceinline__ float warp_sum(float v) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float dot_row(const float* __restrict__ a, const float* __restrict__ b,
                                         int d_h, int lane) {
    float acc = 0.f;
    if ((d_h & 3) == 0) {
        const float4* a4 = reinterpret_cast<const float4*>(a);
        const float4* b4 = reinterpret_cast<const float4*>(b);
        for (int k = lane; k < d_h / 4; k += 32) {
            const float4 u = __ldg(a4 + k), w = __ldg(b4 + k);
            acc = fmaf(u.x, w.x, acc);
            acc = fmaf(u.y, w.y, acc);
            acc = fmaf(u.z, w.z, acc);
            acc = fmaf(u.w, w.w, acc);
        }
    } else {
        for (int k = lane; k < d_h; k += 32) acc = fmaf(__ldg(a + k), __ldg(b + k), acc);
    }
    return warp_sum(acc);
}

__device__ __forceinline__ float dot_row(const __nv_bfloat16* __restrict__ a,
                                         const __nv_bfloat16* __restrict__ b, int d_h, int lane) {
    // d_h % 8 == 0 (checked on the host): 8 bf16 per 16-byte load
    float acc = 0.f;
    const uint4* a4 = reinterpret_cast<const uint4*>(a);
    const uint4* b4 = reinterpret_cast<const uint4*>(b);
    for (int k = lane; k < d_h / 8; k += 32) {
        const uint4 u = __ldg(a4 + k), w = __ldg(b4 + k);
        const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(&u);
        const __nv_bfloat162* w2 = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 uf = __bfloat1622float2(u2[q]), wf = __bfloat1622float2(w2[q]);
            acc = fmaf(uf.x, wf.x, acc);
            acc = fmaf(uf.y, wf.y, acc);
        }
    }
    return warp_sum(acc);
}

template <typename T>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(
    const T* __restrict__ x, const T* __restrict__ W_r, const float* __restrict__ b_r,
    const float* __restrict__ gamma, float eps, int Ttok, int d_h, int E, float* __restrict__ gates) {
    extern __shared__ float s_logit[];  // [kRouteTok][E]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = kRouteThreads / 32;
    const int t0 = blockIdx.x * kRouteTok;
    const int ntok = min(kRouteTok, Ttok - t0);
    for (int w = warp; w < ntok * E; w += nwarps) {
        const int tt = w / E, e = w % E;
        float s = dot_row(x + (size_t)(t0 + tt) * d_h, W_r + (size_t)e * d_h, d_h, lane);
        if (b_r != nullptr) s += b_r[e];
        if (lane == 0) s_logit[tt * E + e] = s;
    }
    __syncthreads();
    for (int tt = warp; tt < ntok; tt += nwarps) {
        float ss = 0.f;
        for (int e = lane; e < E; e += 32) {
            const float r = fmaxf(s_logit[tt * E + e], 0.f);
            ss = fmaf(r, r, ss);
        }
        ss = warp_sum(ss);
        const float denom = sqrtf(ss / (float)E + eps);
        for (int e = lane; e < E; e += 32) {
            const float r = fmaxf(s_logit[tt * E + e], 0.f);
            gates[(size_t)(t0 + tt) * E + e] = r > 0.f ? gamma[e] * r / denom : 0.f;
        }
    }
}

cudaError_t launch_route(const void* x, const void* W_r, const float* b_r, const float* gamma,
                         float eps, int T, int d_h, int E, bool bf16, float* gates,
                         cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const int blocks = (T + kRouteTok - 1) / kRouteTok;
    const size_t smem = sizeof(float) * kRouteTok * E;
    if (bf16) {
        route_kernel<__nv_bfloat16><<<blocks, kRouteThreads, smem, s>>>(
            static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(W_r), b_r,
            gamma, eps, T, d_h, E, gates);
    } else {
        route_kernel<float><<<blocks, kRouteThreads, smem, s>>>(
            static_cast<const float*>(x), static_cast<const float*>(W_r), b_r, gamma, eps, T, d_h,
            E, gates);
    }
    return cudaGetLastError();
}

}  // namespace bffn
