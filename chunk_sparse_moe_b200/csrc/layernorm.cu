// layernorm.cu -- the layer's closing step: out = LayerNorm(y + x) over d_h.
//
// Pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device
// Deployment", Full BlockFFN Layer with Combined Losses (the layer adds its
// input to the expert sum and normalises the result with nn.LayerNorm over the
// hidden dimension: per-feature scale and shift, population variance).
//
// One block per token row (ln_beta may be null: no shift).  v = y + x in fp32; each thread walks k = tid,
// tid + 256, ... in ascending order, the 256 partial sums meet in a fixed tree
// (a warp butterfly, then the 8 warps' sums in warp order), so the statistics do
// not depend on timing.  The variance is a second pass around the mean; a third
// pass writes the row, reading each element before writing it, so out may alias
// y or x.  The row is HBM/L2-bound and tiny next to the layer (3 * d_h elements).
// Launched as a programmatic dependent of the previous kernel on the stream (the
// forward that produced y): it waits for that kernel before reading anything.
// Rows that fit the registers take the one-pass variant below.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"

namespace bffn {

constexpr int kLnThreads = 256;

__device__ __forceinline__ float ln_f32(float v) { return v; }
__device__ __forceinline__ float ln_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void ln_store(float* p, float v) { *p = v; }
__device__ __forceinline__ void ln_store(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// the block's sum of one value per thread, in a fixed order; every thread gets it
__device__ __forceinline__ float ln_block_sum(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kLnThreads / 32; ++w) s += red[w];
    __syncthreads();   // red is reused by the next sum
    return s;
}

template <typename T>
__global__ void __launch_bounds__(kLnThreads) residual_layernorm_kernel(
    const T* __restrict__ y, const T* __restrict__ x, const float* __restrict__ ln_gamma,
    const float* __restrict__ ln_beta, float eps, int d_h, T* out) {
    __shared__ float red[kLnThreads / 32];
    griddep_wait();
    griddep_launch_dependents();
    const size_t row = (size_t)blockIdx.x * d_h;
    const T* yr = y + row;
    const T* xr = x + row;
    T* o = out + row;
    float s = 0.f;
    for (int k = threadIdx.x; k < d_h; k += kLnThreads) s += ln_f32(yr[k]) + ln_f32(xr[k]);
    const float mu = ln_block_sum(s, red) / (float)d_h;
    float q = 0.f;
    for (int k = threadIdx.x; k < d_h; k += kLnThreads) {
        const float dv = (ln_f32(yr[k]) + ln_f32(xr[k])) - mu;
        q = fmaf(dv, dv, q);
    }
    const float var = ln_block_sum(q, red) / (float)d_h;
    const float rstd = 1.0f / sqrtf(var + eps);
    for (int k = threadIdx.x; k < d_h; k += kLnThreads) {
        const float v = ln_f32(yr[k]) + ln_f32(xr[k]);
        ln_store(o + k, ln_gamma[k] * ((v - mu) * rstd) + (ln_beta != nullptr ? ln_beta[k] : 0.f));
    }
}

// The same, one pass over memory: each thread holds up to kLnChunks 16-byte
// chunks of the row (V values each) in registers from the first read to the
// write, so the row is read once (rows of up to 256 * V * kLnChunks values with
// d_h % V == 0 and 16-byte aligned pointers; 8192 bf16 or 4096 fp32).  Thread k
// sums its chunks k, k + 256, ... in order, then the same fixed tree as above.
constexpr int kLnChunks = 4;
template <typename T> struct LnVec;
template <> struct LnVec<__nv_bfloat16> { static constexpr int V = 8; };
template <> struct LnVec<float> { static constexpr int V = 4; };

__device__ __forceinline__ void ln_load_chunk(const __nv_bfloat16* p, float (&f)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
        f[2 * i] = __low2float(h);
        f[2 * i + 1] = __high2float(h);
    }
}
__device__ __forceinline__ void ln_load_chunk(const float* p, float (&f)[4]) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    f[0] = u.x;
    f[1] = u.y;
    f[2] = u.z;
    f[3] = u.w;
}
__device__ __forceinline__ void ln_store_chunk(__nv_bfloat16* p, const float (&f)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ void ln_store_chunk(float* p, const float (&f)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
}

template <typename T>
__global__ void __launch_bounds__(kLnThreads) residual_layernorm_vec_kernel(
    const T* y, const T* x, const float* __restrict__ ln_gamma, const float* __restrict__ ln_beta, float eps,
    int d_h, T* out) {
    constexpr int V = LnVec<T>::V;
    __shared__ float red[kLnThreads / 32];
    griddep_wait();
    griddep_launch_dependents();
    const size_t row = (size_t)blockIdx.x * d_h;
    const int nch = d_h / V;
    float v[kLnChunks][V];
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < kLnChunks; ++c) {
        const int ch = threadIdx.x + c * kLnThreads;
        if (ch < nch) {
            float a[V], b[V];
            ln_load_chunk(y + row + (size_t)ch * V, a);
            ln_load_chunk(x + row + (size_t)ch * V, b);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                v[c][i] = a[i] + b[i];
                s += v[c][i];
            }
        }
    }
    const float mu = ln_block_sum(s, red) / (float)d_h;
    float q = 0.f;
#pragma unroll
    for (int c = 0; c < kLnChunks; ++c)
        if (threadIdx.x + c * kLnThreads < nch) {
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const float dv = v[c][i] - mu;
                q = fmaf(dv, dv, q);
            }
        }
    const float rstd = 1.0f / sqrtf(ln_block_sum(q, red) / (float)d_h + eps);
#pragma unroll
    for (int c = 0; c < kLnChunks; ++c) {
        const int ch = threadIdx.x + c * kLnThreads;
        if (ch < nch) {
            float o[V];
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int k = ch * V + i;
                o[i] = ln_gamma[k] * ((v[c][i] - mu) * rstd) + (ln_beta != nullptr ? ln_beta[k] : 0.f);
            }
            ln_store_chunk(out + row + (size_t)ch * V, o);
        }
    }
}

static bool ln_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaError_t launch_residual_layernorm(const void* y, const void* x, const float* ln_gamma, const float* ln_beta,
                                      float eps, int T, int d_h, bool bf16, void* out, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)T);
    cfg.blockDim = dim3(kLnThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    // may start while the forward before it finishes; it waits before reading
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int V = bf16 ? 8 : 4;
    const bool vec = d_h % V == 0 && d_h <= kLnThreads * V * kLnChunks && ln_aligned16(y) && ln_aligned16(x) &&
                     ln_aligned16(out);
    if (vec && bf16)
        return cudaLaunchKernelEx(&cfg, residual_layernorm_vec_kernel<__nv_bfloat16>,
                                  static_cast<const __nv_bfloat16*>(y), static_cast<const __nv_bfloat16*>(x),
                                  ln_gamma, ln_beta, eps, d_h, static_cast<__nv_bfloat16*>(out));
    if (vec)
        return cudaLaunchKernelEx(&cfg, residual_layernorm_vec_kernel<float>, static_cast<const float*>(y),
                                  static_cast<const float*>(x), ln_gamma, ln_beta, eps, d_h,
                                  static_cast<float*>(out));
    if (bf16)
        return cudaLaunchKernelEx(&cfg, residual_layernorm_kernel<__nv_bfloat16>,
                                  static_cast<const __nv_bfloat16*>(y), static_cast<const __nv_bfloat16*>(x),
                                  ln_gamma, ln_beta, eps, d_h, static_cast<__nv_bfloat16*>(out));
    return cudaLaunchKernelEx(&cfg, residual_layernorm_kernel<float>, static_cast<const float*>(y),
                              static_cast<const float*>(x), ln_gamma, ln_beta, eps, d_h, static_cast<float*>(out));
}

}  // namespace bffn
