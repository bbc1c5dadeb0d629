// route.cu -- the router g = RMSNorm(ReLU(W_r x + b_r)) over the expert axis.
//
// Pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device
// Deployment", Architecture Overview (Router Module: linear transformation,
// ReLU, RMSNorm) and Router Architecture Setup (nn.Linear(hidden, E) without
// bias, nn.RMSNorm(E)); "BlockFFN: Towards End-Side Acceleration-Friendly
// Mixture-of-Experts with Chunk-Level Activation Sparsity", Abstract.
//
// A cluster of KS blocks owns 32 tokens and every expert (E <= 256); block r of
// the cluster multiplies the r-th slice of d_h.  bf16: the block's whole slice
// of x and W_r (up to 256 k at a time) comes in with one burst of 16-byte
// asynchronous copies, so its global latency is paid once, then 32-wide
// k-chunks are widened to fp32 and transposed to k-major in shared memory; fp32
// inputs are staged chunk by chunk.  Each thread keeps a 2-token x
// (4·EV)-expert tile of fp32 sums, k ascending (a warp spans 32 tokens and 8
// experts, so its shared-memory reads are one broadcast wavefront each).  The KS
// partial logit tiles are then added in rank order, through distributed shared
// memory, by the block that owns each token (32/KS tokens per block), which also
// applies the bias, ReLU, the mean of squares over E (a fixed lane-strided
// order and butterfly) and the scale, and writes the gates row.  Every sum has a
// fixed order, so the gates do not depend on timing.  At a decode step's 32
// tokens the whole d_h is spread over 8 SMs.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "common.cuh"
#include "launch.h"

namespace bffn {

constexpr int kRtTok = 32;        // tokens per cluster
constexpr int kRtThreads = 256;
constexpr int kRtKc = 32;         // k-chunk staged in shared memory
constexpr int kRtMaxKS = 8;       // blocks per cluster (slices of d_h)
constexpr int kRtSck = 256;       // k per burst of asynchronous copies (bf16)
constexpr int kRtRaw = kRtSck + 8;  // bf16 row stride of the raw staging (16-byte multiple)

__device__ __forceinline__ float warp_sum(float v) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// fp32 inputs: stage one k-chunk, one element per thread and step, any d_h
// (out of range: 0).
__device__ __forceinline__ void stage_chunk(const float* __restrict__ x, const float* __restrict__ W_r, float* xs,
                                            float* ws, int t0, int Ttok, int d_h, int E, int EP, int k0, int kend,
                                            int tid) {
    for (int q = tid; q < kRtKc * kRtTok; q += kRtThreads) {
        const int t = q / kRtKc, k = q % kRtKc;
        const int gt = t0 + t, gk = k0 + k;
        xs[k * kRtTok + t] = (gt < Ttok && gk < kend) ? __ldg(x + (size_t)gt * d_h + gk) : 0.f;
    }
    for (int q = tid; q < kRtKc * EP; q += kRtThreads) {
        const int e = q / kRtKc, k = q % kRtKc;
        const int gk = k0 + k;
        ws[k * EP + e] = (e < E && gk < kend) ? __ldg(W_r + (size_t)e * d_h + gk) : 0.f;
    }
}

// shared memory: xs [kRtKc][kRtTok], ws [kRtKc][64*EV], part [kRtTok][64*EV] (fp32),
// then for bf16 the raw staging xr [kRtTok][kRtRaw], wr [64*EV][kRtRaw] (bf16)
template <int EV, bool BF16>
constexpr size_t route_smem_bytes() {
    return sizeof(float) * ((size_t)kRtKc * kRtTok + (size_t)kRtKc * 64 * EV + (size_t)kRtTok * 64 * EV) +
           (BF16 ? sizeof(__nv_bfloat16) * (size_t)(kRtTok + 64 * EV) * kRtRaw : 0);
}

template <typename T, int EV>
__global__ void __launch_bounds__(kRtThreads) route_kernel(
    const T* __restrict__ x, const T* __restrict__ W_r, const float* __restrict__ b_r,
    const float* __restrict__ gamma, float eps, int Ttok, int d_h, int E, int KS, int slice,
    float* __restrict__ gates) {
    constexpr int EP = 64 * EV;                 // experts held per block (E padded)
    extern __shared__ float smem_f[];
    float* xs = smem_f;                         // [kRtKc][kRtTok]
    float* ws = xs + kRtKc * kRtTok;            // [kRtKc][EP]
    float* part = ws + kRtKc * EP;              // [kRtTok][EP]
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;     // tokens 2*tx, 2*tx + 1; experts 4*ty + 64*v .. +3
    const int t0 = blockIdx.x * kRtTok;
    const int r = (int)cluster_ctarank();       // = blockIdx.y: this block's slice of d_h
    const int kbeg = min(d_h, r * slice), kend = min(d_h, kbeg + slice);
    // a kernel launched as this one's programmatic dependent (the forward) may
    // be scheduled now; it waits for this grid to complete before reading gates
    griddep_launch_dependents();

    float acc[2][4 * EV];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4 * EV; ++j) acc[i][j] = 0.f;

    // one 32-wide k-chunk from xs / ws into the accumulators
    auto mma_chunk = [&]() {
#pragma unroll 4
        for (int k = 0; k < kRtKc; ++k) {
            const float2 xv = *reinterpret_cast<const float2*>(xs + k * kRtTok + 2 * tx);
#pragma unroll
            for (int v = 0; v < EV; ++v) {
                const float4 wv = *reinterpret_cast<const float4*>(ws + k * EP + 64 * v + 4 * ty);
                const float w4[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[0][4 * v + j] = fmaf(xv.x, w4[j], acc[0][4 * v + j]);
                    acc[1][4 * v + j] = fmaf(xv.y, w4[j], acc[1][4 * v + j]);
                }
            }
        }
    };

    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        // d_h % 64 == 0 (host check), so every bound below is a multiple of 32
        __nv_bfloat16* xr = reinterpret_cast<__nv_bfloat16*>(part + kRtTok * EP);   // [kRtTok][kRtRaw]
        __nv_bfloat16* wr = xr + kRtTok * kRtRaw;                                     // [EP][kRtRaw]
        for (int s0 = kbeg; s0 < kend; s0 += kRtSck) {
            const int sk = min(kRtSck, kend - s0), p8 = sk / 8;
            __syncthreads();   // the previous burst is consumed
            for (int q = tid; q < kRtTok * p8; q += kRtThreads) {
                const int t = q / p8, c = q % p8;
                const bool in = t0 + t < Ttok;
                cp_async_16_zfill(xr + t * kRtRaw + c * 8, in ? x + (size_t)(t0 + t) * d_h + s0 + c * 8 : x,
                                  in ? 16u : 0u);
            }
            for (int q = tid; q < EP * p8; q += kRtThreads) {
                const int e = q / p8, c = q % p8;
                const bool in = e < E;
                cp_async_16_zfill(wr + e * kRtRaw + c * 8, in ? W_r + (size_t)e * d_h + s0 + c * 8 : W_r,
                                  in ? 16u : 0u);
            }
            cp_async_wait_all();
            for (int c0 = 0; c0 < sk; c0 += kRtKc) {
                __syncthreads();   // the burst has landed / the previous chunk is consumed
                for (int q = tid; q < kRtKc * kRtTok; q += kRtThreads) {
                    const int t = q % kRtTok, k = q / kRtTok;
                    xs[k * kRtTok + t] = __bfloat162float(xr[t * kRtRaw + c0 + k]);
                }
                for (int q = tid; q < kRtKc * EP; q += kRtThreads) {
                    const int e = q % EP, k = q / EP;
                    ws[k * EP + e] = __bfloat162float(wr[e * kRtRaw + c0 + k]);
                }
                __syncthreads();
                mma_chunk();
            }
        }
    } else {
        for (int k0 = kbeg; k0 < kend; k0 += kRtKc) {
            __syncthreads();   // the previous chunk is consumed
            stage_chunk(x, W_r, xs, ws, t0, Ttok, d_h, E, EP, k0, kend, tid);
            __syncthreads();
            mma_chunk();
        }
    }
    // this block's partial logits of the cluster's 32 tokens
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int v = 0; v < EV; ++v)
            *reinterpret_cast<float4*>(part + (2 * tx + i) * EP + 64 * v + 4 * ty) =
                make_float4(acc[i][4 * v], acc[i][4 * v + 1], acc[i][4 * v + 2], acc[i][4 * v + 3]);
    cluster_barrier_sync();   // every block's partials are written

    // block r finishes tokens r*TPB .. r*TPB + TPB - 1 of the cluster's 32, one warp
    // per token: logit = sum over ranks 0..KS-1 of their partials (+ b_r)
    const int tpb = kRtTok / KS;
    const int warp = tid >> 5, lane = tid & 31;
    const uint32_t part_u32 = smem_u32(part);
    for (int tt = warp; tt < tpb; tt += kRtThreads / 32) {
        const int tl = r * tpb + tt, gt = t0 + tl;
        float lg[EV * 2];   // this lane's experts: lane + 32*j
        float ss = 0.f;
        // all of this lane's remote partials are requested before the first is
        // added (the ranks' partials were written before the cluster barrier)
        float pv[2 * EV][kRtMaxKS];
#pragma unroll
        for (int j = 0; j < 2 * EV; ++j)
#pragma unroll
            for (int q = 0; q < kRtMaxKS; ++q) {
                pv[j][q] = 0.f;
                if (q < KS) {
                    const uint32_t ra = mapa_shared(part_u32 + (uint32_t)((tl * EP + lane + 32 * j) * 4), (uint32_t)q);
                    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(pv[j][q]) : "r"(ra));
                }
            }
#pragma unroll
        for (int j = 0; j < 2 * EV; ++j) {
            const int e = lane + 32 * j;
            float s = 0.f;
#pragma unroll
            for (int q = 0; q < kRtMaxKS; ++q)
                if (q < KS) s += pv[j][q];
            if (b_r != nullptr && e < E) s += b_r[e];
            const float rl = e < E ? fmaxf(s, 0.f) : 0.f;
            lg[j] = rl;
            ss = fmaf(rl, rl, ss);
        }
        ss = warp_sum(ss);
        const float denom = sqrtf(ss / (float)E + eps);
        if (gt < Ttok) {
#pragma unroll
            for (int j = 0; j < 2 * EV; ++j) {
                const int e = lane + 32 * j;
                if (e < E) gates[(size_t)gt * E + e] = lg[j] > 0.f ? gamma[e] * lg[j] / denom : 0.f;
            }
        }
    }
    cluster_barrier_sync();   // no block leaves while a peer may still read its partials
}

template <typename T, int EV>
static cudaError_t launch_route_ev(const T* x, const T* W_r, const float* b_r, const float* gamma, float eps,
                                   int Ttok, int d_h, int E, float* gates, cudaStream_t s) {
    // d_h in KS slices of whole k-chunks; KS divides the 32 tokens of a cluster
    int KS = d_h / 256;
    KS = KS >= kRtMaxKS ? kRtMaxKS : KS >= 4 ? 4 : KS >= 2 ? 2 : 1;
    const int chunks = (d_h + kRtKc - 1) / kRtKc;
    const int slice = ((chunks + KS - 1) / KS) * kRtKc;
    const size_t smem = route_smem_bytes<EV, std::is_same<T, __nv_bfloat16>::value>();
    cudaError_t err =
        cudaFuncSetAttribute(route_kernel<T, EV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((Ttok + kRtTok - 1) / kRtTok, KS, 1);
    cfg.blockDim = dim3(kRtThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = KS;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, route_kernel<T, EV>, x, W_r, b_r, gamma, eps, Ttok, d_h, E, KS, slice, gates);
}

template <typename T>
static cudaError_t launch_route_t(const T* x, const T* W_r, const float* b_r, const float* gamma, float eps,
                                  int Ttok, int d_h, int E, float* gates, cudaStream_t s) {
    if (E <= 64) return launch_route_ev<T, 1>(x, W_r, b_r, gamma, eps, Ttok, d_h, E, gates, s);
    if (E <= 128) return launch_route_ev<T, 2>(x, W_r, b_r, gamma, eps, Ttok, d_h, E, gates, s);
    return launch_route_ev<T, 4>(x, W_r, b_r, gamma, eps, Ttok, d_h, E, gates, s);
}

cudaError_t launch_route(const void* x, const void* W_r, const float* b_r, const float* gamma,
                         float eps, int T, int d_h, int E, bool bf16, float* gates,
                         cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    if (bf16)
        return launch_route_t(static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(W_r), b_r,
                              gamma, eps, T, d_h, E, gates, s);
    return launch_route_t(static_cast<const float*>(x), static_cast<const float*>(W_r), b_r, gamma, eps, T, d_h,
                          E, gates, s);
}

}  // namespace bffn
