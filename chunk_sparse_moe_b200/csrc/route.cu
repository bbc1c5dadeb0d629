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

// The cluster's KS partial logit tiles [TOK][EP] (one per block, in shared
// memory, complete: the caller has passed a cluster barrier) become gates: block
// r takes tokens r*TOK/KS .. (r+1)*TOK/KS - 1, one warp per token; logit = sum over
// ranks 0..KS-1 of their partials (+ b_r), then ReLU, the mean of squares over E
// and the scale.
template <int EP, int TOK = kRtTok>
__device__ __forceinline__ void route_finish(const float* part, int KS, int r, int t0, int Ttok, int E,
                                             const float* __restrict__ b_r, const float* __restrict__ gamma,
                                             float eps, float* __restrict__ gates) {
    constexpr int NJ = EP / 32;   // experts per lane
    const int tid = threadIdx.x;

    const int tpb = TOK / KS;
    const int warp = tid >> 5, lane = tid & 31;
    const uint32_t part_u32 = smem_u32(part);
    for (int tt = warp; tt < tpb; tt += (int)(blockDim.x / 32)) {
        const int tl = r * tpb + tt, gt = t0 + tl;
        float lg[NJ];   // this lane's experts: lane + 32*j
        float ss = 0.f;
        // all of this lane's remote partials are requested before the first is
        // added (the ranks' partials were written before the cluster barrier)
        float pv[NJ][kRtMaxKS];
#pragma unroll
        for (int j = 0; j < NJ; ++j)
#pragma unroll
            for (int q = 0; q < kRtMaxKS; ++q) {
                pv[j][q] = 0.f;
                if (q < KS) {
                    const uint32_t ra = mapa_shared(part_u32 + (uint32_t)((tl * EP + lane + 32 * j) * 4), (uint32_t)q);
                    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(pv[j][q]) : "r"(ra));
                }
            }
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
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
            for (int j = 0; j < NJ; ++j) {
                const int e = lane + 32 * j;
                if (e < E) gates[(size_t)gt * E + e] = lg[j] > 0.f ? gamma[e] * lg[j] / denom : 0.f;
            }
        }
    }
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
    route_finish<EP>(part, KS, r, t0, Ttok, E, b_r, gamma, eps, gates);
    cluster_barrier_sync();   // no block leaves while a peer may still read its partials
}

// ---------------------------------------------------------------------------
// bf16 with d_h % 256 == 0: the same cluster split, the products on the tensor
// cores.  A block's slice of d_h goes through in groups of 256 k: one TMA box
// per 128-expert tile of W_r ({64, 128, 4}: 64 KB) and one for x ({64, 32, 4}:
// 16 KB), each landing as four 128-byte-swizzled k-blocks; then 16 MMAs per
// expert tile (experts as M = 128, the 32 tokens as N, K = 16), accumulating in
// TMEM.  Experts past E and tokens past T are zeros from the boxes' out-of-range
// fill.  The accumulators come back with tcgen05.ld into the partial tile, and
// route_finish adds the ranks' tiles as in the CUDA-core kernel.  Every wait is
// bounded; a block that runs out writes NaN partials, so the gates it feeds
// come out NaN rather than wrong-but-plausible.
constexpr int kRqThreads = 128;
constexpr int kRqKg = 256;                   // k per group
constexpr uint64_t kRqWaitNs = 2000000000ull;

// TOK tokens per cluster: 32 for short inputs (a decode step), 128 for long ones,
// where the W_r tiles are then reused over four times as many tokens and the grid
// has a quarter of the clusters (one wave at 4096 tokens).
template <int ET, int TOK>
constexpr size_t route_tc_smem_bytes() {
    return 1024 + (size_t)ET * 65536 + (size_t)TOK * 512 + sizeof(float) * TOK * 128 * ET;
}

__device__ __forceinline__ bool rq_wait(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > kRqWaitNs) return false;
    return true;
}

template <int ET, int TOK>
__global__ void __launch_bounds__(kRqThreads, 1) route_tc_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
    const float* __restrict__ b_r, const float* __restrict__ gamma, float eps, int Ttok, int E, int KS,
    int slice, float* __restrict__ gates) {
    constexpr int EP = 128 * ET;
    constexpr uint32_t kCols = TOK * ET;  // one TOK-column accumulator per expert tile (a power of 2)
    constexpr int kXBytes = TOK * 512;    // x box: 4 k-blocks of TOK rows x 128 B
    extern __shared__ uint8_t rq_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(rq_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* wsm = sm;                                   // [ET][4 k-blocks][128 rows x 128 B]
    uint8_t* xsm = sm + ET * 65536;                      // [4 k-blocks][TOK rows x 128 B]
    float* part = reinterpret_cast<float*>(xsm + kXBytes);  // [TOK][EP]
    __shared__ __align__(8) uint64_t full, mma_bar;
    __shared__ uint32_t tmem_base;
    __shared__ int ok_s;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * TOK;
    const int r = (int)cluster_ctarank();
    if (threadIdx.x == 0) {
        mbar_init(&full, 1);
        mbar_init(&mma_bar, 1);
        fence_mbar_init();
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_w);
        ok_s = 1;
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, kCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    griddep_launch_dependents();
    const uint32_t tmem = tmem_base;
    if (threadIdx.x == 0) {
        const uint32_t idesc = idesc_bf16_f32(128, TOK);
        const uint64_t pol = policy_evict_last();
        const uint64_t dw = sw128_kmajor_desc(smem_u32(wsm)), dx = sw128_kmajor_desc(smem_u32(xsm));
        bool ok = true;
        const int ng = slice / kRqKg;
        for (int g = 0; g < ng && ok; ++g) {
            const int kb0 = (r * slice + g * kRqKg) / 64;
            mbar_arrive_expect_tx(&full, (uint32_t)(ET * 65536 + kXBytes));
#pragma unroll
            for (int et = 0; et < ET; ++et) tma_load_3d(wsm + et * 65536, &tm_w, &full, 0, et * 128, kb0, pol);
            tma_load_3d(xsm, &tm_x, &full, 0, t0, kb0, pol);
            ok = rq_wait(&full, (uint32_t)(g & 1));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int et = 0; et < ET; ++et)
#pragma unroll
                for (int kb = 0; kb < 4; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(tmem + (uint32_t)(TOK * et),
                                  dw + (uint64_t)((et * 65536 + kb * 16384 + kk * 32) >> 4),
                                  dx + (uint64_t)((kb * TOK * 128 + kk * 32) >> 4), idesc,
                                  (g > 0 || kb > 0 || kk > 0) ? 1u : 0u);
            umma_commit(&mma_bar);
            // the buffers are reloaded (next group) or the accumulators read only
            // once these MMAs are done
            ok = rq_wait(&mma_bar, (uint32_t)(g & 1));
        }
        if (!ok) {
            ok_s = 0;
            // give copies still in flight a bounded chance to land before leaving
            rq_wait(&full, 0u);
            rq_wait(&full, 1u);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool ok = ok_s != 0;
    // accumulator row = TMEM lane = expert (warp w holds experts 32w .. 32w+31 of each tile)
#pragma unroll
    for (int et = 0; et < ET; ++et)
#pragma unroll 1
        for (int c0 = 0; c0 < TOK; c0 += 32) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)(TOK * et + c0), v);
            tmem_ld_wait();
            const int e = 128 * et + 32 * warp + lane;
#pragma unroll
            for (int t = 0; t < 32; ++t)
                part[(c0 + t) * EP + e] = ok ? __uint_as_float(v[t]) : __int_as_float(0x7fc00000);
        }
    tc_fence_before();
    cluster_barrier_sync();   // every block's partials are written
    route_finish<EP, TOK>(part, KS, r, t0, Ttok, E, b_r, gamma, eps, gates);
    cluster_barrier_sync();   // no block leaves while a peer may still read its partials
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kCols);
    }
}

template <int ET, int TOK>
static cudaError_t launch_route_tc(const __nv_bfloat16* x, const __nv_bfloat16* W_r, const float* b_r,
                                   const float* gamma, float eps, int Ttok, int d_h, int E, int KS, float* gates,
                                   cudaStream_t s) {
    CUtensorMap mx, mw;
    if (!make_map_kblocks(&mx, x, (uint64_t)d_h, (uint64_t)Ttok, TOK, 4) ||
        !make_map_kblocks(&mw, W_r, (uint64_t)d_h, (uint64_t)E, 128, 4))
        return cudaErrorInvalidValue;
    const size_t smem = route_tc_smem_bytes<ET, TOK>();
    cudaError_t err =
        cudaFuncSetAttribute(route_tc_kernel<ET, TOK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((Ttok + TOK - 1) / TOK, KS, 1);
    cfg.blockDim = dim3(kRqThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = KS;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, route_tc_kernel<ET, TOK>, mx, mw, b_r, gamma, eps, Ttok, E, KS, d_h / KS,
                              gates);
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
    if (bf16 && d_h % kRqKg == 0 && E <= 256) {
        // tensor cores: KS slices of whole 256-k groups; long inputs (E <= 128)
        // take 128 tokens per cluster of at most 4 blocks
        const auto* xb = static_cast<const __nv_bfloat16*>(x);
        const auto* wb = static_cast<const __nv_bfloat16*>(W_r);
        if (T >= 1024 && E <= 128) {
            int KS = 4;
            while (KS > 1 && d_h % (kRqKg * KS) != 0) KS /= 2;
            return launch_route_tc<1, 128>(xb, wb, b_r, gamma, eps, T, d_h, E, KS, gates, s);
        }
        int KS = kRtMaxKS;
        while (KS > 1 && d_h % (kRqKg * KS) != 0) KS /= 2;
        return E <= 128 ? launch_route_tc<1, kRtTok>(xb, wb, b_r, gamma, eps, T, d_h, E, KS, gates, s)
                        : launch_route_tc<2, kRtTok>(xb, wb, b_r, gamma, eps, T, d_h, E, KS, gates, s);
    }
    if (bf16)
        return launch_route_t(static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(W_r), b_r,
                              gamma, eps, T, d_h, E, gates, s);
    return launch_route_t(static_cast<const float*>(x), static_cast<const float*>(W_r), b_r, gamma, eps, T, d_h,
                          E, gates, s);
}

}  // namespace bffn
