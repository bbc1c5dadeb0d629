// forward_tc.cu -- union-expert forward on the sm_100a tensor cores (bf16 in,
// fp32 accumulation in TMEM), weights streamed from HBM by TMA.
//
// Pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device
// Deployment", Core Concept (the kernel computes, for n tokens at once, only the
// union of their activated experts, and masks the unneeded activations after
// computing) and Architecture Overview (non-gated MLP experts with Swish,
// d_e << d_h); the layer sums gate * expert output over the experts (Full
// BlockFFN Layer with Combined Losses).
//
// Work.  For every chunk c and every expert e of its union U_c (a "pair" p):
//   expert-in  : h^T[d_e, N]  = W_in_e[d_e, d_h] . x_c^T[d_h, N]      (A units)
//                h'[j, :]     = bit_j ? g[t,e] * Swish(h[j, :]) : 0   (epilogue)
//   expert-out : y_c^T[d_h,N] = sum_{e in U_c, ascending} W_out_e . h'_e^T  (B units)
// The weights are the MMA's M=128 operand and the chunk's tokens its N (16 or
// 32), so one tcgen05.mma is 128 x N x 16 and the weight tile is read once.
//
// Schedule.  One persistent block per SM (cooperative launch, so all blocks are
// resident).  The A work (pairs x m-tiles x 64-wide k-blocks) and the B work
// (chunks x 128-row tiles x pairs x k-blocks) are each cut into equal
// contiguous ranges of 16 KB weight tiles, one range of each per block, so
// every SM streams the same number of bytes and A tiles are requested before B
// tiles everywhere.  A unit (pair, m-tile) or B unit (chunk, row tile) split
// across blocks is reduced by the last block to arrive, summing the partials
// in block order (a fixed order: results do not depend on timing).  B tiles of
// a pair wait, with a bounded spin, on a per-unit flag that the block which
// finishes the pair's A unit sets after writing the gated activations.
//
// Roles (224 threads): warp 0 issues the weight/x TMA loads, warp 1 issues the
// MMAs (one thread), warp 2 owns TMEM and loads gated activations once their
// flag is set, warps 3-6 drain the accumulators (TMEM -> registers) and do the
// split reductions, Swish, gate, mask and stores.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace bffn {

constexpr int kStages = 10;
constexpr int kWBytes = 128 * 128;             // 128 rows x 64 bf16
constexpr int kActBytes = 32 * 128;            // up to 32 rows x 64 bf16
constexpr int kStageBytes = kWBytes + kActBytes;
constexpr int kNAcc = 4;                       // TMEM accumulators (32 columns each)
constexpr int kTmemCols = 128;
constexpr int kThreads = 224;
constexpr int kMaxE = 256;

struct TcShared {
    uint64_t full_w[kStages];    // weight (+x) tile landed
    uint64_t full_h[kStages];    // gated-activation tile landed (or A stage: no tile)
    uint64_t empty[kStages];     // MMAs reading the stage are done
    uint64_t acc_full[kNAcc];    // accumulator complete
    uint64_t acc_empty[kNAcc];   // accumulator drained
    uint64_t mma_done;
    uint32_t tmem_base;
    volatile int abort;
    uint32_t epoch;
    int P;
    int ep_wait[2];   // acc-full wait result, double-buffered by segment parity
    int ep_last;      // "this block arrived last" for the current split unit
    // single-chunk tables (fuse_union)
    int32_t s_counts[1];
    int32_t s_offsets[2];
    int32_t s_pair_ce[kMaxE];
    uint32_t s_tmask[kMaxE];
    int32_t s_elist[kMaxE];      // producer: expert ids of the current B unit
};

struct Tables {
    const int32_t* counts;
    const int32_t* offsets;
    const int32_t* pair_ce;
    const uint32_t* tmask;
};

struct Seg {
    int kind;                  // 0: expert-in (A), 1: expert-out (B)
    long long lo, hi;          // this block's tiles of the unit, [lo, hi)
    long long first, last;     // all tiles of the unit, [first, last]
    int c, e, p, mt;           // A
    int rt, cnt, off;          // B
    uint32_t unit;
};

__device__ __forceinline__ long long range_lo(long long total, int G, int i) {
    return total * i / G;
}
// the block whose range holds tile j
__device__ __forceinline__ int block_of(long long j, long long total, int G) {
    return (int)(((j + 1) * G - 1) / total);
}

struct SegIter {
    long long aLo, aHi, bLo, bHi, cur;
    int phase;
    __device__ void init(long long a0, long long a1, long long b0, long long b1) {
        aLo = a0; aHi = a1; bLo = b0; bHi = b1; cur = a0; phase = 0;
    }
    __device__ bool next(const TcArgs& a, const Tables& tb, Seg& s) {
        if (phase == 0) {
            if (cur < aHi) {
                const long long u = cur / a.KB;
                s.kind = 0;
                s.p = (int)(u / a.MT);
                s.mt = (int)(u % a.MT);
                const int ce = tb.pair_ce[s.p];
                s.c = ce >> 8;
                s.e = ce & 255;
                s.first = u * a.KB;
                s.last = s.first + a.KB - 1;
                s.unit = (uint32_t)u;
                s.lo = cur;
                s.hi = min(aHi, s.last + 1);
                cur = s.hi;
                return true;
            }
            phase = 1;
            cur = bLo;
        }
        if (phase == 1) {
            if (cur < bHi) {
                const long long per_pair = (long long)a.RT * a.KBe;
                const int q = (int)(cur / per_pair);
                const int c = tb.pair_ce[q] >> 8;
                const int off = tb.offsets[c];
                const int cnt = tb.counts[c];
                const long long base = (long long)off * per_pair;
                const long long unit_tiles = (long long)cnt * a.KBe;
                const int rt = (int)((cur - base) / unit_tiles);
                s.kind = 1;
                s.c = c;
                s.off = off;
                s.cnt = cnt;
                s.rt = rt;
                s.first = base + rt * unit_tiles;
                s.last = s.first + unit_tiles - 1;
                s.unit = (uint32_t)(c * a.RT + rt);
                s.lo = cur;
                s.hi = min(bHi, s.last + 1);
                cur = s.hi;
                return true;
            }
            phase = 2;
        }
        return false;
    }
};

__device__ __forceinline__ float swish(float z) { return z / (1.0f + __expf(-z)); }

__global__ void __launch_bounds__(kThreads, 1)
union_expert_forward_tc(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_win,
                        const __grid_constant__ CUtensorMap tm_wout,
                        const __grid_constant__ CUtensorMap tm_h, const TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    TcShared& sh = *reinterpret_cast<TcShared*>(smem + kStages * kStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, cta = blockIdx.x;
    const int N = a.N;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sh.full_w[s], 1);
            mbar_init(&sh.full_h[s], 1);
            mbar_init(&sh.empty[s], 1);
        }
        for (int s = 0; s < kNAcc; ++s) {
            mbar_init(&sh.acc_full[s], 1);
            mbar_init(&sh.acc_empty[s], 4);
        }
        mbar_init(&sh.mma_done, 1);
        fence_mbar_init();
        sh.abort = (ld_acquire_gpu(reinterpret_cast<const uint32_t*>(&a.ctl->status)) != 0);
        sh.epoch = ld_acquire_gpu(&a.ctl->epoch);
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_win);
        prefetch_tmap(&tm_wout);
        prefetch_tmap(&tm_h);
    }
    if (warp == 2) {
        tmem_alloc(&sh.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (a.fuse_union && warp == 3) {
        // union of the single chunk (c = 0), ascending, into shared memory
        int base = 0;
        const int nt = min(a.n, a.T);
        for (int g0 = 0; g0 < a.E; g0 += 32) {
            const int e = g0 + lane;
            uint32_t bits = 0u;
            if (e < a.E) {
                for (int j = 0; j < nt; ++j)
                    bits |= (__ldg(a.gates + (size_t)j * a.E + e) != 0.0f ? 1u : 0u) << j;
                sh.s_tmask[e] = bits;
            }
            const uint32_t bal = __ballot_sync(0xffffffffu, bits != 0u);
            if (bits != 0u) sh.s_pair_ce[base + __popc(bal & ((1u << lane) - 1u))] = e;
            base += __popc(bal);
        }
        if (lane == 0) {
            sh.s_counts[0] = base;
            sh.s_offsets[0] = 0;
            sh.s_offsets[1] = base;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    Tables tb;
    if (a.fuse_union) {
        tb.counts = sh.s_counts;
        tb.offsets = sh.s_offsets;
        tb.pair_ce = sh.s_pair_ce;
        tb.tmask = sh.s_tmask;
    } else {
        tb.counts = a.counts;
        tb.offsets = a.offsets;
        tb.pair_ce = a.pair_ce;
        tb.tmask = a.tmask;
    }
    const uint32_t tmem = sh.tmem_base;
    const int P = tb.offsets[a.C];
    const uint32_t stamp = sh.epoch + 1u;
    const long long NA = (long long)P * a.MT * a.KB;
    const long long NB = (long long)P * a.RT * a.KBe;
    const long long aLo = NA > 0 ? range_lo(NA, G, cta) : 0, aHi = NA > 0 ? range_lo(NA, G, cta + 1) : 0;
    const long long bLo = NB > 0 ? range_lo(NB, G, cta) : 0, bHi = NB > 0 ? range_lo(NB, G, cta + 1) : 0;
    const uint64_t limit = a.wait_ns;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer --
        const uint64_t pol_stream = policy_evict_first();
        const uint64_t pol_keep = policy_evict_last();
        SegIter it;
        it.init(aLo, aHi, bLo, bHi);
        Seg sg;
        long long i = 0;
        bool stop = sh.abort != 0;
        while (!stop && it.next(a, tb, sg)) {
            if (sg.kind == 1) {
                for (int k = lane; k < sg.cnt; k += 32) sh.s_elist[k] = tb.pair_ce[sg.off + k] & 255;
                __syncwarp();
            }
            if (lane == 0) {
                for (long long j = sg.lo; j < sg.hi; ++j, ++i) {
                    const int st = (int)(i % kStages);
                    const uint32_t ph = (uint32_t)((i / kStages) & 1);
                    if (!wait_bar(&sh.empty[st], ph ^ 1u, limit, &sh.abort, a.ctl, kWaitEmpty)) {
                        stop = true;
                        break;
                    }
                    uint8_t* w = smem + st * kStageBytes;
                    if (sg.kind == 0) {
                        const int kb = (int)(j - sg.first);
                        mbar_arrive_expect_tx(&sh.full_w[st], kWBytes + N * 128);
                        tma_load_2d(w, &tm_win, &sh.full_w[st], kb * 64, sg.e * a.d_e + sg.mt * 128,
                                    pol_stream);
                        tma_load_2d(w + kWBytes, &tm_x, &sh.full_w[st], kb * 64, sg.c * a.n,
                                    pol_keep);
                    } else {
                        const long long local = j - sg.first;
                        const int sidx = (int)(local / a.KBe), kb = (int)(local % a.KBe);
                        const int e = sh.s_elist[sidx];
                        mbar_arrive_expect_tx(&sh.full_w[st], kWBytes);
                        tma_load_2d(w, &tm_wout, &sh.full_w[st], kb * 64, e * a.d_h + sg.rt * 128,
                                    pol_stream);
                    }
                }
            }
            stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
            i = __shfl_sync(0xffffffffu, i, 0);
            __syncwarp();
        }
        if (lane == 0) {
            // let every issued copy land before the block can exit
            const long long issued = i;
            for (long long k = issued - kStages < 0 ? 0 : issued - kStages; k < issued; ++k)
                wait_bar_drain(&sh.full_w[k % kStages], (uint32_t)((k / kStages) & 1), limit, a.ctl);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer --
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(128, N);
            SegIter it;
            it.init(aLo, aHi, bLo, bHi);
            Seg sg;
            long long i = 0;
            uint32_t acc_i = 0;
            bool stop = sh.abort != 0;
            while (!stop && it.next(a, tb, sg)) {
                const int ab = (int)(acc_i % kNAcc);
                const uint32_t aph = (acc_i / kNAcc) & 1u;
                if (!wait_bar(&sh.acc_empty[ab], aph ^ 1u, limit, &sh.abort, a.ctl, kWaitAccEmpty))
                    break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(ab * 32);
                for (long long j = sg.lo; j < sg.hi; ++j, ++i) {
                    const int st = (int)(i % kStages);
                    const uint32_t ph = (uint32_t)((i / kStages) & 1);
                    if (!wait_bar(&sh.full_w[st], ph, limit, &sh.abort, a.ctl, kWaitFullW) ||
                        !wait_bar(&sh.full_h[st], ph, limit, &sh.abort, a.ctl, kWaitFullH)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t wb = smem_u32(smem + st * kStageBytes);
                    const uint32_t xb = wb + kWBytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(d, sw128_kmajor_desc(wb + kk * 32), sw128_kmajor_desc(xb + kk * 32),
                                  idesc, (j > sg.lo || kk > 0) ? 1u : 0u);
                    umma_commit(&sh.empty[st]);
                }
                if (stop) break;
                umma_commit(&sh.acc_full[ab]);
                ++acc_i;
            }
            umma_commit(&sh.mma_done);
        }
    } else if (warp == 2) {
        // ------------------------------------- gated-activation loader --
        if (lane == 0) {
            const uint64_t pol_keep = policy_evict_last();
            SegIter it;
            it.init(aLo, aHi, bLo, bHi);
            Seg sg;
            long long i = 0;
            bool stop = sh.abort != 0;
            while (!stop && it.next(a, tb, sg)) {
                for (long long j = sg.lo; j < sg.hi; ++j, ++i) {
                    const int st = (int)(i % kStages);
                    const uint32_t ph = (uint32_t)((i / kStages) & 1);
                    if (!wait_bar(&sh.empty[st], ph ^ 1u, limit, &sh.abort, a.ctl, kWaitEmpty)) {
                        stop = true;
                        break;
                    }
                    if (sg.kind == 0) {
                        mbar_arrive(&sh.full_h[st]);
                        continue;
                    }
                    const long long local = j - sg.first;
                    const int sidx = (int)(local / a.KBe), kb = (int)(local % a.KBe);
                    const int p = sg.off + sidx;
                    const uint32_t u = (uint32_t)(p * a.MT + (kb >> 1));
                    if (!wait_flag(&a.flags[u], stamp, limit, &sh.abort, a.ctl)) {
                        stop = true;
                        break;
                    }
                    fence_proxy_async_global();
                    mbar_arrive_expect_tx(&sh.full_h[st], N * 128);
                    tma_load_2d(smem + st * kStageBytes + kWBytes, &tm_h, &sh.full_h[st], kb * 64,
                                p * N, pol_keep);
                }
            }
            // drain: only B stages carry copies; A stages were completed by arrive
            const long long issued = i;
            for (long long k = issued - kStages < 0 ? 0 : issued - kStages; k < issued; ++k)
                wait_bar_drain(&sh.full_h[k % kStages], (uint32_t)((k / kStages) & 1), limit, a.ctl);
        }
    } else {
        // ------------------------------------------------ epilogue (warps 3-6) --
        const int q = warp & 3;
        const int row = q * 32 + lane;           // accumulator row = TMEM lane
        const int et = threadIdx.x - 96;         // 0..127
        if (a.fuse_union && cta == 0 && P == 0 && !sh.abort) {
            // empty union: y is all zeros
            const size_t total = (size_t)min(a.n, a.T) * a.d_h;
            for (size_t k = et; k < total; k += 128) a.y[k] = __float2bfloat16_rn(0.f);
        }
        SegIter it;
        it.init(aLo, aHi, bLo, bHi);
        Seg sg;
        uint32_t acc_i = 0;
        while (it.next(a, tb, sg)) {
            const int ab = (int)(acc_i % kNAcc);
            const uint32_t aph = (acc_i / kNAcc) & 1u;
            // one thread waits and the 128 threads take its decision together, so
            // the named barriers below always see all of them
            if (et == 0)
                sh.ep_wait[acc_i & 1u] =
                    wait_bar(&sh.acc_full[ab], aph, limit, &sh.abort, a.ctl, kWaitAccFull) ? 1 : 0;
            named_bar_sync(1, 128);
            if (!sh.ep_wait[acc_i & 1u]) break;
            tc_fence_after();
            uint32_t r[32];
            const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * 32);
            if (N == 32) tmem_ld_32x32b_x32(taddr, r);
            else tmem_ld_32x32b_x16(taddr, r);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.acc_empty[ab]);
            ++acc_i;
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = j < N ? __uint_as_float(r[j]) : 0.f;

            // split reduction across blocks, in block order
            const long long total = sg.kind == 0 ? NA : NB;
            const long long myLo = sg.kind == 0 ? aLo : bLo;
            const int q0 = block_of(sg.first, total, G), q1 = block_of(sg.last, total, G);
            if (q0 != q1) {
                // contributors: the blocks in [q0, q1] whose range is not empty (ranges
                // are empty only when there are fewer tiles than blocks)
                int ncontrib = 0;
                for (int qq = q0; qq <= q1; ++qq)
                    ncontrib += range_lo(total, G, qq + 1) > range_lo(total, G, qq) ? 1 : 0;
                float* part = sg.kind == 0 ? a.partA : a.partB;
                uint32_t* cnt = sg.kind == 0 ? a.cntA : a.cntB;
                const int myslot = myLo >= sg.first ? 0 : 1;
                float* dst = part + (size_t)(cta * 2 + myslot) * (size_t)(N * 128);
                for (int j = 0; j < N; ++j) dst[j * 128 + row] = v[j];
                __threadfence();
                named_bar_sync(1, 128);
                if (et == 0) {
                    const uint32_t old = atomicAdd(&cnt[sg.unit], 1u);
                    const int last = old == (uint32_t)(ncontrib - 1);
                    if (last) cnt[sg.unit] = 0u;
                    sh.ep_last = last;
                }
                named_bar_sync(1, 128);
                if (!sh.ep_last) continue;
                __threadfence();
                float s[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) s[j] = 0.f;
                for (int qq = q0; qq <= q1; ++qq) {
                    if (range_lo(total, G, qq + 1) == range_lo(total, G, qq)) continue;
                    if (qq == cta) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) s[j] += v[j];
                    } else {
                        const int sl = range_lo(total, G, qq) >= sg.first ? 0 : 1;
                        const float* src = part + (size_t)(qq * 2 + sl) * (size_t)(N * 128);
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (j < N) s[j] += __ldcg(src + j * 128 + row);
                    }
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = s[j];
            }

            if (sg.kind == 0) {
                // gated Swish with the post-hoc token mask -> bf16 activations
                const uint32_t bits = tb.tmask[(size_t)sg.c * a.E + sg.e];
                __nv_bfloat16* hrow = a.hbuf + (size_t)sg.p * N * a.d_e + sg.mt * 128 + row;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    if (j < N) {
                        const int t = sg.c * a.n + j;
                        float h = 0.f;
                        if (j < a.n && t < a.T && ((bits >> j) & 1u))
                            h = __ldg(a.gates + (size_t)t * a.E + sg.e) * swish(v[j]);
                        hrow[(size_t)j * a.d_e] = __float2bfloat16_rn(h);
                    }
                }
                fence_proxy_async_global();
                __threadfence();
                named_bar_sync(1, 128);
                if (et == 0 && (int)sg.unit != a.skip_flag_unit) st_release_gpu(&a.flags[sg.unit], stamp);
            } else {
                __nv_bfloat16* ycol = a.y + sg.rt * 128 + row;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int t = sg.c * a.n + j;
                    if (j < a.n && t < a.T) ycol[(size_t)t * a.d_h] = __float2bfloat16_rn(v[j]);
                }
            }
        }
    }

    // ------------------------------------------------------------ teardown --
    __syncthreads();
    if (warp == 2) {
        if (lane == 0) wait_bar_drain(&sh.mma_done, 0, limit, a.ctl);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (threadIdx.x == 0) {
        __threadfence();
        const uint32_t old = atomicAdd(&a.ctl->done, 1u);
        if (old == (uint32_t)(G - 1)) {
            a.ctl->done = 0u;
            atomicExch(&a.ctl->epoch, stamp);
        }
    }
}

size_t forward_tc_smem_bytes() { return 1024 + (size_t)kStages * kStageBytes + sizeof(TcShared); }

cudaError_t launch_forward_tc(const TcArgs& a, const CUtensorMap* maps, int grid, cudaStream_t s) {
    const size_t smem = forward_tc_smem_bytes();
    cudaError_t err = cudaFuncSetAttribute(union_expert_forward_tc,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, union_expert_forward_tc, maps[0], maps[1], maps[2], maps[3], a);
}

}  // namespace bffn
