// forward_group.cu -- the multi-chunk union-expert forward on the sm_100a tensor
// cores (bf16 in, fp32 accumulation in TMEM), expert-major over groups of chunks.
//
// Pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device
// Deployment", Core Concept (for n tokens at once only the union of their
// activated experts is computed; unneeded activations are masked after
// computing) and Architecture Overview (non-gated Swish experts, d_e << d_h);
// the layer sums gate * expert output over the experts (Full BlockFFN Layer with
// Combined Losses).
//
// Groups.  The chunks are taken NG at a time: a group is NT = NG * n consecutive
// tokens (NT <= N, the MMA's token count, 128 or 256) made of whole chunks.  The
// group's expert set is the union of its chunks' unions, ascending; each expert
// of it runs once over all NT tokens, and every token's own mask selects its
// activations afterwards.  A token whose gate is zero contributes an exact zero,
// so the result is the per-chunk union-then-mask result; each weight tile is
// read once per group instead of once per chunk, and every MMA is 128 x N x 16.
//
// Work.  For every group G and expert e of its set (a "pair" p):
//   expert-in  : h^T[d_e, N]  = W_in_e[d_e, d_h] . x_G^T[d_h, N]           (A units)
//                h'[j, :]     = bit_j ? g[t_j, e] * Swish(h[j, :] + b_in_e) : 0   (epilogue)
//   expert-out : y_G^T[d_h,N] = sum_{e in U_G, ascending} W_out_e . h'_e^T  (B units)
//                y[t, :]     += ybias[t, :]   (the gated fc2 biases, expert_bias.cu)
// bit_j is token t_j's bit in its chunk's token mask (the chunk union tables);
// the biases (the experts' nn.Linear biases, Router Architecture Setup) are
// optional.
//
// Schedule.  One persistent block per SM (cooperative launch: all resident).  The
// A work is dealt out in whole units (a pair's 128-row tile of W_in_e over all of
// d_h), an equal count per block, so h' comes straight from one accumulator.  The
// B work (groups x 128-row tiles of y x (expert, k-block)) is cut into equal
// contiguous ranges of 16 KB weight tiles, one per block; an expert-out unit split
// across blocks is finished by each contributor for its share of the rows,
// summing the partials in block order (a fixed order: results do not depend on
// timing).  A tiles come before B tiles everywhere, and an expert-out tile waits,
// with a bounded spin, until the block owning the expert-in unit it reads has
// written that unit's h'.
//
// Roles (352 threads): warp 0 issues the weight-tile TMA loads, warp 1 issues
// the MMAs (the whole warp runs the loop, one elected lane issues), warp 2 owns
// TMEM and issues the activation-tile TMA loads (x, or h' once its flag is set),
// warps 3-10 drain the accumulators (TMEM -> registers, 32 columns at a time, two
// warp groups on alternate column slices) and do the split reductions, Swish,
// gate, mask and stores.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace bffn {

namespace {

constexpr int kGrThreads = 352;               // 3 role warps + 8 epilogue warps
constexpr int kGrEpi = 256;                    // epilogue threads
constexpr int kGrWBytes = 128 * 128;            // weight tile: 128 rows x 64 bf16
constexpr int kGrMaxE = 256;
constexpr int kGrMaxContrib = 160;              // >= blocks per launch (one per SM)
constexpr int kGrSmemBudget = 200 * 1024;       // pipeline stages
// epilogue output staging: one [32 tokens][128 rows] bf16 slice (8 KB) per
// epilogue warp group
constexpr int kGrOutStageBytes = 2 * 32 * 128 * 2;

template <int N>
struct GrCfg {
    static constexpr int kActBytes = N * 128;   // activation tile: N rows x 64 bf16
    static constexpr int kStageBytes = kGrWBytes + kActBytes;
    static constexpr int kStages = kGrSmemBudget / kStageBytes;
    static constexpr int kTmemCols = 2 * N;     // two accumulators of N columns
};

template <int N>
struct GrShared {
    uint64_t full_w[GrCfg<N>::kStages];    // weight (+x) tile landed
    uint64_t full_h[GrCfg<N>::kStages];    // h' tile landed (B) or nothing to load (A)
    uint64_t empty[GrCfg<N>::kStages];     // MMAs reading the stage are done
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t mma_done;
    uint64_t a_pub;                        // this block's expert-in results are announced
    uint64_t flush_bar;                    // partial tiles landed in the idle ring (TMA bytes)
    uint32_t tmem_base;
    volatile int abort;
    int abort0;                            // abort as set before the first block barrier
    uint32_t epoch;
    int ep_wait[2];
    int ep_ok;
    int s_contrib[kGrMaxContrib];
    int32_t s_elist[kGrMaxE];              // producer: experts of the current B unit
    alignas(16) float s_gv[N];             // epilogue: the unit's gates (0 where masked)
    uint32_t s_bits[N / 32];               // epilogue: the unit's token bits
};

struct GrSeg {
    int kind;                  // 0: expert-in (A), 1: expert-out (B)
    long long lo, hi;          // this block's tiles of the unit, [lo, hi)
    long long first, last;     // all tiles of the unit, [first, last]
    int g, e, p, mt;           // A: group, expert, pair, row tile of W_in_e
    int rt, cnt, off;          // B: row tile of y, the group's union size and first pair
    uint32_t unit;
};

__device__ __forceinline__ long long gr_range_lo(long long total, int G, int i) {
    if (total < (1LL << 31) / (G + 1)) return (long long)((uint32_t)total * (uint32_t)i / (uint32_t)G);
    return total * i / G;
}
__device__ __forceinline__ int gr_block_of(long long j, long long total, int G) {
    if (total < (1LL << 31) / (G + 1)) return (int)((((uint32_t)j + 1u) * (uint32_t)G - 1u) / (uint32_t)total);
    return (int)(((j + 1) * G - 1) / total);
}

// The blocks holding tiles of a unit spanning tiles [first, last]: q0..q1 with a
// non-empty range; n of them, and the rank of `me` among them (-1 if none).
struct GrContrib {
    int q0, q1, n, rank;
};
__device__ __forceinline__ GrContrib gr_contributors(long long first, long long last, long long total, int G,
                                                     int me) {
    GrContrib c;
    c.q0 = gr_block_of(first, total, G);
    c.q1 = gr_block_of(last, total, G);
    if (total >= G) {
        c.n = c.q1 - c.q0 + 1;
        c.rank = (me >= c.q0 && me <= c.q1) ? me - c.q0 : -1;
        return c;
    }
    c.n = 0;
    c.rank = -1;
    for (int qq = c.q0; qq <= c.q1; ++qq) {
        if (gr_range_lo(total, G, qq + 1) > gr_range_lo(total, G, qq)) {
            if (qq == me) c.rank = c.n;
            ++c.n;
        }
    }
    return c;
}

struct GrIter {
    long long aLo, aHi, bLo, bHi, cur;
    int phase;
    __device__ void init(long long a0, long long a1, long long b0, long long b1) {
        aLo = a0; aHi = a1; bLo = b0; bHi = b1; cur = a0; phase = 0;
    }
    __device__ bool next(const GrArgs& a, GrSeg& s) {
        if (phase == 0) {
            if (cur < aHi) {
                const long long u = cur / a.KB;
                s.kind = 0;
                s.p = (int)(u / a.MT);
                s.mt = (int)(u % a.MT);
                const int ge = a.gpair[s.p];
                s.g = ge >> 8;
                s.e = ge & 255;
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
                const int g = a.gpair[q] >> 8;
                const int off = a.goffsets[g];
                const int cnt = a.gcounts[g];
                const long long base = (long long)off * per_pair;
                const long long unit_tiles = (long long)cnt * a.KBe;
                const int rt = (int)((cur - base) / unit_tiles);
                s.kind = 1;
                s.g = g;
                s.off = off;
                s.cnt = cnt;
                s.rt = rt;
                s.first = base + rt * unit_tiles;
                s.last = s.first + unit_tiles - 1;
                s.unit = (uint32_t)(g * a.RT + rt);
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

__device__ __forceinline__ float gr_swish(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// Timeline stamps (globaltimer, ns) of one launch, written only when a trace
// buffer is attached: per block 64 slots.
enum : int {
    kGtStart = 0, kGtPrologue = 1, kGtFirstLoad = 2, kGtLastALoad = 3, kGtLastACommit = 4,
    kGtAFlushed = 5, kGtFirstFlag = 6, kGtLastBCommit = 7, kGtEpiEnd = 8, kGtEnd = 9,
    kGtFirstAcc = 10, kGtFirstBLoad = 11, kGtLastLoad = 12, kGtADrained = 13, kGtAnnounce = 14,
    kGtFirstSlice = 15, kGtSliceBase = 16,   // 16 + 4*slice + step, first unit only (steps: TMEM read,
                                             // staged, barrier passed, stores issued)
    kGtLoopEnd = 48, kGtFlushAnnounced = 49, kGtFinBase = 50,   // 50 + 3*k + {counted, copied, summed}
    kGtSlots = 64
};
#define GR_TRACE(slot) \
    do { if (a.trace) a.trace[(size_t)blockIdx.x * kGtSlots + (slot)] = globaltimer_ns(); } while (0)

}  // namespace

template <int N>
__global__ void __launch_bounds__(kGrThreads, 1)
union_expert_group(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_win,
                   const __grid_constant__ CUtensorMap tm_wout, const __grid_constant__ CUtensorMap tm_h,
                   const __grid_constant__ CUtensorMap tm_part, const GrArgs a) {
    using Cfg = GrCfg<N>;
    constexpr int kStages = Cfg::kStages;
    constexpr int kStageBytes = Cfg::kStageBytes;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned by pointer arithmetic on the shared array itself (an
    // integer round trip would make every access through it a generic one)
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    GrShared<N>& sh = *reinterpret_cast<GrShared<N>*>(smem + kStages * kStageBytes);
    __nv_bfloat16* ostage = reinterpret_cast<__nv_bfloat16*>(
        (reinterpret_cast<uintptr_t>(&sh + 1) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, cta = blockIdx.x;

    // Set-up that touches only this block's shared memory, TMEM and the tensor
    // maps runs first; the kernel is a programmatic dependent of the group-plan
    // kernel and waits for it (griddepcontrol.wait) before reading the control
    // block, the tables or any input.
    if (threadIdx.x == 0) {
        GR_TRACE(kGtStart);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sh.full_w[s], 1);
            mbar_init(&sh.full_h[s], 1);
            mbar_init(&sh.empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sh.acc_full[s], 1);
            mbar_init(&sh.acc_empty[s], 8);   // one arrival per epilogue warp
        }
        mbar_init(&sh.mma_done, 1);
        mbar_init(&sh.a_pub, 1);
        mbar_init(&sh.flush_bar, 1);
        fence_mbar_init();
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_win);
        prefetch_tmap(&tm_wout);
        prefetch_tmap(&tm_h);
        prefetch_tmap(&tm_part);
    }
    if (warp == 2) {
        tmem_alloc(&sh.tmem_base, Cfg::kTmemCols);
        tmem_relinquish();
    }
    griddep_wait();
    if (threadIdx.x == 0) {
        griddep_launch_dependents();
        const int32_t st0 = __ldcg(&a.ctl->status);
        const unsigned long long tk = atomicAdd(&a.ctl->ticket, 1ull);   // launch index = ticket / grid
        const unsigned long long key0 = claim_shape_key(a.ctl, a.shape_key);
        const uint32_t ep0 = (uint32_t)(tk / gridDim.x);
        const bool key_ok = key0 == 0ull || key0 == a.shape_key;
        if (!key_ok) record_error(a.ctl, kErrWorkspace, kShapeKey);
        sh.abort = st0 != 0 || !key_ok;
        sh.abort0 = st0 != 0 || !key_ok;
        sh.epoch = ep0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0) GR_TRACE(kGtPrologue);

    const uint32_t tmem = sh.tmem_base;
    const int P = a.goffsets[a.NGr];
    const int par = (int)(sh.epoch & 1u);
    uint32_t* const readyA = a.readyA + (size_t)par * a.cnt_a_len;
    uint32_t* const cntB = a.cntB + (size_t)par * a.cnt_b_len;
    const long long NB = (long long)P * a.RT * a.KBe;
    // Expert-in work goes to blocks in whole units (a unit is one pair's 128-row
    // tile of W_in_e over all of d_h: KB tiles), so no expert-in result is ever
    // split and h' is written straight from the accumulator; block i takes units
    // [i*UA/G, (i+1)*UA/G).  Expert-out work is cut into equal tile ranges.
    const long long UA = (long long)P * a.MT;
    const long long aLo = UA > 0 ? gr_range_lo(UA, G, cta) * a.KB : 0;
    const long long aHi = UA > 0 ? gr_range_lo(UA, G, cta + 1) * a.KB : 0;
    const long long bLo = NB > 0 ? gr_range_lo(NB, G, cta) : 0, bHi = NB > 0 ? gr_range_lo(NB, G, cta + 1) : 0;
    // waits on other blocks run out after wait_ns; waits on this block's own
    // pipeline are downstream of those and get twice as long, so the first
    // timeout recorded names the root cause
    const uint64_t limit_peer = a.wait_ns;
    const uint64_t limit = 2 * a.wait_ns;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer --
        // Weight tiles only (the activation tiles come from warp 2: one thread
        // issues bulk copies at a bounded rate, so two issuers keep the stages
        // full).  A weight tile is read once per group that uses the expert, by
        // blocks that run at about the same time: the normal L2 policy.
        const uint64_t pol_weights = policy_evict_normal();
        GrIter it;
        it.init(aLo, aHi, bLo, bHi);
        GrSeg sg;
        long long i = 0;
        int st = 0;
        uint32_t ph = 0u;
        bool stop = sh.abort0 != 0;   // the same in all 32 lanes
        while (!stop && it.next(a, sg)) {
            if (sg.kind == 1) {
                for (int k = lane; k < sg.cnt; k += 32) sh.s_elist[k] = a.gpair[sg.off + k] & 255;
                __syncwarp();
            }
            if (lane == 0) {
                int sidx = 0, kb = 0;
                if (sg.kind == 1) {
                    const long long local = sg.lo - sg.first;
                    sidx = (int)(local / a.KBe);
                    kb = (int)(local - (long long)sidx * a.KBe);
                    // no expert-out copy is in flight while the block announces its
                    // h' (a fence waits for the block's bulk copies in flight)
                    if (sg.lo == bLo && aHi > aLo &&
                        !wait_bar(&sh.a_pub, 0u, limit, &sh.abort, a.ctl, kWaitEmpty))
                        stop = true;
                }
                for (long long j = sg.lo; j < sg.hi && !stop; ++j, ++i) {
                    if (!wait_bar(&sh.empty[st], ph ^ 1u, limit, &sh.abort, a.ctl, kWaitEmpty)) {
                        stop = true;
                        break;
                    }
                    uint8_t* w = smem + st * kStageBytes;
                    if (i == 0) GR_TRACE(kGtFirstLoad);
                    if (sg.kind == 0) {
                        GR_TRACE(kGtLastALoad);
                        const int kbA = (int)(j - sg.first);
                        mbar_arrive_expect_tx(&sh.full_w[st], kGrWBytes);
                        tma_load_2d(w, &tm_win, &sh.full_w[st], kbA * 64, sg.e * a.d_e + sg.mt * 128, pol_weights);
                    } else {
                        const int e = sh.s_elist[sidx];
                        mbar_arrive_expect_tx(&sh.full_w[st], kGrWBytes);
                        tma_load_2d(w, &tm_wout, &sh.full_w[st], kb * 64, e * a.d_h + sg.rt * 128, pol_weights);
                        if (++kb == a.KBe) {
                            kb = 0;
                            ++sidx;
                        }
                    }
                    if (++st == kStages) {
                        st = 0;
                        ph ^= 1u;
                    }
                }
            }
            stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
            i = __shfl_sync(0xffffffffu, i, 0);
            st = __shfl_sync(0xffffffffu, st, 0);
            ph = __shfl_sync(0xffffffffu, ph, 0);
            __syncwarp();
        }
        if (lane == 0) {
            GR_TRACE(kGtLastLoad);
            // let every issued copy land before the block can exit
            for (long long k = i - kStages < 0 ? 0 : i - kStages; k < i; ++k)
                wait_bar_drain(&sh.full_w[k % kStages], (uint32_t)((k / kStages) & 1), limit, a.ctl);
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer --
        const bool leader = elect_one();
        const uint32_t idesc = idesc_bf16_f32(128, N);
        const uint64_t desc0 = sw128_kmajor_desc(smem_u32(smem));
        GrIter it;
        it.init(aLo, aHi, bLo, bHi);
        GrSeg sg;
        int st = 0;
        uint32_t ph = 0u;
        uint32_t rw = 0u, rh = 0u;   // the current stage's barriers as last tested
        uint32_t acc_i = 0;
        bool stop = __shfl_sync(0xffffffffu, sh.abort, 0) != 0;
        while (!stop && it.next(a, sg)) {
            const int ab = (int)(acc_i & 1u);
            const uint32_t aph = (acc_i >> 1) & 1u;
            if (!wait_bar_warp(&sh.acc_empty[ab], aph ^ 1u, limit, &sh.abort, a.ctl, kWaitAccEmpty)) break;
            tc_fence_after();
            const uint32_t d = tmem + (uint32_t)(ab * N);
            for (long long j = sg.lo; j < sg.hi; ++j) {
                if (!__all_sync(0xffffffffu, rw & rh) &&
                    (!wait_bar_warp(&sh.full_w[st], ph, limit, &sh.abort, a.ctl, kWaitFullW) ||
                     !wait_bar_warp(&sh.full_h[st], ph, limit, &sh.abort, a.ctl, kWaitFullH))) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                const int st_n = st + 1 == kStages ? 0 : st + 1;
                const uint32_t ph_n = st + 1 == kStages ? ph ^ 1u : ph;
                rw = mbar_test_wait(&sh.full_w[st_n], ph_n);
                rh = mbar_test_wait(&sh.full_h[st_n], ph_n);
                if (leader) {
                    const uint64_t ds = desc0 + (uint64_t)(st * (kStageBytes >> 4));
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(d, ds + (uint64_t)((kk * 32) >> 4), ds + (uint64_t)((kGrWBytes + kk * 32) >> 4),
                                  idesc, (j > sg.lo || kk > 0) ? 1u : 0u);
                    umma_commit(&sh.empty[st]);
                }
                __syncwarp();
                st = st_n;
                ph = ph_n;
            }
            if (stop) break;
            if (leader) {
                umma_commit(&sh.acc_full[ab]);
                GR_TRACE(sg.kind == 0 ? kGtLastACommit : kGtLastBCommit);
            }
            __syncwarp();
            ++acc_i;
        }
        if (leader) umma_commit(&sh.mma_done);
        __syncwarp();
    } else if (warp == 2) {
        // ------------------------------------------------ activation loader --
        // An expert-in stage's activations are the group's x tile (read once per
        // expert of the group's set: kept in L2).  For an expert-out tile, lane 0
        // waits (bounded) until every contributor of the expert-in unit holding
        // the tile's 64 columns of h' has written its rows, then moves the
        // [N x 64] slice by TMA (it lands in the 128-byte-swizzled layout the MMA
        // reads).
        GrIter it;
        it.init(aLo, aHi, bLo, bHi);
        GrSeg sg;
        int st = 0;
        uint32_t ph = 0u;
        long long i = 0, nB = 0;
        bool stop = sh.abort != 0;
        uint32_t last_u = 0xffffffffu;
        const uint64_t pol = policy_evict_last();   // x: once per expert; h': once per row tile of y
        if (lane == 0) {
            while (!stop && it.next(a, sg)) {
                int sidx = 0, kb = 0;
                if (sg.kind == 1) {
                    const long long local = sg.lo - sg.first;
                    sidx = (int)(local / a.KBe);
                    kb = (int)(local - (long long)sidx * a.KBe);
                    if (sg.lo == bLo && aHi > aLo &&
                        !wait_bar(&sh.a_pub, 0u, limit, &sh.abort, a.ctl, kWaitEmpty)) {
                        stop = true;
                        break;
                    }
                }
                for (long long j = sg.lo; j < sg.hi; ++j, ++i) {
                    if (!wait_bar(&sh.empty[st], ph ^ 1u, limit, &sh.abort, a.ctl, kWaitEmpty)) {
                        stop = true;
                        break;
                    }
                    if (sg.kind == 0) {
                        mbar_arrive_expect_tx(&sh.full_h[st], (uint32_t)Cfg::kActBytes);
                        tma_load_2d(smem + st * kStageBytes + kGrWBytes, &tm_x, &sh.full_h[st],
                                    (int)(j - sg.first) * 64, sg.g * a.NT, pol);
                    } else {
                        const int p = sg.off + sidx;
                        const uint32_t u = (uint32_t)(p * a.MT + (kb >> 1));
                        if (u != last_u) {
                            // one block computes the whole expert-in unit and counts it in once
                            if (!wait_count(&readyA[u], 1u, limit_peer, &sh.abort, a.ctl)) {
                                stop = true;
                                break;
                            }
                            if (nB == 0) GR_TRACE(kGtFirstFlag);
                            // the h' stores were made visible to this thread by the
                            // acquire; the async proxy reads them next
                            fence_proxy_async_global();
                            last_u = u;
                        }
                        mbar_arrive_expect_tx(&sh.full_h[st], (uint32_t)Cfg::kActBytes);
                        tma_load_2d(smem + st * kStageBytes + kGrWBytes, &tm_h, &sh.full_h[st], kb * 64, p * N,
                                    pol);
                        ++nB;
                        if (++kb == a.KBe) {
                            kb = 0;
                            ++sidx;
                        }
                    }
                    if (++st == kStages) {
                        st = 0;
                        ph ^= 1u;
                    }
                }
            }
            // no copy into this block's shared memory outlives it: the last
            // kStages stages issued
            for (long long k = i - kStages < 0 ? 0 : i - kStages; k < i; ++k)
                wait_bar_drain(&sh.full_h[k % kStages], (uint32_t)((k / kStages) & 1), limit, a.ctl);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (warps 3-10) --
        // Eight warps: two per TMEM lane quadrant (a warp reads the quadrant of its
        // index modulo 4).  Warp group eg (warps 3-6: 0, warps 7-10: 1) drains the
        // accumulator's 32-column slices eg, eg + 2, ...; named barrier 1 joins all
        // 256 threads, barrier 2 + eg the 128 threads of one group.
        const int q = warp & 3;
        const int row = q * 32 + lane;           // accumulator row = TMEM lane
        const int et = threadIdx.x - 96;         // 0..255
        const int eg = et >> 7;                  // warp group
        const int gt = et & 127;                 // thread within the group
        {
            // zero the other parity's counters: the launch before this one used
            // them and has finished; the launch after this one will use them
            const int oth = par ^ 1;
            const long long step = (long long)G * kGrEpi;
            for (long long k = (long long)cta * kGrEpi + et; k < a.cnt_a_len; k += step)
                a.readyA[(size_t)oth * a.cnt_a_len + k] = 0u;
            for (long long k = (long long)cta * kGrEpi + et; k < a.cnt_b_len; k += step)
                a.cntB[(size_t)oth * a.cnt_b_len + k] = 0u;
        }
        // the gates of expert e for the tokens of group g, zero where the token's
        // bit in its chunk's mask is clear or the token lies past the group or T,
        // and the bits themselves; staged in shared memory by the 256 threads
        auto stage_gates = [&](int g, int e) {
            for (int j = et; j < N; j += kGrEpi) {
                const int t = g * a.NT + j;
                bool bit = false;
                float gv = 0.f;
                if (j < a.NT && t < a.T) {
                    const int c = t / a.n;
                    bit = ((a.tmask[(size_t)c * a.E + e] >> (t - c * a.n)) & 1u) != 0u;
                    gv = a.gates[(size_t)t * a.E + e];
                }
                sh.s_gv[j] = bit ? gv : 0.f;
                const uint32_t bal = __ballot_sync(0xffffffffu, bit);
                if (lane == 0) sh.s_bits[j >> 5] = bal;
            }
            named_bar_sync(1, kGrEpi);
        };

        // at most two split expert-out units per block (its first and its last),
        // kept in fixed slots (no dynamically indexed local array)
        GrSeg pend_sg[2] = {};
        GrContrib pend_cb[2] = {};
        int npend = 0;
        // the same in every epilogue thread (fixed before the first barrier); later
        // decisions come from shared words read after named barriers
        bool failed = sh.abort0 != 0;   // (the tables are not read after an error)
        uint32_t flush_phase = 0u;

        // Finish the rows [r0, r1) slice of split expert-out unit (sg, cb): sum the
        // contributors' partial tiles in block order (a fixed order) and store those
        // rows of y.  This runs after the block's last accumulator, when the stage
        // ring is idle: the contributors' rows come by TMA, one box of 32 rows x N
        // tokens per (contributor, 32 rows), as many at a time as the ring holds
        // beside a running-sum region, and are added in shared memory.  The loops
        // are kept rolled: this code runs once per launch, so its size (fetched
        // cold) costs more than its loop overhead.
        constexpr int kBoxF4 = 32 * (N / 4);                // float4 per box: 32 rows x N tokens
        constexpr int kBoxBytes = kBoxF4 * 16;
        constexpr int kRingBoxes = kStages * kStageBytes / kBoxBytes;
        auto finish_split = [&](const GrSeg& sg, const GrContrib& cb, int kslot) -> bool {
            uint32_t* cnt = cntB + sg.unit;
            if (et == 0) {
                sh.ep_ok = wait_count(cnt, (uint32_t)cb.n, limit_peer, &sh.abort, a.ctl, kWaitPeers) ? 1 : 0;
                GR_TRACE(kGtFinBase + 3 * kslot);
                int k = 0;
                for (int qq = cb.q0; qq <= cb.q1 && k < kGrMaxContrib; ++qq) {
                    const long long lo = gr_range_lo(NB, G, qq);
                    if (gr_range_lo(NB, G, qq + 1) > lo) sh.s_contrib[k++] = qq * 2 + (lo >= sg.first ? 0 : 1);
                }
            }
            named_bar_sync(1, kGrEpi);
            if (!sh.ep_ok) return false;
            // rows in whole 8-row pieces (16-byte stores of y): rank r of n takes
            // [8 floor(16 r / n), 8 floor(16 (r + 1) / n)), possibly none
            const int r0 = 8 * (cb.rank * 16 / cb.n), r1 = 8 * ((cb.rank + 1) * 16 / cb.n);
            const int nrows = r1 - r0;                        // <= 64 (n >= 2), a multiple of 8
            if (nrows == 0) return true;                      // (the same in every thread)
            const int nb = (nrows + 31) / 32;                 // boxes per contributor
            const int cap = kRingBoxes / nb - 1;              // contributors per batch
            const int nitems = nrows * (N / 4);               // (row, token quad) items
            float4* ring4 = reinterpret_cast<float4*>(smem);  // boxes [0, nb): running sums
            const int nvalid = min(a.NT, a.T - sg.g * a.NT);   // tokens of the group
            for (int c0 = 0; c0 < cb.n; c0 += cap) {
                const int cn = min(cap, cb.n - c0);
                const bool last = c0 + cn == cb.n;
                if (et == 0) {
                    // the boxes about to be overwritten were last read by generic loads
                    fence_proxy_async_smem();
                    mbar_arrive_expect_tx(&sh.flush_bar, (uint32_t)(cn * nb * kBoxBytes));
                    const uint64_t pol = policy_evict_first();
#pragma unroll 1
                    for (int c = 0; c < cn; ++c)
#pragma unroll 1
                        for (int b = 0; b < nb; ++b)
                            tma_load_2d(smem + (size_t)((1 + c) * nb + b) * kBoxBytes, &tm_part, &sh.flush_bar,
                                        (r0 + 32 * b) * 4, sh.s_contrib[c0 + c] * (N / 4), pol);
                    sh.ep_ok = wait_bar_drain(&sh.flush_bar, flush_phase, limit, a.ctl) ? 1 : 0;
                }
                flush_phase ^= 1u;
                named_bar_sync(1, kGrEpi);
                if (!sh.ep_ok) return false;
                if (et == 0) GR_TRACE(kGtFinBase + 3 * kslot + 1);
                if (!last) {
                    // running sums of this batch's contributors
#pragma unroll 1
                    for (int i = et; i < nitems; i += kGrEpi) {
                        const int kq = i / nrows, rr = i - kq * nrows;
                        const int off = (rr >> 5) * kBoxF4 + kq * 32 + (rr & 31);
                        float4 acc = c0 == 0 ? make_float4(0.f, 0.f, 0.f, 0.f) : ring4[off];
#pragma unroll 1
                        for (int c = 0; c < cn; ++c) {
                            const float4 v = ring4[(1 + c) * nb * kBoxF4 + off];
                            acc.x += v.x;
                            acc.y += v.y;
                            acc.z += v.z;
                            acc.w += v.w;
                        }
                        ring4[off] = acc;
                    }
                    named_bar_sync(1, kGrEpi);   // the ring is read; the next batch may land
                    continue;
                }
                // the last batch: 128 tokens at a time, the sums (plus the fc2 bias
                // sums) rounded into the output staging [128 tokens][64 rows], then
                // written as 16-byte pieces of 8 rows
#pragma unroll 1
                for (int h = 0; h < N / 128; ++h) {
#pragma unroll 1
                    for (int i = et; i < nrows * 32; i += kGrEpi) {
                        const int kql = i / nrows, rr = i - kql * nrows;
                        const int kq = 32 * h + kql;
                        const int off = (rr >> 5) * kBoxF4 + kq * 32 + (rr & 31);
                        float4 acc = c0 == 0 ? make_float4(0.f, 0.f, 0.f, 0.f) : ring4[off];
#pragma unroll 1
                        for (int c = 0; c < cn; ++c) {
                            const float4 v = ring4[(1 + c) * nb * kBoxF4 + off];
                            acc.x += v.x;
                            acc.y += v.y;
                            acc.z += v.z;
                            acc.w += v.w;
                        }
                        const float z[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int tok = 4 * kq + u;
                            const float yb = (a.ybias != nullptr && tok < nvalid)
                                                 ? __ldg(a.ybias + (size_t)(sg.g * a.NT + tok) * a.d_h + sg.rt * 128 +
                                                         r0 + rr)
                                                 : 0.f;
                            ostage[(4 * kql + u) * 64 + rr] = __float2bfloat16_rn(z[u] + yb);
                        }
                    }
                    named_bar_sync(1, kGrEpi);
                    const int np = nrows / 8;
#pragma unroll 1
                    for (int c = et; c < 128 * np; c += kGrEpi) {
                        const int tl = c / np, pc = c - tl * np;
                        const int tok = 128 * h + tl;
                        if (tok < nvalid)
                            *reinterpret_cast<uint4*>(a.y + (size_t)(sg.g * a.NT + tok) * a.d_h + sg.rt * 128 + r0 +
                                                      8 * pc) =
                                *reinterpret_cast<const uint4*>(ostage + tl * 64 + 8 * pc);
                    }
                    named_bar_sync(1, kGrEpi);   // the staging and the ring are free again
                }
            }
            if (et == 0) GR_TRACE(kGtFinBase + 3 * kslot + 2);
            return true;
        };

        // Announcements.  A release waits for the block's bulk copies in flight, so
        // the block announces in two batches, each when none of its copies is in
        // flight: all its expert-in units once the last one's h' is written (the
        // producer and the loader hold their first expert-out copy until then), and
        // all its expert-out partials after its last accumulator.  One thread fences
        // after a barrier that orders every thread's stores before it.
        const long long uLo = aLo / a.KB, uHi = aHi / a.KB;   // this block's expert-in units
        auto announce_a = [&]() {
            named_bar_sync(1, kGrEpi);
            if (et == 0) {
                GR_TRACE(kGtAnnounce);
                fence_acq_rel_gpu();
                for (long long u = uLo; u < uHi; ++u)
                    if ((int)u != a.skip_flag_unit) atomicAdd(&readyA[u], 1u);
                mbar_arrive(&sh.a_pub);
                GR_TRACE(kGtAFlushed);
            }
        };
        auto flush_pending = [&]() -> bool {
            if (npend == 0) return true;
            named_bar_sync(1, kGrEpi);
            if (et == 0) {
                GR_TRACE(kGtLoopEnd);
                fence_acq_rel_gpu();
                if (npend >= 1) atomicAdd(cntB + pend_sg[0].unit, 1u);
                if (npend >= 2) atomicAdd(cntB + pend_sg[1].unit, 1u);
                GR_TRACE(kGtFlushAnnounced);
            }
            // one copy of the finisher's code, run once per pending unit (its
            // instructions are fetched cold once per launch, not once per call
            // site); the slot is picked field by field, in registers
#pragma unroll 1
            for (int k = 0; k < npend; ++k) {
                const GrSeg sgk = k == 0 ? pend_sg[0] : pend_sg[1];
                const GrContrib cbk = k == 0 ? pend_cb[0] : pend_cb[1];
                if (!finish_split(sgk, cbk, k)) return false;
            }
            npend = 0;
            return true;
        };

        GrIter it;
        it.init(aLo, aHi, bLo, bHi);
        GrSeg sg;
        uint32_t acc_i = 0;
        int cur_kind = 0;
        __nv_bfloat16* const stg = ostage + eg * (32 * 128);   // this group's staging slice
        while (!failed && it.next(a, sg)) {
            if (sg.kind != cur_kind) {
                if (uHi > uLo) announce_a();
                cur_kind = sg.kind;
            }
            GrContrib cb;
            if (sg.kind == 0) {
                cb.q0 = cb.q1 = cta;   // whole expert-in units: never split
                cb.n = 1;
                cb.rank = 0;
            } else {
                cb = gr_contributors(sg.first, sg.last, NB, G, cta);
            }
            // stage this unit's gates while its accumulator completes
            if (sg.kind == 0 && cb.n == 1) stage_gates(sg.g, sg.e);
            const int ab = (int)(acc_i & 1u);
            const uint32_t aph = (acc_i >> 1) & 1u;
            // one thread waits and the 256 threads take its decision together, so
            // the named barriers below always see all of them
            if (et == 0)
                sh.ep_wait[acc_i & 1u] =
                    wait_bar(&sh.acc_full[ab], aph, limit, &sh.abort, a.ctl, kWaitAccFull) ? 1 : 0;
            named_bar_sync(1, kGrEpi);
            if (!sh.ep_wait[acc_i & 1u]) { failed = true; break; }
            tc_fence_after();
            if (et == 0 && acc_i == 0) GR_TRACE(kGtFirstAcc);
            const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * N);
            const int nvalid = min(a.NT, a.T - sg.g * a.NT);   // tokens of the group
            if (cb.n == 1) {
                // The whole unit is here: all 128 rows straight from the accumulator,
                // 32 tokens at a time, each group its own slices.  A slice is staged
                // token-major in shared memory ([32 tokens][128 rows] bf16: a token's
                // 128 rows are 256 contiguous bytes of h' or y) and written with
                // 16-byte stores.
                __nv_bfloat16* dst;
                size_t ld;
                int ntok;
                // fc1 bias of this accumulator row (expert-in units), or 0
                const float bin = (sg.kind == 0 && a.b_in != nullptr)
                                      ? __ldg(a.b_in + (size_t)sg.e * a.d_e + sg.mt * 128 + row) : 0.f;
                if (sg.kind == 0) {
                    dst = a.hbuf + (size_t)sg.p * N * a.d_e + sg.mt * 128;
                    ld = (size_t)a.d_e;
                    ntok = N;                      // h' rows of every token (masked ones are 0)
                } else {
                    dst = a.y + (size_t)sg.g * a.NT * a.d_h + sg.rt * 128;
                    ld = (size_t)a.d_h;
                    ntok = nvalid;
                }
#pragma unroll 1
                for (int c0 = 32 * eg; c0 < N; c0 += 64) {
                    uint32_t r[32];
                    const bool stamp = et == 0 && acc_i == 0;
                    tmem_ld_32x32b_x32(tbase + (uint32_t)c0, r);
                    tmem_ld_wait();
                    if (stamp) GR_TRACE(kGtSliceBase + 4 * (c0 >> 5));
                    __nv_bfloat16 hb[32];
                    if (sg.kind == 0) {
                        // the slice's gates and bits into registers first: loads from
                        // shared memory interleaved with the staging stores would each
                        // wait for the store before them (the compiler cannot tell the
                        // two shared arrays apart), serialising the 32 tokens
                        const uint32_t bits = sh.s_bits[c0 >> 5];
                        float gv[32];
#pragma unroll
                        for (int u4 = 0; u4 < 8; ++u4) {
                            const float4 g4 = reinterpret_cast<const float4*>(sh.s_gv + c0)[u4];
                            gv[4 * u4] = g4.x;
                            gv[4 * u4 + 1] = g4.y;
                            gv[4 * u4 + 2] = g4.z;
                            gv[4 * u4 + 3] = g4.w;
                        }
#pragma unroll
                        for (int u = 0; u < 32; ++u) {
                            const float h =
                                ((bits >> u) & 1u) ? gv[u] * gr_swish(__uint_as_float(r[u]) + bin) : 0.f;
                            hb[u] = __float2bfloat16_rn(h);
                        }
                    } else if (a.ybias != nullptr) {
                        // the tokens' fc2 bias sums of this row (fp32, added before rounding)
                        float yb[32];
                        const float* ybc = a.ybias + (size_t)(sg.g * a.NT + c0) * a.d_h + sg.rt * 128 + row;
#pragma unroll
                        for (int u = 0; u < 32; ++u) yb[u] = c0 + u < ntok ? __ldg(ybc + (size_t)u * a.d_h) : 0.f;
#pragma unroll
                        for (int u = 0; u < 32; ++u) hb[u] = __float2bfloat16_rn(__uint_as_float(r[u]) + yb[u]);
                    } else {
#pragma unroll
                        for (int u = 0; u < 32; ++u) hb[u] = __float2bfloat16_rn(__uint_as_float(r[u]));
                    }
                    // the group's previous slice has been copied out (barrier below)
#pragma unroll
                    for (int u = 0; u < 32; ++u) stg[u * 128 + row] = hb[u];
                    if (stamp) GR_TRACE(kGtSliceBase + 4 * (c0 >> 5) + 1);
                    named_bar_sync(2 + eg, 128);
                    if (stamp) GR_TRACE(kGtSliceBase + 4 * (c0 >> 5) + 2);
                    if (et == 0 && acc_i == 0 && c0 == 0) GR_TRACE(kGtFirstSlice);
                    // 32 tokens x 16 pieces of 16 bytes
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int c = gt + 128 * k;
                        const int tok = c >> 4, piece = c & 15;
                        if (c0 + tok < ntok)
                            *reinterpret_cast<uint4*>(dst + (size_t)(c0 + tok) * ld + piece * 8) =
                                reinterpret_cast<const uint4*>(stg + tok * 128)[piece];
                    }
                    named_bar_sync(2 + eg, 128);   // the staging slice is free again
                    if (stamp) GR_TRACE(kGtSliceBase + 4 * (c0 >> 5) + 3);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.acc_empty[ab]);
                if (et == 0 && acc_i == 0) GR_TRACE(kGtADrained);
                ++acc_i;
                if (sg.kind == 0) named_bar_sync(1, kGrEpi);   // the staged gates are free again
            } else {
                // publish this block's partial tile and count it in; the slice is
                // finished after the last accumulator.  Layout: float4 (token quad
                // k, row) at k * 128 + row.  (Only expert-out units are ever split.)
                float* part = a.partB;
                const int myslot = bLo >= sg.first ? 0 : 1;
                float4* dst = reinterpret_cast<float4*>(part + (size_t)(cta * 2 + myslot) * (N * 128)) + row;
#pragma unroll 1
                for (int c0 = 32 * eg; c0 < N; c0 += 64) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tbase + (uint32_t)c0, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        dst[(c0 / 4 + k) * 128] = make_float4(__uint_as_float(r[4 * k]), __uint_as_float(r[4 * k + 1]),
                                                              __uint_as_float(r[4 * k + 2]),
                                                              __uint_as_float(r[4 * k + 3]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.acc_empty[ab]);
                ++acc_i;
                if (npend == 0) { pend_sg[0] = sg; pend_cb[0] = cb; ++npend; }
                else if (npend == 1) { pend_sg[1] = sg; pend_cb[1] = cb; ++npend; }
            }
        }
        if (!failed && cur_kind == 0 && uHi > uLo) announce_a();   // expert-in work only
        if (!failed) flush_pending();
        if (et == 0) GR_TRACE(kGtEpiEnd);
    }

    // ------------------------------------------------------------ teardown --
    __syncthreads();
    if (warp == 2) {
        if (lane == 0) wait_bar_drain(&sh.mma_done, 0, limit, a.ctl);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::kTmemCols);
    }
    if (threadIdx.x == 0) GR_TRACE(kGtEnd);
}

template <int N>
static size_t group_smem_bytes() {
    return 1024 + (size_t)GrCfg<N>::kStages * GrCfg<N>::kStageBytes + sizeof(GrShared<N>) + 1024 +
           kGrOutStageBytes;
}

template <int N>
static cudaError_t launch_group_n(const GrArgs& a, const CUtensorMap* maps, int grid, cudaStream_t s) {
    const size_t smem = group_smem_bytes<N>();
    cudaError_t err =
        cudaFuncSetAttribute(union_expert_group<N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kGrThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    // One block per SM, all resident at once (blocks wait on one another's
    // results, with bounded waits), and a programmatic dependent of the
    // group-plan kernel: its blocks are scheduled while that kernel runs and
    // start their set-up early.
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, union_expert_group<N>, maps[0], maps[1], maps[2], maps[3], maps[4], a);
}

cudaError_t launch_forward_group(const GrArgs& a, const CUtensorMap* maps, int grid, cudaStream_t s) {
    if (grid > kGrMaxContrib || a.E > kGrMaxE) return cudaErrorInvalidValue;
    if (a.N == 256) return launch_group_n<256>(a, maps, grid, s);
    if (a.N == 128) return launch_group_n<128>(a, maps, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace bffn
