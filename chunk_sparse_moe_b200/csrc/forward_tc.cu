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
// MMAs (the whole warp runs the loop, one elected lane issues), warp 2 owns
// TMEM and copies gated activations into the
// stages once their flag is set, warps 3-6 drain the accumulators (TMEM ->
// registers) and do the split reductions, Swish, gate, mask and stores.
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
constexpr int kMaxContrib = 160;               // >= blocks per launch (one per SM)

struct TcShared {
    uint64_t full_w[kStages];    // weight (+x) tile landed
    uint64_t full_h[kStages];    // gated-activation tile landed (or A stage: no tile); 32 arrivals
    uint64_t empty[kStages];     // MMAs reading the stage are done
    uint64_t acc_full[kNAcc];    // accumulator complete
    uint64_t acc_empty[kNAcc];   // accumulator drained
    uint64_t mma_done;
    uint32_t tmem_base;
    volatile int abort;
    uint32_t epoch;
    int P;
    int ep_wait[2];   // acc-full wait result, double-buffered by segment parity
    int ep_ok;        // the contributors of the current split unit have all arrived
    int s_contrib[kMaxContrib];  // their partial slots, in block order
    // single-chunk tables (fuse_union)
    int32_t s_counts[1];
    int32_t s_offsets[2];
    int32_t s_pair_ce[kMaxE];
    uint32_t s_tmask[kMaxE];
    int32_t s_elist[kMaxE];      // producer: expert ids of the current B unit
    uint32_t s_bal[kMaxE / 32];  // per 32-expert group: which experts are active
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

// Tile ranges: block i owns tiles [range_lo(i), range_lo(i + 1)) of a kind.
// 32-bit arithmetic whenever the products fit (64-bit division is a long
// software sequence).
__device__ __forceinline__ long long range_lo(long long total, int G, int i) {
    if (total < (1LL << 31) / (G + 1))
        return (long long)((uint32_t)total * (uint32_t)i / (uint32_t)G);
    return total * i / G;
}
// the block whose range holds tile j
__device__ __forceinline__ int block_of(long long j, long long total, int G) {
    if (total < (1LL << 31) / (G + 1))
        return (int)((((uint32_t)j + 1u) * (uint32_t)G - 1u) / (uint32_t)total);
    return (int)(((j + 1) * G - 1) / total);
}

// The blocks that hold tiles of a unit spanning tiles [first, last]: the blocks
// q0..q1 whose ranges are not empty (ranges are empty only when there are fewer
// tiles than blocks); n of them, and the rank of block `me` among them (-1 if
// it is not one).
struct Contrib {
    int q0, q1, n, rank;
};
__device__ __forceinline__ Contrib contributors(long long first, long long last, long long total,
                                                int G, int me) {
    Contrib c;
    c.q0 = block_of(first, total, G);
    c.q1 = block_of(last, total, G);
    if (total >= G) {                       // no empty ranges
        c.n = c.q1 - c.q0 + 1;
        c.rank = (me >= c.q0 && me <= c.q1) ? me - c.q0 : -1;
        return c;
    }
    c.n = 0;
    c.rank = -1;
    for (int qq = c.q0; qq <= c.q1; ++qq) {
        if (range_lo(total, G, qq + 1) > range_lo(total, G, qq)) {
            if (qq == me) c.rank = c.n;
            ++c.n;
        }
    }
    return c;
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

// Timeline stamps of one launch (globaltimer, ns), written only when a trace
// buffer is attached: per block 16 slots.
enum : int {
    kTrStart = 0, kTrPrologue = 1, kTrFirstLoad = 2, kTrLastLoad = 3, kTrFirstFull = 4,
    kTrLastACommit = 5, kTrFirstAcc = 6, kTrLastAEpi = 7, kTrFirstFlag = 8, kTrLastFlag = 9,
    kTrLastCommit = 10, kTrLastEpi = 11, kTrTeardown = 12, kTrEnd = 13,
    // first expert-in / expert-out unit of the block, step by step
    kTrAPartial = 14, kTrAArrive = 15, kTrAReduced = 16, kTrAPublished = 17,
    kTrGatesLoaded = 18, kTrCtlLoaded = 19, kTrTmemAlloc = 20,
    kTrBPartial = 21, kTrBArrive = 22, kTrBReduced = 23, kTrFirstHCopied = 24, kTrFirstBMma = 25,
    kTrSlots = 32
};
#define BFFN_TRACE(slot) \
    do { if (a.trace) a.trace[(size_t)blockIdx.x * kTrSlots + (slot)] = globaltimer_ns(); } while (0)
#define BFFN_TRACE_ONCE(slot) \
    do { \
        if (a.trace && a.trace[(size_t)blockIdx.x * kTrSlots + (slot)] == 0ull) \
            a.trace[(size_t)blockIdx.x * kTrSlots + (slot)] = globaltimer_ns(); \
    } while (0)

// N: tokens per MMA (the chunk padded to 16 or 32); a compile-time constant so
// every per-token loop below is unrolled with no predicates and its loads are
// issued together.
template <int N>
__global__ void __launch_bounds__(kThreads, 1)
union_expert_forward_tc(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_win,
                        const __grid_constant__ CUtensorMap tm_wout, const TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    TcShared& sh = *reinterpret_cast<TcShared*>(smem + kStages * kStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, cta = blockIdx.x;

    if (threadIdx.x == 0) {
        BFFN_TRACE(kTrStart);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sh.full_w[s], 1);
            mbar_init(&sh.full_h[s], 32);   // one arrival per loader lane
            mbar_init(&sh.empty[s], 1);
        }
        for (int s = 0; s < kNAcc; ++s) {
            mbar_init(&sh.acc_full[s], 1);
            mbar_init(&sh.acc_empty[s], 4);
        }
        mbar_init(&sh.mma_done, 1);
        fence_mbar_init();
        // written by earlier launches only: plain L2 loads, issued together
        const int32_t st0 = __ldcg(&a.ctl->status);
        const uint32_t ep0 = __ldcg(&a.ctl->epoch);
        const unsigned long long key0 = claim_shape_key(a.ctl, a.shape_key);
        const bool key_ok = key0 == 0ull || key0 == a.shape_key;
        if (!key_ok) record_error(a.ctl, kErrWorkspace, kShapeKey);
        sh.abort = st0 != 0 || !key_ok;
        sh.epoch = ep0;
        BFFN_TRACE(kTrCtlLoaded);
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_win);
        prefetch_tmap(&tm_wout);
    }
    if (warp == 2) {
        tmem_alloc(&sh.tmem_base, kTmemCols);
        tmem_relinquish();
        if (lane == 0) BFFN_TRACE(kTrTmemAlloc);
    }
    if (a.fuse_union && warp >= 3) {
        // union of the single chunk (c = 0) into shared memory.  Warps 3-6 take
        // 32-expert groups; each lane loads its expert's gates of all tokens at once
        // (independent, coalesced across lanes), ORs the non-zero bits, and the
        // group's ballot is compacted in ascending order afterwards.
        const int nt = min(a.n, a.T);
        const int ngroups = (a.E + 31) / 32;
        for (int g = warp - 3; g < ngroups; g += 4) {
            const int e = g * 32 + lane;
            // unconditional loads from clamped (valid) addresses, selected afterwards
            const int ec = min(e, a.E - 1);
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __ldg(a.gates + (size_t)min(j, nt - 1) * a.E + ec);
            uint32_t bits = 0u;
#pragma unroll
            for (int j = 0; j < 32; ++j) bits |= ((e < a.E && j < nt && v[j] != 0.f) ? 1u : 0u) << j;
            if (e < a.E) sh.s_tmask[e] = bits;
            const uint32_t bal = __ballot_sync(0xffffffffu, bits != 0u);
            if (lane == 0) sh.s_bal[g] = bal;
            if (lane == 0 && g == 0) BFFN_TRACE(kTrGatesLoaded);
        }
        named_bar_sync(1, 128);
        if (warp == 3) {
            int base = 0;
            for (int g = 0; g < ngroups; ++g) {
                const uint32_t bal = sh.s_bal[g];
                if ((bal >> lane) & 1u)
                    sh.s_pair_ce[base + __popc(bal & ((1u << lane) - 1u))] = g * 32 + lane;
                base += __popc(bal);
            }
            if (lane == 0) {
                sh.s_counts[0] = base;
                sh.s_offsets[0] = 0;
                sh.s_offsets[1] = base;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0) BFFN_TRACE(kTrPrologue);

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
    // counters of this launch: one of two sets, by launch parity; this launch
    // zeroes the other set for the next one
    const int par = (int)(sh.epoch & 1u);
    uint32_t* const cntA = a.cntA + (size_t)par * a.cnt_a_len;
    uint32_t* const readyA = a.readyA + (size_t)par * a.cnt_a_len;
    uint32_t* const cntB = a.cntB + (size_t)par * a.cnt_b_len;
    const long long NA = (long long)P * a.MT * a.KB;
    const long long NB = (long long)P * a.RT * a.KBe;
    const long long aLo = NA > 0 ? range_lo(NA, G, cta) : 0, aHi = NA > 0 ? range_lo(NA, G, cta + 1) : 0;
    const long long bLo = NB > 0 ? range_lo(NB, G, cta) : 0, bHi = NB > 0 ? range_lo(NB, G, cta + 1) : 0;
    // Waits on other blocks (activations ready, split-unit peers) run out after
    // wait_ns; waits on this block's own pipeline are downstream of those and get
    // twice as long, so the first timeout recorded names the root cause.
    const uint64_t limit_peer = a.wait_ns;
    const uint64_t limit = 2 * a.wait_ns;

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
                    if (i == 0) BFFN_TRACE(kTrFirstLoad);
                    BFFN_TRACE(kTrLastLoad);
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
        // The whole warp runs the loop with warp-wide waits and one elected lane
        // issues: a loop run by one lane while the other 31 wait issued tcgen05
        // work at about half the rate.  Each operand descriptor is the stage's
        // base descriptor plus a constant, and the next stage's barriers are
        // tested while the current stage's MMAs issue.
        {
            const bool leader = elect_one();
            const uint32_t idesc = idesc_bf16_f32(128, N);
            const uint64_t desc0 = sw128_kmajor_desc(smem_u32(smem));
            SegIter it;
            it.init(aLo, aHi, bLo, bHi);
            Seg sg;
            long long i = 0;
            int st = 0;
            uint32_t ph = 0u;
            uint32_t rw = 0u, rh = 0u;   // the current stage's barriers as last tested
            uint32_t acc_i = 0;
            bool stop = __shfl_sync(0xffffffffu, sh.abort, 0) != 0;
            while (!stop && it.next(a, tb, sg)) {
                const int ab = (int)(acc_i % kNAcc);
                const uint32_t aph = (acc_i / kNAcc) & 1u;
                if (!wait_bar_warp(&sh.acc_empty[ab], aph ^ 1u, limit, &sh.abort, a.ctl, kWaitAccEmpty))
                    break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(ab * 32);
                for (long long j = sg.lo; j < sg.hi; ++j, ++i) {
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
                        fence_proxy_async_smem();   // activation tiles were written by cp.async
                        if (i == 0) BFFN_TRACE(kTrFirstFull);
                        if (sg.kind == 1) BFFN_TRACE_ONCE(kTrFirstBMma);
                        const uint64_t ds = desc0 + (uint64_t)(st * (kStageBytes >> 4));
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16(d, ds + (uint64_t)((kk * 32) >> 4), ds + (uint64_t)((kWBytes + kk * 32) >> 4),
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
                    if (sg.kind == 0) BFFN_TRACE(kTrLastACommit);
                    BFFN_TRACE(kTrLastCommit);
                }
                __syncwarp();
                ++acc_i;
            }
            if (leader) umma_commit(&sh.mma_done);
            __syncwarp();
        }
    } else if (warp == 2) {
        // ------------------------------------- gated-activation loader --
        // For an expert-out tile the gated activations h' of its pair must have
        // been written by the block that finished the pair's expert-in unit.  Lane 0
        // spins (bounded) on that unit's flag; then the warp copies the tile's
        // [N x 64] bf16 slice from L2 into the stage with plain loads, writing it in
        // the 128-byte-swizzled layout the MMA descriptor expects, and fences the
        // shared-memory writes for the tensor core (async proxy).  Staying in the
        // generic proxy on the global side keeps this path clear of the weight
        // stream's bulk copies.
        SegIter it;
        it.init(aLo, aHi, bLo, bHi);
        Seg sg;
        long long i = 0;
        bool stop = sh.abort != 0;
        constexpr int kPieces = N * 8 / 32;       // 16-byte pieces of one [N x 64] slice per lane
        while (!stop && it.next(a, tb, sg)) {
            for (long long j = sg.lo; j < sg.hi; ++j, ++i) {
                const int st = (int)(i % kStages);
                const uint32_t ph = (uint32_t)((i / kStages) & 1);
                int ok = 1;
                if (lane == 0)
                    ok = wait_bar(&sh.empty[st], ph ^ 1u, limit, &sh.abort, a.ctl, kWaitEmpty) ? 1 : 0;
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
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
                if (lane == 0) {
                    // every holder of a slice of expert-in unit u counts itself in once
                    // its slice of h' is written
                    const long long fA = (long long)u * a.KB;
                    const int ncA = contributors(fA, fA + a.KB - 1, NA, G, -1).n;
                    ok = wait_count(&readyA[u], (uint32_t)ncA, limit_peer, &sh.abort, a.ctl) ? 1 : 0;
                    if (ok) {
                        BFFN_TRACE_ONCE(kTrFirstFlag);
                        BFFN_TRACE(kTrLastFlag);
                    }
                }
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    stop = true;
                    break;
                }
                (void)ld_acquire_gpu(&readyA[u]);     // every lane acquires the releases
                // asynchronous 16-byte copies into the 128-byte-swizzled stage; each
                // lane's arrival on full_h fires when its copies have landed, so the
                // loader moves on to the next tile at once
                const uint4* src = reinterpret_cast<const uint4*>(
                    a.hbuf + (size_t)p * N * a.d_e + (size_t)kb * 64);
                uint8_t* dst = smem + st * kStageBytes + kWBytes;
#pragma unroll
                for (int k = 0; k < kPieces; ++k) {
                    const int c = lane + 32 * k;
                    const int r = c >> 3, c16 = c & 7;
                    cp_async_16(dst + r * 128 + ((c16 ^ (r & 7)) << 4), src + (size_t)r * (a.d_e / 8) + c16);
                }
                cp_async_mbar_arrive(&sh.full_h[st]);
                if (lane == 0) BFFN_TRACE_ONCE(kTrFirstHCopied);
            }
        }
        cp_async_wait_all();   // no copy into this block's shared memory outlives it
    } else {
        // ------------------------------------------------ epilogue (warps 3-6) --
        const int q = warp & 3;
        const int row = q * 32 + lane;           // accumulator row = TMEM lane
        const int et = threadIdx.x - 96;         // 0..127
        {
            // zero the other parity's counters: the launch before this one used
            // them and has finished; the launch after this one will use them
            const int oth = par ^ 1;
            const long long step = (long long)G * 128;
            for (long long k = (long long)cta * 128 + et; k < a.cnt_a_len; k += step) {
                a.cntA[(size_t)oth * a.cnt_a_len + k] = 0u;
                a.readyA[(size_t)oth * a.cnt_a_len + k] = 0u;
            }
            for (long long k = (long long)cta * 128 + et; k < a.cnt_b_len; k += step)
                a.cntB[(size_t)oth * a.cnt_b_len + k] = 0u;
        }
        if (a.fuse_union && cta == 0 && P == 0 && !sh.abort) {
            // empty union: y is all zeros
            const size_t total = (size_t)min(a.n, a.T) * a.d_h;
            for (size_t k = et; k < total; k += 128) a.y[k] = __float2bfloat16_rn(0.f);
        }
        // Units split across blocks are finished in two passes per kind: first
        // every partial of the kind is published as its accumulator arrives, then
        // the block waits for the units' other contributors and reduces its slice.
        // Publishing all partials before any wait keeps blocks from waiting on
        // one another in a chain.  A block holds at most two split units per kind
        // (its first and its last).
        Seg pend_sg[2];
        Contrib pend_cb[2];
        int npend = 0;
        bool failed = false;

        // finish the rows [r0, r1) slice of split unit (sg, cb): sum the partials
        // in block order, then gated Swish + mask into h' (A) or store y (B)
        auto finish_split = [&](const Seg& sg, const Contrib& cb) -> bool {
            const long long total = sg.kind == 0 ? NA : NB;
            uint32_t* cnt = (sg.kind == 0 ? cntA : cntB) + sg.unit;
            if (et == 0) {
                sh.ep_ok = wait_count(cnt, (uint32_t)cb.n, limit_peer, &sh.abort, a.ctl, kWaitPeers) ? 1 : 0;
                int k = 0;
                for (int qq = cb.q0; qq <= cb.q1 && k < kMaxContrib; ++qq) {
                    const long long lo = range_lo(total, G, qq);
                    if (range_lo(total, G, qq + 1) > lo) sh.s_contrib[k++] = qq * 2 + (lo >= sg.first ? 0 : 1);
                }
            }
            named_bar_sync(1, 128);
            if (!sh.ep_ok) return false;
            const int c = sg.c;
            const int nt = min(a.n, a.T - c * a.n);
            const float* part = sg.kind == 0 ? a.partA : a.partB;
            const float4* pbase = reinterpret_cast<const float4*>(part);
            const int r0 = cb.rank * 128 / cb.n, r1 = (cb.rank + 1) * 128 / cb.n;
            const int nrows = r1 - r0;
            uint32_t bits = 0u;
            const float* gcol = nullptr;
            if (sg.kind == 0) {
                bits = tb.tmask[(size_t)c * a.E + sg.e];
                gcol = a.gates + (size_t)c * a.n * a.E + sg.e;
            }
            // Items (row, token quad) of the slice, two per thread per pass; for each
            // pass every contributor's float4 (and the four gates of an A item) is
            // requested before any is used, 8 contributors at a time.
            const int nitems = nrows * (N / 4);
            for (int base = 0; base < nitems; base += 256) {
                int rr[2], kq[2];
                bool on[2];
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    const int itx = base + m * 128 + et;
                    on[m] = itx < nitems;
                    const int ic = on[m] ? itx : 0;
                    rr[m] = r0 + ic % nrows;       // consecutive threads: consecutive rows
                    kq[m] = ic / nrows;            // token quad
                }
                float gq[2][4];
                if (sg.kind == 0) {
#pragma unroll
                    for (int m = 0; m < 2; ++m)
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            gq[m][u] = __ldg(gcol + (size_t)min(4 * kq[m] + u, nt - 1) * a.E);
                }
                float4 acc[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
                for (int c0 = 0; c0 < cb.n; c0 += 8) {
                    float4 t4[2][8];
#pragma unroll
                    for (int m = 0; m < 2; ++m)
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            t4[m][u] = __ldcg(pbase + (size_t)sh.s_contrib[min(c0 + u, cb.n - 1)] * (N * 32) +
                                              kq[m] * 128 + rr[m]);
#pragma unroll
                    for (int m = 0; m < 2; ++m)
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            if (c0 + u < cb.n) {
                                acc[m].x += t4[m][u].x;
                                acc[m].y += t4[m][u].y;
                                acc[m].z += t4[m][u].z;
                                acc[m].w += t4[m][u].w;
                            }
                        }
                }
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    if (!on[m]) continue;
                    const float z[4] = {acc[m].x, acc[m].y, acc[m].z, acc[m].w};
                    if (sg.kind == 0) {
                        __nv_bfloat16* hrow = a.hbuf + (size_t)sg.p * N * a.d_e + sg.mt * 128 + rr[m];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int j = 4 * kq[m] + u;
                            const float h = ((bits >> j) & 1u) ? gq[m][u] * swish(z[u]) : 0.f;
                            hrow[(size_t)j * a.d_e] = __float2bfloat16_rn(h);
                        }
                    } else {
                        __nv_bfloat16* ycol = a.y + (size_t)c * a.n * a.d_h + sg.rt * 128 + rr[m];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int j = 4 * kq[m] + u;
                            if (j < nt) ycol[(size_t)j * a.d_h] = __float2bfloat16_rn(z[u]);
                        }
                    }
                }
            }
            if (et == 0) BFFN_TRACE_ONCE(sg.kind == 0 ? kTrAReduced : kTrBReduced);
            return true;
        };
        // this block's rows of h' for expert-in unit `unit` are written: count it in
        auto announce_ready = [&](uint32_t unit) {
            __threadfence();
            named_bar_sync(1, 128);
            if (et == 0) {
                if ((int)unit != a.skip_flag_unit) atomicAdd(&readyA[unit], 1u);
                BFFN_TRACE(kTrLastAEpi);
                BFFN_TRACE_ONCE(kTrAPublished);
            }
        };
        auto flush_pending = [&]() -> bool {
            for (int k = 0; k < npend; ++k) {
                if (!finish_split(pend_sg[k], pend_cb[k])) return false;
                if (pend_sg[k].kind == 0) announce_ready(pend_sg[k].unit);
            }
            npend = 0;
            return true;
        };

        SegIter it;
        it.init(aLo, aHi, bLo, bHi);
        Seg sg;
        uint32_t acc_i = 0;
        int cur_kind = 0;
        while (!failed && it.next(a, tb, sg)) {
            if (sg.kind != cur_kind) {
                if (!flush_pending()) { failed = true; break; }
                cur_kind = sg.kind;
            }
            const int ab = (int)(acc_i % kNAcc);
            const uint32_t aph = (acc_i / kNAcc) & 1u;
            // one thread waits and the 128 threads take its decision together, so
            // the named barriers below always see all of them
            if (et == 0)
                sh.ep_wait[acc_i & 1u] =
                    wait_bar(&sh.acc_full[ab], aph, limit, &sh.abort, a.ctl, kWaitAccFull) ? 1 : 0;
            named_bar_sync(1, 128);
            if (!sh.ep_wait[acc_i & 1u]) { failed = true; break; }
            tc_fence_after();
            if (et == 0 && acc_i == 0) BFFN_TRACE(kTrFirstAcc);
            uint32_t r[32];
            const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * 32);
            if constexpr (N == 32) tmem_ld_32x32b_x32(taddr, r);
            else tmem_ld_32x32b_x16(taddr, r);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.acc_empty[ab]);
            ++acc_i;
            float v[N];
#pragma unroll
            for (int j = 0; j < N; ++j) v[j] = __uint_as_float(r[j]);

            const long long total = sg.kind == 0 ? NA : NB;
            const Contrib cb = contributors(sg.first, sg.last, total, G, cta);
            if (cb.n == 1) {
                // the whole unit is here: all 128 rows straight from the accumulator
                const int c = sg.c;
                const int nt = min(a.n, a.T - c * a.n);      // tokens of the chunk, >= 1
                if (sg.kind == 0) {
                    const uint32_t bits = tb.tmask[(size_t)c * a.E + sg.e];   // tokens that exist
                    const float* gcol = a.gates + (size_t)c * a.n * a.E + sg.e;
                    float gv[N];
#pragma unroll
                    for (int j = 0; j < N; ++j) gv[j] = __ldg(gcol + (size_t)min(j, nt - 1) * a.E);
                    __nv_bfloat16* hrow = a.hbuf + (size_t)sg.p * N * a.d_e + sg.mt * 128 + row;
#pragma unroll
                    for (int j = 0; j < N; ++j) {
                        const float h = ((bits >> j) & 1u) ? gv[j] * swish(v[j]) : 0.f;
                        hrow[(size_t)j * a.d_e] = __float2bfloat16_rn(h);
                    }
                    announce_ready(sg.unit);
                } else {
                    __nv_bfloat16* ycol = a.y + (size_t)c * a.n * a.d_h + sg.rt * 128 + row;
#pragma unroll
                    for (int j = 0; j < N; ++j)
                        if (j < nt) ycol[(size_t)j * a.d_h] = __float2bfloat16_rn(v[j]);
                    if (et == 0) BFFN_TRACE(kTrLastEpi);
                }
            } else {
                // publish this block's partial tile and count it in; the slice is
                // finished in the second pass
                float* part = sg.kind == 0 ? a.partA : a.partB;
                uint32_t* cnt = (sg.kind == 0 ? cntA : cntB) + sg.unit;
                const long long myLo = sg.kind == 0 ? aLo : bLo;
                const int myslot = myLo >= sg.first ? 0 : 1;
                // partial tile layout: float4 (k, row) at k * 128 + row, k = token quad
                float4* dst = reinterpret_cast<float4*>(part + (size_t)(cta * 2 + myslot) * (N * 128)) + row;
#pragma unroll
                for (int k = 0; k < N / 4; ++k)
                    dst[k * 128] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
                __threadfence();
                named_bar_sync(1, 128);
                if (et == 0) {
                    BFFN_TRACE_ONCE(sg.kind == 0 ? kTrAPartial : kTrBPartial);
                    atomicAdd(cnt, 1u);
                    BFFN_TRACE_ONCE(sg.kind == 0 ? kTrAArrive : kTrBArrive);
                }
                if (npend < 2) {
                    pend_sg[npend] = sg;
                    pend_cb[npend] = cb;
                    ++npend;
                }
            }
        }
        if (!failed) flush_pending();
        if (et == 0) BFFN_TRACE(kTrLastEpi);
    }

    // ------------------------------------------------------------ teardown --
    __syncthreads();
    if (threadIdx.x == 0) BFFN_TRACE(kTrTeardown);
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
        BFFN_TRACE(kTrEnd);
    }
}

size_t forward_tc_smem_bytes() { return 1024 + (size_t)kStages * kStageBytes + sizeof(TcShared); }

template <int N>
static cudaError_t launch_n(const TcArgs& a, const CUtensorMap* maps, int grid, cudaStream_t s) {
    const size_t smem = forward_tc_smem_bytes();
    cudaError_t err = cudaFuncSetAttribute(union_expert_forward_tc<N>,
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
    return cudaLaunchKernelEx(&cfg, union_expert_forward_tc<N>, maps[0], maps[1], maps[2], a);
}

cudaError_t launch_forward_tc(const TcArgs& a, const CUtensorMap* maps, int grid, cudaStream_t s) {
    if (a.N == 32) return launch_n<32>(a, maps, grid, s);
    if (a.N == 16) return launch_n<16>(a, maps, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace bffn
