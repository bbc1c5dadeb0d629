// forward_decode.cu -- the single-chunk (decode / verification step) forward on
// sm_100a.
//
// Pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device
// Deployment", Core Concept (for n tokens at once only the union of their
// activated experts is computed; unneeded activations are masked after
// computing) and Architecture Overview (non-gated Swish experts, d_e << d_h);
// the gated outputs are summed over experts (Full BlockFFN Layer with Combined
// Losses).
//
// One chunk of n <= 32 tokens; every block forms the chunk's union U (ascending)
// from the gates itself.
//
// Expert-in (A).  Blocks work in pairs (thread-block clusters of 2).  A unit is
// one union expert e and one 128-row tile of W_in_e (d_e = 128: the whole
// expert); pair c takes the units c, c + #pairs, ..., and its block of rank r
// multiplies the k-half r of W_in_e (tcgen05; weights as the M = 128 operand,
// the chunk's N tokens as N) into a TMEM accumulator.  The two partial h^T tiles
// meet in distributed shared memory: rank r adds them for rows [64r, 64r + 64),
// applies the post-hoc mask, the gate and Swish, writes those rows of h' (bf16)
// to global memory and counts them in for the expert.  With up to ~74 union
// experts about one unit per pair, and each block streams its A tiles first;
// a stage is a 16 KB weight tile and the 4 KB x tile that multiplies it.
// Expert-out (B).  y^T = sum_e W_out_e h'_e^T with W_out_e's 128-row tiles as
// the M operand and the tokens as N.  Tiles (row tile, expert, 64-wide k-block)
// are cut into contiguous ranges, one per block, sized so every block moves the
// same number of weight bytes counting its A work.  A tile waits (bounded) until
// all quarters of its expert are counted in, then its h' slice is copied into
// the stage with cp.async.  A row tile split across blocks is finished in two
// passes: every contributor publishes its partial tile, then each sums one
// slice of rows over all the partials in block order (a fixed order).
//
// Roles (224 threads): warp 0 TMA producer, warp 1 MMA issuer, warp 2 TMEM owner
// and h' loader, warps 3-6 epilogue (warp 4 also finishes the A units).  Every
// wait is bounded; a timeout records BLOCKFFN_ERR_TIMEOUT and the block winds
// down without leaving copies in flight.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace bffn {

constexpr int kRsThreads = 224;
constexpr int kRsStages = 10;
constexpr int kRsStageBytes = 16384 + 4096;  // weight tile [128 x 64] + activation tile [<=32 x 64]
constexpr int kRsNAccB = 4;                  // expert-out accumulators (32 columns each)
constexpr int kRsTmemCols = 256;             // 2 x 32 expert-in + 4 x 32 expert-out columns
constexpr int kRsMaxE = 256;
constexpr int kRsMaxG = 160;
constexpr int kRsPartBytes = 16 * 128 * 4;   // fp32 partial h^T for the peer's half [<=16 tokens][128 rows]
constexpr int kRsHStageBytes = 16 * 128 * 2; // this block's half of h' [<=16 tokens][128 rows] bf16

struct RsShared {
    uint64_t full_w[kRsStages];   // TMA bytes landed
    uint64_t full_h[kRsStages];   // h' slice landed (B, TMA bytes) / nothing to copy (A, one arrival)
    uint64_t empty[kRsStages];    // MMAs reading the stage are done
    uint64_t accA_full[2];
    uint64_t accA_empty[2];
    uint64_t accB_full[kRsNAccB];
    uint64_t accB_empty[kRsNAccB];
    uint64_t part_ready;          // 2 arrivals: both blocks of the pair wrote their partial
    uint64_t part_free;           // 1 arrival: the peer finished reading this block's partial
    uint64_t mma_done;
    uint64_t a_pub;               // 1 arrival: this block's expert-in results are published
    uint32_t tmem_base;
    volatile int abort;
    uint32_t epoch;
    int P;
    int ep_wait[2];
    int ep_ok;
    uint32_t trace_once;          // trace slots already stamped (first occurrence only)
    float s_gate[2][32];          // gates of the current expert-in unit's expert, per token
    int s_contrib[kRsMaxG];
    long long s_blo[kRsMaxG + 1];   // first expert-out tile of every block
    int32_t s_pair_e[kRsMaxE];
    uint32_t s_tmask[kRsMaxE];
    uint32_t s_bal[kRsMaxE / 32];
};

enum : int {
    kRtStart = 0, kRtPrologue = 1, kRtFirstLoad = 2, kRtLastLoad = 3, kRtFirstFull = 4,
    kRtLastACommit = 5, kRtADone = 7, kRtFirstFlag = 8, kRtLastFlag = 9, kRtLastCommit = 10,
    kRtLastEpi = 11, kRtEnd = 13, kRtATmem = 14, kRtAPart = 15, kRtAReady = 16, kRtARead = 17,
    kRtAWritten = 18, kRtBPartial = 21, kRtBReduced = 23, kRtFirstBMma = 24, kRtSlots = 64
};
#define RS_TRACE(slot) \
    do { if (a.trace) a.trace[(size_t)blockIdx.x * kRtSlots + (slot)] = globaltimer_ns(); } while (0)
#define RS_TRACE_ONCE(slot)                                                            \
    do {                                                                               \
        if (a.trace && !(atomicOr(&sh.trace_once, 1u << (slot)) & (1u << (slot))))     \
            a.trace[(size_t)blockIdx.x * kRtSlots + (slot)] = globaltimer_ns();        \
    } while (0)

__device__ __forceinline__ float rs_swish(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// block holding expert-out tile j: the last i with blo[i] <= j (ranges may be empty)
__device__ __forceinline__ int rs_owner(const long long* blo, int G, long long j) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (blo[mid] <= j) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Position in the ring of pipeline stages: the stage and the parity of its
// current use, stepped without divisions.
struct RingPos {
    int st = 0;
    uint32_t ph = 0u;
    __device__ __forceinline__ void advance() {
        if (++st == kRsStages) {
            st = 0;
            ph ^= 1u;
        }
    }
};

// Expert-out tile j = (rt * P + s) * KBe + kb (row tile, expert slot, k-block),
// stepped without divisions.
struct BTile {
    int rt, s, kb;
    __device__ __forceinline__ void init(long long j, int P, int KBe) {
        const long long per = (long long)P * KBe;
        rt = (int)(j / per);
        const int rem = (int)(j - (long long)rt * per);
        s = rem / KBe;
        kb = rem - s * KBe;
    }
    __device__ __forceinline__ void advance(int P, int KBe) {
        if (++kb == KBe) {
            kb = 0;
            if (++s == P) {
                s = 0;
                ++rt;
            }
        }
    }
};

template <int N>
__global__ void __launch_bounds__(kRsThreads, 1)
union_expert_decode(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_win,
                    const __grid_constant__ CUtensorMap tm_wout, const __grid_constant__ CUtensorMap tm_h,
                    const DcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float* part = reinterpret_cast<float*>(smem + kRsStages * kRsStageBytes);     // [N][128] fp32
    __nv_bfloat16* hstage = reinterpret_cast<__nv_bfloat16*>(smem + kRsStages * kRsStageBytes + kRsPartBytes);
    RsShared& sh = *reinterpret_cast<RsShared*>(smem + kRsStages * kRsStageBytes + kRsPartBytes + kRsHStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, cta = blockIdx.x;
    const int KBe = a.d_e / 64;     // 64-wide k-blocks of one expert in the expert-out GEMM
    const int MT = a.d_e / 128;     // 128-row tiles of W_in_e
    const int KBh = a.KB / 2;       // k-tiles of one k-half
    const int NCL = G / 2;          // pairs
    const int pr = cta >> 1;        // this block's pair
    const int hk = cta & 1;         // its rank in the pair = its k-half

    if (threadIdx.x == 0) {
        RS_TRACE(kRtStart);
        for (int s = 0; s < kRsStages; ++s) {
            mbar_init(&sh.full_w[s], 1);
            mbar_init(&sh.full_h[s], 1);
            mbar_init(&sh.empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sh.accA_full[s], 1);
            mbar_init(&sh.accA_empty[s], 1);
        }
        for (int s = 0; s < kRsNAccB; ++s) {
            mbar_init(&sh.accB_full[s], 1);
            mbar_init(&sh.accB_empty[s], 4);
        }
        mbar_init(&sh.part_ready, 2);
        mbar_init(&sh.part_free, 1);
        mbar_init(&sh.mma_done, 1);
        mbar_init(&sh.a_pub, 1);
        sh.trace_once = 0u;
        fence_mbar_init();
        const int32_t st0 = __ldcg(&a.ctl->status);
        const uint32_t ep0 = __ldcg(&a.ctl->epoch);
        sh.abort = st0 != 0;
        sh.epoch = ep0;
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_win);
        prefetch_tmap(&tm_wout);
        prefetch_tmap(&tm_h);
    }
    if (warp == 2) {
        tmem_alloc(&sh.tmem_base, kRsTmemCols);
        tmem_relinquish();
    }
    if (warp >= 3) {
        // the chunk's union, ascending (warps 3-6 take 32-expert groups; all of a
        // lane's gate loads are issued before their first use)
        const int nt = min(a.n, a.T);
        const int ngroups = (a.E + 31) / 32;
        for (int g = warp - 3; g < ngroups; g += 4) {
            const int e = g * 32 + lane;
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
        }
        named_bar_sync(1, 128);
        if (warp == 3) {
            int base = 0;
            for (int g = 0; g < ngroups; ++g) {
                const uint32_t bal = sh.s_bal[g];
                if ((bal >> lane) & 1u) sh.s_pair_e[base + __popc(bal & ((1u << lane) - 1u))] = g * 32 + lane;
                base += __popc(bal);
            }
            if (lane == 0) sh.P = base;
            // Expert-out tile ranges: an even split over all blocks.  The expert-out
            // MMAs all run after the h' hand-off, so it is their count per block
            // that sets the length of that phase; the expert-in blocks load their
            // share after publishing h' (their weights were sent towards L2 early).
            const long long NB = (long long)a.RT * base * KBe;
            for (int i = lane; i < G; i += 32) sh.s_blo[i] = NB * i / G;
            if (lane == 0) sh.s_blo[G] = NB;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_barrier_sync();   // the peer's barriers are initialised before any remote arrival
    if (threadIdx.x == 0) RS_TRACE(kRtPrologue);

    const uint32_t tmem = sh.tmem_base;
    const int P = sh.P;
    const int par = (int)(sh.epoch & 1u);
    uint32_t* const readyA = a.readyA + (size_t)par * a.E;
    const int VA = P * MT;                                          // A units (expert, 128-row tile)
    const int nA = VA / NCL + (pr < VA % NCL ? 1 : 0);               // A units of this pair
    const long long bLo = sh.s_blo[cta], bHi = sh.s_blo[cta + 1];
    const long long per_rt = (long long)P * KBe;                     // expert-out tiles per row tile
    const uint64_t limit_peer = a.wait_ns;
    const uint64_t limit = 2 * a.wait_ns;
    const uint32_t accA_col = 0, accB_col = 64;

    // expert-out segments: a row tile rt is the unit, tiles [rt*per_rt, (rt+1)*per_rt)
    auto seg_of = [&](long long j, long long& first, long long& last, int& rt) {
        rt = (int)(j / per_rt);
        first = (long long)rt * per_rt;
        last = first + per_rt - 1;
    };

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer --
        if (lane == 0 && !sh.abort) {
            const uint64_t pol_stream = policy_evict_first();
            const uint64_t pol_keep = policy_evict_last();
            long long i = 0;
            RingPos rp;
            bool stop = false;
            for (int ua = 0; ua < nA && !stop; ++ua) {
                const int v = pr + ua * NCL;
                const int e = sh.s_pair_e[v / MT], mt = v % MT;
                for (int t = 0; t < KBh; ++t, ++i, rp.advance()) {
                    const int kt = hk * KBh + t;
                    if (!wait_bar(&sh.empty[rp.st], rp.ph ^ 1u, limit, &sh.abort, a.ctl, kWaitEmpty)) {
                        stop = true;
                        break;
                    }
                    uint8_t* w = smem + rp.st * kRsStageBytes;
                    mbar_arrive_expect_tx(&sh.full_w[rp.st], 16384 + N * 128);
                    tma_load_2d(w, &tm_win, &sh.full_w[rp.st], kt * 64, e * a.d_e + mt * 128, pol_stream);
                    tma_load_2d(w + 16384, &tm_x, &sh.full_w[rp.st], kt * 64, 0, pol_keep);
                    if (i == 0) RS_TRACE(kRtFirstLoad);
                }
            }
            // Expert-out weights.  A block with expert-in units sends all of its
            // tiles towards L2 now and loads them into the ring only after its h' is
            // published: a release waits for the block's bulk loads in flight, and
            // no expert-out MMA can start before every h' is out anyway.  Other
            // blocks load at once and prefetch what the ring cannot hold yet.
            {
                const long long nB = bHi - bLo;
                const long long j0 = nA > 0 ? bLo : bHi - min(nB, max(0LL, nB - (long long)kRsStages));
                if (j0 < bHi) {
                    BTile bt;
                    bt.init(j0, P, KBe);
                    for (long long j = j0; j < bHi; ++j, bt.advance(P, KBe))
                        tma_prefetch_l2_2d(&tm_wout, bt.kb * 64, sh.s_pair_e[bt.s] * a.d_h + bt.rt * 128);
                }
                if (nA > 0 && bLo < bHi && !stop &&
                    !wait_bar(&sh.a_pub, 0u, limit, &sh.abort, a.ctl, kWaitEmpty))
                    stop = true;
            }
            if (bLo < bHi) {
                BTile bt;
                bt.init(bLo, P, KBe);
                for (long long j = bLo; j < bHi && !stop; ++j, ++i, rp.advance(), bt.advance(P, KBe)) {
                    if (!wait_bar(&sh.empty[rp.st], rp.ph ^ 1u, limit, &sh.abort, a.ctl, kWaitEmpty)) {
                        stop = true;
                        break;
                    }
                    mbar_arrive_expect_tx(&sh.full_w[rp.st], 16384);
                    tma_load_2d(smem + rp.st * kRsStageBytes, &tm_wout, &sh.full_w[rp.st], bt.kb * 64,
                                sh.s_pair_e[bt.s] * a.d_h + bt.rt * 128, pol_stream);
                    if (i == 0) RS_TRACE(kRtFirstLoad);
                }
            }
            RS_TRACE(kRtLastLoad);
            for (long long q = i - kRsStages < 0 ? 0 : i - kRsStages; q < i; ++q)
                wait_bar_drain(&sh.full_w[q % kRsStages], (uint32_t)((q / kRsStages) & 1), limit, a.ctl);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer --
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(128, N);     // 128 weight rows x tokens
            long long i = 0;
            RingPos rp;
            bool stop = sh.abort != 0;
            for (int ua = 0; ua < nA && !stop; ++ua) {
                const int ab = ua & 1;
                if (!wait_bar(&sh.accA_empty[ab], (uint32_t)(((ua >> 1) & 1) ^ 1), limit, &sh.abort, a.ctl,
                              kWaitAccEmpty))
                    break;
                tc_fence_after();
                const uint32_t d = tmem + accA_col + (uint32_t)(ab * 32);
                for (int t = 0; t < KBh; ++t, ++i, rp.advance()) {
                    const int st = rp.st;
                    if (!wait_bar(&sh.full_w[st], rp.ph, limit, &sh.abort, a.ctl, kWaitFullW) ||
                        !wait_bar(&sh.full_h[st], rp.ph, limit, &sh.abort, a.ctl, kWaitFullH)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    if (i == 0) RS_TRACE(kRtFirstFull);
                    const uint32_t wb = smem_u32(smem + st * kRsStageBytes);
                    const uint32_t xb = wb + 16384;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(d, sw128_kmajor_desc(wb + kk * 32), sw128_kmajor_desc(xb + kk * 32), idesc,
                                  (t > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&sh.empty[st]);
                }
                if (stop) break;
                umma_commit(&sh.accA_full[ab]);
                RS_TRACE(kRtLastACommit);
            }
            uint32_t acc_i = 0;
            long long j = bLo;
            while (!stop && j < bHi) {
                long long first, last;
                int rt;
                seg_of(j, first, last, rt);
                const long long shi = min(bHi, last + 1);
                const int ab = (int)(acc_i % kRsNAccB);
                if (!wait_bar(&sh.accB_empty[ab], ((acc_i / kRsNAccB) & 1u) ^ 1u, limit, &sh.abort, a.ctl,
                              kWaitAccEmpty))
                    break;
                tc_fence_after();
                const uint32_t d = tmem + accB_col + (uint32_t)(ab * 32);
                for (long long jj = j; jj < shi; ++jj, ++i, rp.advance()) {
                    const int st = rp.st;
                    if (!wait_bar(&sh.full_w[st], rp.ph, limit, &sh.abort, a.ctl, kWaitFullW) ||
                        !wait_bar(&sh.full_h[st], rp.ph, limit, &sh.abort, a.ctl, kWaitFullH)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    if (jj == bLo) RS_TRACE(kRtFirstBMma);
                    const uint32_t wb = smem_u32(smem + st * kRsStageBytes);
                    const uint32_t hb = wb + 16384;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(d, sw128_kmajor_desc(wb + kk * 32), sw128_kmajor_desc(hb + kk * 32), idesc,
                                  (jj > j || kk > 0) ? 1u : 0u);
                    umma_commit(&sh.empty[st]);
                }
                if (stop) break;
                umma_commit(&sh.accB_full[ab]);
                RS_TRACE(kRtLastCommit);
                ++acc_i;
                j = shi;
            }
            umma_commit(&sh.mma_done);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------- h' loader --
        // A stages carry no h': lane 0 just arrives.  Before the first expert-out
        // tile the warp waits (bounded) until every expert slot's h' is counted in;
        // then lane 0 moves each tile's [N x 64] h' slice with one TMA load, which
        // lands in the same 128-byte-swizzled layout as the weight tile's operand.
        const long long nAt = (long long)nA * KBh;
        const long long total_tiles = nAt + (bHi - bLo);
        long long i = 0;
        RingPos rp;
        int stop = sh.abort != 0;
        if (lane == 0) {
            for (; i < nAt; ++i, rp.advance()) {
                if (!wait_bar(&sh.empty[rp.st], rp.ph ^ 1u, limit, &sh.abort, a.ctl, kWaitEmpty)) {
                    stop = 1;
                    break;
                }
                mbar_arrive(&sh.full_h[rp.st]);
            }
        }
        stop = __shfl_sync(0xffffffffu, stop, 0);
        if (!stop && total_tiles > nAt) {
            // The expert-in units all finish at about the same time, so one combined
            // wait costs no more than the slowest slot; each poll round checks 32
            // slots at once (one acquire load per lane).
            const uint64_t t0 = globaltimer_ns();
            bool done = false;
            while (!done) {
                bool mine_ok = true;
                for (int q = lane; q < P; q += 32)
                    if (ld_acquire_gpu(&readyA[q]) < (uint32_t)(2 * MT)) mine_ok = false;
                done = __all_sync(0xffffffffu, mine_ok);
                if (done) break;
                __nanosleep(64);
                if (__any_sync(0xffffffffu, sh.abort != 0)) break;
                if (globaltimer_ns() - t0 > limit_peer) {
                    if (lane == 0) {
                        record_error(a.ctl, kErrTimeout, kWaitFlag);
                        sh.abort = 1;
                    }
                    break;
                }
            }
            __syncwarp();
            if (lane == 0 && done) {
                // the h' stores were made visible to this thread by the acquires; the
                // async proxy reads them next
                fence_proxy_async_global();
                RS_TRACE_ONCE(kRtFirstFlag);
                RS_TRACE(kRtLastFlag);
                const uint64_t pol = policy_evict_first();
                BTile bt;
                bt.init(bLo, P, KBe);
                for (; i < total_tiles; ++i, rp.advance(), bt.advance(P, KBe)) {
                    if (!wait_bar(&sh.empty[rp.st], rp.ph ^ 1u, limit, &sh.abort, a.ctl, kWaitEmpty)) break;
                    mbar_arrive_expect_tx(&sh.full_h[rp.st], (uint32_t)(N * 128));
                    tma_load_2d(smem + rp.st * kRsStageBytes + 16384, &tm_h, &sh.full_h[rp.st], bt.kb * 64,
                                bt.s * N, pol);
                }
                // no copy into this block's shared memory outlives it
                for (long long q = i - kRsStages < nAt ? nAt : i - kRsStages; q < i; ++q)
                    wait_bar_drain(&sh.full_h[q % kRsStages], (uint32_t)((q / kRsStages) & 1), limit, a.ctl);
            }
        }
    } else {
        // --------------------------------------------------------- epilogue --
        const int qd = warp & 3;
        const int row = qd * 32 + lane;              // TMEM lane = accumulator row
        const int et = threadIdx.x - 96;             // 0..127
        {
            // zero the other parity's counters for the next launch
            const int oth = par ^ 1;
            for (int k2 = cta * 128 + et; k2 < a.E; k2 += G * 128) a.readyA[(size_t)oth * a.E + k2] = 0u;
        }
        bool failed = sh.abort != 0;
        const int nt = min(a.n, a.T);
        if (P == 0 && cta == 0 && !failed) {
            // empty union: y is all zeros
            for (size_t k2 = et; k2 < (size_t)nt * a.d_h; k2 += 128) a.y[k2] = __float2bfloat16_rn(0.f);
        }
        // ---- A units: the pair's two k-half partials meet in shared memory
        {
            const uint32_t peer = (uint32_t)(hk ^ 1);
            const uint32_t peer_part = mapa_shared(smem_u32(part), peer);
            const uint32_t peer_ready = mapa_shared(smem_u32(&sh.part_ready), peer);
            const uint32_t own_ready = mapa_shared(smem_u32(&sh.part_ready), (uint32_t)hk);
            const uint32_t peer_free = mapa_shared(smem_u32(&sh.part_free), peer);
            for (int ua = 0; ua < nA && !failed; ++ua) {
                const int ab = ua & 1;
                const int v = pr + ua * NCL;
                const int s = v / MT, mt = v % MT;
                const int e = sh.s_pair_e[s];
                // stage the unit's gates now: the accumulator wait hides their latency,
                // and the activation loop below then reads shared memory only
                if (et < 32) sh.s_gate[ab][et] = a.gates[(size_t)min(et, nt - 1) * a.E + e];
                if (et == 0) {
                    int ok = wait_bar(&sh.accA_full[ab], (uint32_t)((ua >> 1) & 1), limit, &sh.abort, a.ctl,
                                      kWaitAccFull) ? 1 : 0;
                    // the peer finished reading this block's previous partial
                    if (ok && ua > 0)
                        ok = wait_bar_cluster(&sh.part_free, (uint32_t)((ua - 1) & 1), limit_peer, &sh.abort,
                                              a.ctl, kWaitPeers) ? 1 : 0;
                    sh.ep_ok = ok;
                }
                named_bar_sync(1, 128);
                if (!sh.ep_ok) { failed = true; break; }
                tc_fence_after();
                uint32_t r[32];
                const uint32_t taddr = tmem + ((uint32_t)(qd * 32) << 16) + accA_col + (uint32_t)(ab * 32);
                if constexpr (N == 32) tmem_ld_32x32b_x32(taddr, r);
                else tmem_ld_32x32b_x16(taddr, r);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.accA_empty[ab]);
                if (et == 0) RS_TRACE_ONCE(kRtATmem);
                // The pair splits the chunk's tokens: this block finishes tokens
                // [tg, tg + NH) of all 128 rows and the peer the other half.  Each block
                // hands the peer its partial for the peer's tokens: float4 of the half's
                // tokens 4k..4k+3 of a row at k*128 + row.
                constexpr int NH = N / 2;
                const int tg = hk * NH;
                {
                    float4* p4 = reinterpret_cast<float4*>(part) + row;
#pragma unroll
                    for (int k4 = 0; k4 < NH / 4; ++k4) {
                        float f[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            f[u] = __uint_as_float(hk ? r[4 * k4 + u] : r[NH + 4 * k4 + u]);
                        p4[k4 * 128] = make_float4(f[0], f[1], f[2], f[3]);
                    }
                }
                const uint32_t bits = sh.s_tmask[e] >> tg;   // this half's token bits
                named_bar_sync(1, 128);
                if (et == 0) {
                    RS_TRACE_ONCE(kRtAPart);
                    mbar_arrive_cluster(own_ready);
                    mbar_arrive_cluster(peer_ready);
                    sh.ep_ok = wait_bar_cluster(&sh.part_ready, (uint32_t)(ua & 1), limit_peer, &sh.abort, a.ctl,
                                                kWaitPeers) ? 1 : 0;
                    RS_TRACE_ONCE(kRtAReady);
                }
                named_bar_sync(1, 128);
                if (!sh.ep_ok) { failed = true; break; }
                // h = (k-half 0) + (k-half 1): two terms, and the sum does not depend on
                // which block of the pair forms it
                float z[NH];
                {
                    float4 pv[NH / 4];
#pragma unroll
                    for (int k4 = 0; k4 < NH / 4; ++k4)
                        pv[k4] = ld_shared_cluster_f4(peer_part + (uint32_t)((k4 * 128 + row) * 16));
#pragma unroll
                    for (int k4 = 0; k4 < NH / 4; ++k4) {
                        const float pw[4] = {pv[k4].x, pv[k4].y, pv[k4].z, pv[k4].w};
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            z[4 * k4 + u] = __uint_as_float(hk ? r[NH + 4 * k4 + u] : r[4 * k4 + u]) + pw[u];
                    }
                }
                named_bar_sync(1, 128);
                if (et == 0) {
                    RS_TRACE_ONCE(kRtARead);
                    mbar_arrive_cluster(peer_free);   // done with the peer's partial
                }
                // h' = bit ? g * Swish(h) : 0 (a select, so a masked token gives 0 even if
                // its h is not finite), staged token-major in shared memory, then written
                // with 16-byte stores: token t's 128 rows are 256 contiguous bytes
                {
                    __nv_bfloat16* stg = hstage + row;
#pragma unroll
                    for (int tl = 0; tl < NH; ++tl) {
                        const float gsw = sh.s_gate[ab][tg + tl] * rs_swish(z[tl]);
                        stg[tl * 128] = __float2bfloat16_rn(((bits >> tl) & 1u) ? gsw : 0.f);
                    }
                }
                named_bar_sync(1, 128);
                {
                    const uint4* src4 = reinterpret_cast<const uint4*>(hstage);
                    for (int c = et; c < NH * 16; c += 128) {
                        const int tl = c >> 4, c16 = c & 15;
                        uint4* dst4 =
                            reinterpret_cast<uint4*>(a.hbuf + ((size_t)s * N + tg + tl) * a.d_e + mt * 128) + c16;
                        *dst4 = src4[c];
                    }
                }
                // one release for the whole block: the barrier orders every thread's
                // stores before thread 0's releasing count
                named_bar_sync(1, 128);
                if (et == 0) {
                    if ((v * 2 + hk) != a.skip_unit) red_release_add_gpu(&readyA[s], 1u);
                    RS_TRACE_ONCE(kRtAWritten);
                }
            }
            if (et == 0) {
                RS_TRACE(kRtADone);
                if (nA > 0) mbar_arrive(&sh.a_pub);   // the producer may load expert-out tiles now
            }
        }
        // ---- expert-out row tiles.  A row tile whose k-range is split over several
        // blocks is summed without a flag: every contributor stores its partial as
        // (launch tag, fp32) pairs with relaxed stores, and the block that sums a
        // slice of the tile's rows polls those pairs until each carries this
        // launch's tag, then adds the contributors in block order.
        const uint32_t tag = sh.epoch + 1u;
        const unsigned long long tag_hi = (unsigned long long)tag << 32;
        const size_t slot_pairs = (size_t)(N / 2) * 128;   // 16-byte pairs in one partial slot
        ulonglong2* const partD = reinterpret_cast<ulonglong2*>(a.partD);
        auto contributors = [&](long long first, long long last, int& q0, int& q1, int& n, int& rank) {
            q0 = rs_owner(sh.s_blo, G, first);
            q1 = rs_owner(sh.s_blo, G, last);
            n = 0;
            rank = -1;
            for (int qq = q0; qq <= q1; ++qq) {
                if (sh.s_blo[qq + 1] > sh.s_blo[qq]) {
                    if (qq == cta) rank = n;
                    ++n;
                }
            }
        };
        long long pend_first[2], pend_last[2];
        int pend_rt[2];
        int npend = 0;
        uint32_t acc_i = 0;
        long long j = bLo;
        failed = failed || sh.abort;
        while (!failed && j < bHi) {
            long long first, last;
            int rt;
            seg_of(j, first, last, rt);
            const long long shi = min(bHi, last + 1);
            const int ab = (int)(acc_i % kRsNAccB);
            if (et == 0)
                sh.ep_wait[acc_i & 1u] =
                    wait_bar(&sh.accB_full[ab], (acc_i / kRsNAccB) & 1u, limit, &sh.abort, a.ctl, kWaitAccFull)
                        ? 1 : 0;
            named_bar_sync(1, 128);
            if (!sh.ep_wait[acc_i & 1u]) { failed = true; break; }
            tc_fence_after();
            uint32_t r[32];
            const uint32_t taddr = tmem + ((uint32_t)(qd * 32) << 16) + accB_col + (uint32_t)(ab * 32);
            if constexpr (N == 32) tmem_ld_32x32b_x32(taddr, r);
            else tmem_ld_32x32b_x16(taddr, r);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.accB_empty[ab]);
            ++acc_i;
            int q0, q1, nc, rank;
            contributors(first, last, q0, q1, nc, rank);
            if (nc == 1) {
                __nv_bfloat16* ycol = a.y + rt * 128 + row;
#pragma unroll
                for (int t = 0; t < N; ++t)
                    if (t < nt) ycol[(size_t)t * a.d_h] = __float2bfloat16_rn(__uint_as_float(r[t]));
                if (et == 0) RS_TRACE(kRtLastEpi);
            } else {
                // pair kp of a row holds tokens 2kp and 2kp+1: [kp][row] x 16 bytes
                const int myslot = bLo >= first ? 0 : 1;
                ulonglong2* dst = partD + (size_t)(cta * 2 + myslot) * slot_pairs + row;
#pragma unroll
                for (int kp = 0; kp < N / 2; ++kp)
                    st_relaxed_v2_b64(dst + kp * 128, tag_hi | r[2 * kp], tag_hi | r[2 * kp + 1]);
                if (et == 0) RS_TRACE_ONCE(kRtBPartial);
                if (npend < 2) {
                    pend_first[npend] = first;
                    pend_last[npend] = last;
                    pend_rt[npend] = rt;
                    ++npend;
                }
            }
            j = shi;
        }
        // second pass: sum my slice of each split row tile's rows
        for (int pi = 0; pi < npend && !failed; ++pi) {
            int q0, q1, nc, rank;
            contributors(pend_first[pi], pend_last[pi], q0, q1, nc, rank);
            const int rt = pend_rt[pi];
            if (et == 0) {
                int k2 = 0;
                for (int qq = q0; qq <= q1 && k2 < kRsMaxG; ++qq)
                    if (sh.s_blo[qq + 1] > sh.s_blo[qq])
                        sh.s_contrib[k2++] = qq * 2 + (sh.s_blo[qq] >= pend_first[pi] ? 0 : 1);
            }
            named_bar_sync(1, 128);
            const int r0 = rank * 128 / nc, r1 = (rank + 1) * 128 / nc, nrows = r1 - r0;
            const int nitems = nrows * (N / 2);
            const uint64_t t0 = globaltimer_ns();
            for (int it = et; it < nitems && !failed; it += 128) {
                const int rr = r0 + it % nrows, kp = it / nrows;
                float sx = 0.f, sy = 0.f;
                for (int c0 = 0; c0 < nc && !failed; c0 += 8) {
                    const ulonglong2* src[8];
                    ulonglong2 v[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        src[u] = partD + (size_t)sh.s_contrib[min(c0 + u, nc - 1)] * slot_pairs + kp * 128 + rr;
                        v[u] = ld_relaxed_v2_b64(src[u]);
                    }
                    while (true) {   // re-read the pairs that are not this launch's yet (bounded)
                        bool all = true;
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            if ((uint32_t)(v[u].x >> 32) != tag || (uint32_t)(v[u].y >> 32) != tag) {
                                all = false;
                                v[u] = ld_relaxed_v2_b64(src[u]);
                            }
                        if (all) break;
                        if (sh.abort) { failed = true; break; }
                        if (globaltimer_ns() - t0 > limit_peer) {
                            record_error(a.ctl, kErrTimeout, kWaitPeers);
                            sh.abort = 1;
                            failed = true;
                            break;
                        }
                    }
                    if (failed) break;
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        if (c0 + u < nc) {
                            sx += __uint_as_float((uint32_t)v[u].x);
                            sy += __uint_as_float((uint32_t)v[u].y);
                        }
                }
                if (failed) break;
                __nv_bfloat16* ycol = a.y + rt * 128 + rr;
                if (2 * kp < nt) ycol[(size_t)(2 * kp) * a.d_h] = __float2bfloat16_rn(sx);
                if (2 * kp + 1 < nt) ycol[(size_t)(2 * kp + 1) * a.d_h] = __float2bfloat16_rn(sy);
            }
            if (et == 0) RS_TRACE_ONCE(kRtBReduced);
        }
        if (et == 0) {
            RS_TRACE(kRtLastEpi);
            // the peer may still read this block's last partial
            if (nA > 0 && !failed)
                wait_bar_cluster(&sh.part_free, (uint32_t)((nA - 1) & 1), limit_peer, &sh.abort, a.ctl, kWaitPeers);
        }
    }

    // --------------------------------------------------------------- teardown --
    __syncthreads();
    if (warp == 2) {
        if (lane == 0) wait_bar_drain(&sh.mma_done, 0, 2 * a.wait_ns, a.ctl);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kRsTmemCols);
    }
    if (threadIdx.x == 0) {
        __threadfence();
        const uint32_t old = atomicAdd(&a.ctl->done, 1u);
        if (old == (uint32_t)(G - 1)) {
            a.ctl->done = 0u;
            atomicExch(&a.ctl->epoch, sh.epoch + 1u);
        }
        RS_TRACE(kRtEnd);
    }
    // no block leaves while its peer might still use its shared memory
    cluster_barrier_sync();
}

size_t forward_decode_smem_bytes() {
    return 1024 + (size_t)kRsStages * kRsStageBytes + kRsPartBytes + kRsHStageBytes + sizeof(RsShared);
}

template <int N>
static cudaError_t launch_decode_n(const DcArgs& a, const CUtensorMap* maps, int grid, cudaStream_t s,
                                   bool cooperative) {
    const size_t smem = forward_decode_smem_bytes();
    cudaError_t err =
        cudaFuncSetAttribute(union_expert_decode<N>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kRsThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = cooperative ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, union_expert_decode<N>, maps[0], maps[1], maps[2], maps[3], a);
}

cudaError_t launch_forward_decode(const DcArgs& a, const CUtensorMap* maps, int grid, cudaStream_t s,
                                  bool cooperative) {
    if (a.N == 32) return launch_decode_n<32>(a, maps, grid, s, cooperative);
    if (a.N == 16) return launch_decode_n<16>(a, maps, grid, s, cooperative);
    return cudaErrorInvalidValue;
}

// Pairs of blocks (one block per SM) that can be resident at once, -1 on error.
int decode_max_pairs() {
    const size_t smem = forward_decode_smem_bytes();
    if (cudaFuncSetAttribute(union_expert_decode<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return -1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kRsThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, union_expert_decode<32>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    return n;
}

}  // namespace bffn
