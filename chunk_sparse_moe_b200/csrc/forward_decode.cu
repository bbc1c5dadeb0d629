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
constexpr int kRsPartBytes = 32 * 128 * 4;   // one fp32 partial h^T tile [<=32 tokens][128 rows]

struct RsShared {
    uint64_t full_w[kRsStages];   // TMA bytes landed
    uint64_t full_h[kRsStages];   // 32 arrivals: h' copies landed (B) / nothing to copy (A)
    uint64_t empty[kRsStages];    // MMAs reading the stage are done
    uint64_t accA_full[2];
    uint64_t accA_empty[2];
    uint64_t accB_full[kRsNAccB];
    uint64_t accB_empty[kRsNAccB];
    uint64_t part_ready;          // 2 arrivals: both blocks of the pair wrote their partial
    uint64_t part_free;           // 1 arrival: the peer finished reading this block's partial
    uint64_t mma_done;
    uint32_t tmem_base;
    volatile int abort;
    uint32_t epoch;
    int P;
    int ep_wait[2];
    int ep_ok;
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
    kRtAWritten = 18, kRtBPartial = 21, kRtBArrive = 22, kRtBReduced = 23, kRtFirstBMma = 24, kRtSlots = 32
};
#define RS_TRACE(slot) \
    do { if (a.trace) a.trace[(size_t)blockIdx.x * kRtSlots + (slot)] = globaltimer_ns(); } while (0)
#define RS_TRACE_ONCE(slot)                                                            \
    do {                                                                               \
        if (a.trace && a.trace[(size_t)blockIdx.x * kRtSlots + (slot)] == 0ull)        \
            a.trace[(size_t)blockIdx.x * kRtSlots + (slot)] = globaltimer_ns();        \
    } while (0)

__device__ __forceinline__ float rs_swish(float z) { return z / (1.0f + __expf(-z)); }

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

template <int N>
__global__ void __launch_bounds__(kRsThreads, 1)
union_expert_decode(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_win,
                    const __grid_constant__ CUtensorMap tm_wout, const DcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float* part = reinterpret_cast<float*>(smem + kRsStages * kRsStageBytes);     // [N][128] fp32
    RsShared& sh = *reinterpret_cast<RsShared*>(smem + kRsStages * kRsStageBytes + kRsPartBytes);
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
            mbar_init(&sh.full_h[s], 32);
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
        fence_mbar_init();
        const int32_t st0 = __ldcg(&a.ctl->status);
        const uint32_t ep0 = __ldcg(&a.ctl->epoch);
        sh.abort = st0 != 0;
        sh.epoch = ep0;
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_win);
        prefetch_tmap(&tm_wout);
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
            // Expert-out tile ranges, weighted so that every block moves about the
            // same number of weight bytes (in tiles of 16 KB: an A k-tile or an
            // expert-out tile).  Pair c has VA/#pairs or one more A units, each
            // KB/2 k-tiles per block; a block's capacity is what the target leaves
            // (target = ceil(total / blocks), so the capacities cover all NB tiles);
            // a warp scan turns them into range starts, clipped at NB.
            const long long VA = (long long)base * (a.d_e / 128);
            const long long NB = (long long)a.RT * base * KBe;
            const long long npairs = G / 2;
            const long long total = VA * a.KB + NB;
            const long long target = (total + G - 1) / G;
            const long long q_ua = VA / npairs, r_ua = VA % npairs;
            long long run = 0;
            for (int b0 = 0; b0 < G; b0 += 32) {
                const int i = b0 + lane;
                long long cap = 0;
                if (i < G) {
                    const long long nAi = q_ua + ((i >> 1) < r_ua ? 1 : 0);
                    cap = target - nAi * (a.KB / 2);
                    if (cap < 0) cap = 0;
                }
                long long incl = cap;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const long long t = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += t;
                }
                // the capacities add up to at least NB; ranges stop at NB
                if (i < G) sh.s_blo[i] = min(NB, run + incl - cap);
                run += __shfl_sync(0xffffffffu, incl, 31);
            }
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
    uint32_t* const cntB = a.cntB + (size_t)par * a.RT;
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
            bool stop = false;
            for (int ua = 0; ua < nA && !stop; ++ua) {
                const int v = pr + ua * NCL;
                const int e = sh.s_pair_e[v / MT], mt = v % MT;
                for (int t = 0; t < KBh; ++t, ++i) {
                    const int kt = hk * KBh + t;
                    const int st = (int)(i % kRsStages);
                    if (!wait_bar(&sh.empty[st], (uint32_t)(((i / kRsStages) & 1) ^ 1), limit, &sh.abort, a.ctl,
                                  kWaitEmpty)) {
                        stop = true;
                        break;
                    }
                    uint8_t* w = smem + st * kRsStageBytes;
                    mbar_arrive_expect_tx(&sh.full_w[st], 16384 + N * 128);
                    tma_load_2d(w, &tm_win, &sh.full_w[st], kt * 64, e * a.d_e + mt * 128, pol_stream);
                    tma_load_2d(w + 16384, &tm_x, &sh.full_w[st], kt * 64, 0, pol_keep);
                    if (i == 0) RS_TRACE(kRtFirstLoad);
                }
            }
            // expert-out tiles beyond what the ring holds at once: start them
            // towards L2 now, so they are near when stages free up
            {
                const long long ahead = (long long)nA * KBh + (bHi - bLo) - kRsStages;
                for (long long j = bHi - (ahead > 0 ? min(ahead, bHi - bLo) : 0); j < bHi; ++j) {
                    const int rt = (int)(j / per_rt);
                    const int rem = (int)(j % per_rt);
                    tma_prefetch_l2_2d(&tm_wout, (rem % KBe) * 64, sh.s_pair_e[rem / KBe] * a.d_h + rt * 128);
                }
            }
            for (long long j = bLo; j < bHi && !stop; ++j, ++i) {
                const int rt = (int)(j / per_rt);
                const int rem = (int)(j % per_rt);
                const int e = sh.s_pair_e[rem / KBe], kb = rem % KBe;
                const int st = (int)(i % kRsStages);
                if (!wait_bar(&sh.empty[st], (uint32_t)(((i / kRsStages) & 1) ^ 1), limit, &sh.abort, a.ctl,
                              kWaitEmpty)) {
                    stop = true;
                    break;
                }
                mbar_arrive_expect_tx(&sh.full_w[st], 16384);
                tma_load_2d(smem + st * kRsStageBytes, &tm_wout, &sh.full_w[st], kb * 64, e * a.d_h + rt * 128,
                            pol_stream);
                if (i == 0) RS_TRACE(kRtFirstLoad);
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
            bool stop = sh.abort != 0;
            for (int ua = 0; ua < nA && !stop; ++ua) {
                const int ab = ua & 1;
                if (!wait_bar(&sh.accA_empty[ab], (uint32_t)(((ua >> 1) & 1) ^ 1), limit, &sh.abort, a.ctl,
                              kWaitAccEmpty))
                    break;
                tc_fence_after();
                const uint32_t d = tmem + accA_col + (uint32_t)(ab * 32);
                for (int t = 0; t < KBh; ++t, ++i) {
                    const int st = (int)(i % kRsStages);
                    const uint32_t ph = (uint32_t)((i / kRsStages) & 1);
                    if (!wait_bar(&sh.full_w[st], ph, limit, &sh.abort, a.ctl, kWaitFullW) ||
                        !wait_bar(&sh.full_h[st], ph, limit, &sh.abort, a.ctl, kWaitFullH)) {
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
                for (long long jj = j; jj < shi; ++jj, ++i) {
                    const int st = (int)(i % kRsStages);
                    const uint32_t ph = (uint32_t)((i / kRsStages) & 1);
                    if (!wait_bar(&sh.full_w[st], ph, limit, &sh.abort, a.ctl, kWaitFullW) ||
                        !wait_bar(&sh.full_h[st], ph, limit, &sh.abort, a.ctl, kWaitFullH)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    fence_proxy_async_smem();   // h' slices were written by cp.async
                    RS_TRACE_ONCE(kRtFirstBMma);
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
        // ------------------------------------------------ h' loader (whole warp) --
        // A stages carry no h': the 32 lanes just arrive.  An expert-out tile of
        // expert slot s waits (lane 0, bounded) until both halves of every 128-row
        // tile of s are counted in, then every lane copies its 16-byte pieces of the [N x 64]
        // slice with cp.async; each lane's arrival fires when its copies land.
        constexpr int kPieces = N * 8 / 32;
        long long i = 0;
        bool stop = sh.abort != 0;
        uint32_t seen[kRsMaxE / 32];
#pragma unroll
        for (int w = 0; w < kRsMaxE / 32; ++w) seen[w] = 0u;
        const long long nAt = (long long)nA * KBh;
        const long long total_tiles = nAt + (bHi - bLo);
        for (; i < total_tiles && !stop; ++i) {
            const int st = (int)(i % kRsStages);
            int ok = 1;
            if (lane == 0)
                ok = wait_bar(&sh.empty[st], (uint32_t)(((i / kRsStages) & 1) ^ 1), limit, &sh.abort, a.ctl,
                              kWaitEmpty) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            if (i < nAt) {
                mbar_arrive(&sh.full_h[st]);
                continue;
            }
            const long long j = bLo + (i - nAt);
            const int rem = (int)(j % per_rt);
            const int s = rem / KBe, kb = rem % KBe;
            // slots already seen complete need no further acquire (lane 0 keeps a
            // bitmask of them; after its acquire the warp barrier orders the
            // lanes' copies behind it)
            if (lane == 0 && !((seen[s >> 5] >> (s & 31)) & 1u)) {
                ok = wait_count(&readyA[s], (uint32_t)(2 * MT), limit_peer, &sh.abort, a.ctl, kWaitFlag) ? 1 : 0;
                if (ok) {
                    seen[s >> 5] |= 1u << (s & 31);
                    RS_TRACE_ONCE(kRtFirstFlag);
                    RS_TRACE(kRtLastFlag);
                }
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            const uint4* src = reinterpret_cast<const uint4*>(a.hbuf + (size_t)s * N * a.d_e + (size_t)kb * 64);
            uint8_t* dst = smem + st * kRsStageBytes + 16384;
#pragma unroll
            for (int k = 0; k < kPieces; ++k) {
                const int c = lane + 32 * k;
                const int r = c >> 3, c16 = c & 7;
                cp_async_16(dst + r * 128 + ((c16 ^ (r & 7)) << 4), src + (size_t)r * (a.d_e / 8) + c16);
            }
            cp_async_mbar_arrive(&sh.full_h[st]);
        }
        cp_async_wait_all();   // no copy into this block's shared memory outlives it
    } else {
        // --------------------------------------------------------- epilogue --
        const int qd = warp & 3;
        const int row = qd * 32 + lane;              // TMEM lane = accumulator row
        const int et = threadIdx.x - 96;             // 0..127
        {
            // zero the other parity's counters for the next launch
            const int oth = par ^ 1;
            for (int k2 = cta * 128 + et; k2 < a.E; k2 += G * 128) a.readyA[(size_t)oth * a.E + k2] = 0u;
            for (int k2 = cta * 128 + et; k2 < a.RT; k2 += G * 128) a.cntB[(size_t)oth * a.RT + k2] = 0u;
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
            const bool mine = (row >> 6) == hk;             // rows [64*hk, 64*hk + 64) are reduced here
            for (int ua = 0; ua < nA && !failed; ++ua) {
                const int ab = ua & 1;
                const int v = pr + ua * NCL;
                const int s = v / MT, mt = v % MT;
                const int e = sh.s_pair_e[s];
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
                // this block's partial h^T tile: float4 of tokens 4k..4k+3 of a row at k*128 + row
                {
                    float4* p4 = reinterpret_cast<float4*>(part) + row;
#pragma unroll
                    for (int k4 = 0; k4 < N / 4; ++k4)
                        p4[k4 * 128] = make_float4(__uint_as_float(r[4 * k4]), __uint_as_float(r[4 * k4 + 1]),
                                                   __uint_as_float(r[4 * k4 + 2]), __uint_as_float(r[4 * k4 + 3]));
                }
                // the gates of expert e for this chunk (independent of the peer)
                const uint32_t bits = sh.s_tmask[e];
                float gv[N];
#pragma unroll
                for (int t = 0; t < N; ++t) gv[t] = __ldg(a.gates + (size_t)min(t, nt - 1) * a.E + e);
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
                float z[N];
                if (mine) {
                    // h = (k-half 0) + (k-half 1); two terms, so the order is fixed
                    float4 pv[N / 4];
#pragma unroll
                    for (int k4 = 0; k4 < N / 4; ++k4)
                        pv[k4] = ld_shared_cluster_f4(peer_part + (uint32_t)((k4 * 128 + row) * 16));
#pragma unroll
                    for (int k4 = 0; k4 < N / 4; ++k4) {
                        z[4 * k4] = __uint_as_float(r[4 * k4]) + pv[k4].x;
                        z[4 * k4 + 1] = __uint_as_float(r[4 * k4 + 1]) + pv[k4].y;
                        z[4 * k4 + 2] = __uint_as_float(r[4 * k4 + 2]) + pv[k4].z;
                        z[4 * k4 + 3] = __uint_as_float(r[4 * k4 + 3]) + pv[k4].w;
                    }
                }
                named_bar_sync(1, 128);
                if (et == 0) {
                    RS_TRACE_ONCE(kRtARead);
                    mbar_arrive_cluster(peer_free);   // done with the peer's partial
                }
                if (mine) {
                    __nv_bfloat16* hrow = a.hbuf + (size_t)s * N * a.d_e + mt * 128 + row;
#pragma unroll
                    for (int t = 0; t < N; ++t) {
                        const float hv = ((bits >> t) & 1u) ? gv[t] * rs_swish(z[t]) : 0.f;
                        hrow[(size_t)t * a.d_e] = __float2bfloat16_rn(hv);
                    }
                }
                __threadfence();
                named_bar_sync(1, 128);
                if (et == 0) RS_TRACE_ONCE(kRtAWritten);
                if (et == 0 && (v * 2 + hk) != a.skip_unit) atomicAdd(&readyA[s], 1u);
            }
            if (et == 0) RS_TRACE(kRtADone);
        }
        // ---- expert-out row tiles: contributors publish partials, then each sums a slice
        const float* partB = a.partB;
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
                const int myslot = bLo >= first ? 0 : 1;
                float4* dst = reinterpret_cast<float4*>(a.partB + (size_t)(cta * 2 + myslot) * (N * 128)) + row;
#pragma unroll
                for (int kq = 0; kq < N / 4; ++kq)
                    dst[kq * 128] = make_float4(__uint_as_float(r[4 * kq]), __uint_as_float(r[4 * kq + 1]),
                                                __uint_as_float(r[4 * kq + 2]), __uint_as_float(r[4 * kq + 3]));
                __threadfence();
                named_bar_sync(1, 128);
                if (et == 0) {
                    RS_TRACE_ONCE(kRtBPartial);
                    atomicAdd(&cntB[rt], 1u);
                    RS_TRACE_ONCE(kRtBArrive);
                }
                if (npend < 2) {
                    pend_first[npend] = first;
                    pend_last[npend] = last;
                    pend_rt[npend] = rt;
                    ++npend;
                }
            }
            j = shi;
        }
        // second pass: wait for each split row tile's contributors, sum my slice
        for (int pi = 0; pi < npend && !failed; ++pi) {
            int q0, q1, nc, rank;
            contributors(pend_first[pi], pend_last[pi], q0, q1, nc, rank);
            const int rt = pend_rt[pi];
            if (et == 0) {
                sh.ep_ok = wait_count(&cntB[rt], (uint32_t)nc, limit_peer, &sh.abort, a.ctl, kWaitPeers) ? 1 : 0;
                int k2 = 0;
                for (int qq = q0; qq <= q1 && k2 < kRsMaxG; ++qq)
                    if (sh.s_blo[qq + 1] > sh.s_blo[qq])
                        sh.s_contrib[k2++] = qq * 2 + (sh.s_blo[qq] >= pend_first[pi] ? 0 : 1);
            }
            named_bar_sync(1, 128);
            if (!sh.ep_ok) { failed = true; break; }
            const int r0 = rank * 128 / nc, r1 = (rank + 1) * 128 / nc, nrows = r1 - r0;
            const float4* pbase = reinterpret_cast<const float4*>(partB);
            const int nitems = nrows * (N / 4);
            for (int base = 0; base < nitems; base += 256) {
                int rr[2], kq[2];
                bool on2[2];
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    const int itx = base + m * 128 + et;
                    on2[m] = itx < nitems;
                    const int ic = on2[m] ? itx : 0;
                    rr[m] = r0 + ic % nrows;
                    kq[m] = ic / nrows;
                }
                float4 acc[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
                for (int c0 = 0; c0 < nc; c0 += 8) {
                    float4 t4[2][8];
#pragma unroll
                    for (int m = 0; m < 2; ++m)
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            t4[m][u] = __ldcg(pbase + (size_t)sh.s_contrib[min(c0 + u, nc - 1)] * (N * 32) +
                                              kq[m] * 128 + rr[m]);
#pragma unroll
                    for (int m = 0; m < 2; ++m)
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            if (c0 + u < nc) {
                                acc[m].x += t4[m][u].x;
                                acc[m].y += t4[m][u].y;
                                acc[m].z += t4[m][u].z;
                                acc[m].w += t4[m][u].w;
                            }
                }
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    if (!on2[m]) continue;
                    const float z[4] = {acc[m].x, acc[m].y, acc[m].z, acc[m].w};
                    __nv_bfloat16* ycol = a.y + rt * 128 + rr[m];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int t = 4 * kq[m] + u;
                        if (t < nt) ycol[(size_t)t * a.d_h] = __float2bfloat16_rn(z[u]);
                    }
                }
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
    return 1024 + (size_t)kRsStages * kRsStageBytes + kRsPartBytes + sizeof(RsShared);
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
    return cudaLaunchKernelEx(&cfg, union_expert_decode<N>, maps[0], maps[1], maps[2], a);
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
