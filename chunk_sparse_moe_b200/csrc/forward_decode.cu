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
// from the gates itself.  Blocks run in thread-block clusters of 4: ranks 0-1
// and 2-3 are two k-half pairs.
//
// Expert-in (A).  A unit is one union expert e and one 128-row tile of W_in_e
// (d_e = 128: the whole expert).  The pair at position p of the A order takes
// units p, p + #pairs, ...; its block of rank r in the pair multiplies the
// k-half r of W_in_e (tcgen05; weights as the M = 128 operand, the chunk's N
// tokens as N) into a TMEM accumulator, two 64-wide k-blocks per pipeline stage.  The two blocks split the tokens: each
// sends the peer its partial for the peer's half with st.async straight into
// the peer's shared memory (the bytes are counted on the peer's mbarrier), adds
// the peer's partial for its own half, applies the post-hoc mask, the gate and
// Swish, writes its half of h' (bf16) to global memory and counts it in for the
// expert.  The A order lists first the pairs whose cluster has no expert-out
// row tile, so that those clusters start expert-out work with free hands.
//
// Expert-out (B).  y^T = sum_e W_out_e h'_e^T with W_out_e's 128-row tiles as the
// M operand and the tokens as N.  Cluster c owns the row tiles c, c + #clusters,
// ...; each of its 4 blocks takes a quarter of a row tile's (expert, pair of
// 64-wide k-blocks) tiles.  A tile waits (bounded) until its expert's h' is counted
// in, then its h' slice arrives by TMA.  The 4 partial tiles are summed inside
// the cluster: warp q of every block st.async's its 32 accumulator rows to the
// block of rank q, which adds the 4 contributions in rank order (a fixed order)
// and writes those 32 rows of y.
//
// Optional expert biases (the experts' nn.Linear layers, Router Architecture
// Setup).  The fc1 bias of an accumulator row is added before Swish.  The summing
// warp of a row slice starts from the gated fc2 biases of its rows, sum over the
// union, ascending, of bit_t ? g[t,e] b_out[e,i] : 0 (formed while the
// expert-out MMAs run), and adds the four partials to it.  (The layer's closing
// LayerNorm runs as a kernel of its own after this one: done here, its
// statistics would need every cluster's rows before any row could be stored,
// and that chain measured slower than the separate launch.)
//
// Roles (224 threads): warp 0 TMA producer (one lane), warp 1 MMA issuer (the
// whole warp runs its loops and waits, one elected lane issues), warp 2 TMEM
// owner and activation loader (x; the even expert-out stages' h'), warps 3-6
// epilogue (one lane of warp 6, or 5, also issues the odd expert-out stages' h'
// copies of the first two row tiles).  Every wait is bounded; a timeout
// records BLOCKFFN_ERR_TIMEOUT and the block winds down without leaving copies
// in flight.
//
// Launch.  A programmatic dependent of the previous kernel on the stream: a
// block initialises its barriers, allocates TMEM and prefetches its tensor maps,
// then waits for that kernel (griddepcontrol.wait) before it reads any input or
// the workspace.  The cluster barrier after set-up is split: every thread
// arrives, but only the epilogue warps, the one role that writes into a peer's
// shared memory, wait before their first remote access; the other roles wait
// at teardown.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace bffn {

constexpr int kRsThreads = 224;
constexpr int kRsCluster = 4;
constexpr int kRsStages = 5;
// a stage: weight tile [128 rows x 128] + activation tile [<=32 rows x 128], each
// as two 64-wide k-blocks of 128-byte-swizzled rows, each fetched by one 3-D TMA
// operation (a TMA operation costs about the same below ~32 KB, so fewer and
// larger ones move more bytes per SM)
constexpr int kRsWBytes = 32768;
constexpr int kRsStageBytes = kRsWBytes + 8192;
constexpr int kRsTmemCols = 128;             // 2 expert-in + 2 expert-out accumulators of <=32 columns
constexpr int kRsMaxE = 256;
constexpr int kRsMaxG = 160;
// receive area: two expert-in partials for this block's half of the tokens
// ([<=16 tokens][128 rows] fp32 each); later the expert-out quadrant partials
// from the other 3 ranks ([4 slots][<=32 tokens][32 rows] fp32) reuse it
constexpr int kRsRecvBytes = 2 * 16 * 128 * 4;
constexpr int kRsHStageBytes = 16 * 128 * 2;  // this block's half of h' [<=16 tokens][128 rows] bf16
static_assert(4 * 32 * 32 * 4 <= kRsRecvBytes, "expert-out quadrants fit the receive area");

struct RsShared {
    uint64_t full_w[kRsStages];   // TMA bytes landed
    uint64_t full_h[kRsStages];   // h' slice landed (B, TMA bytes) / nothing to copy (A, one arrival)
    uint64_t empty[kRsStages];    // MMAs reading the stage are done
    uint64_t accA_full[2];
    uint64_t accA_empty[2];
    uint64_t accB_full[2];
    uint64_t accB_empty[2];
    uint64_t recvA[2];            // the peer's expert-in partial landed here (st.async bytes)
    uint64_t freeA[2];            // 1 arrival: the peer has read what this block sent it
    uint64_t recvB;               // the other ranks' expert-out quadrant partials landed
    uint64_t freeB;               // 3 arrivals: the other ranks have summed the last quadrants sent them
    uint64_t mma_done;
    uint64_t a_pub;               // 1 arrival: this block's expert-in results are published
    uint32_t tmem_base;
    volatile int abort;
    int abort0;                   // abort as thread 0 set it before the first block barrier
    int tab_bad;                  // the caller's union tables disagree with their token masks
    int ep_okA[2];                // epilogue: the two waits of an expert-in unit
    int ep_okB[2];                // epilogue: the two waits of an expert-out row tile
    int b_go, b_fail;             // epilogue: expert-out work may start / a summing warp gave up
    uint32_t epoch;
    int P;
    uint32_t trace_once;          // trace slots already stamped (first occurrence only)
    int pendA[2], pendB;          // parity of a receive phase armed but not seen complete, or -1
    long long h_last;             // ring index of the last h' copy the epilogue lane issued, or -1
    int mma_all;                  // the MMAs read every stage of the launch (so every copy landed)
    float s_gate[2][32];          // gates of the current expert-in unit's expert, per token
    int32_t s_pair_e[kRsMaxE];    // the union, ascending
    uint32_t s_tmask[kRsMaxE];    // per expert: bit t = token t's gate is nonzero
    uint32_t s_bal[kRsMaxE / 32];
};

enum : int {
    kRtStart = 0, kRtPrologue = 1, kRtFirstLoad = 2, kRtLastLoad = 3, kRtFirstFull = 4,
    kRtLastACommit = 5, kRtADone = 7, kRtFirstFlag = 8, kRtLastFlag = 9, kRtLastCommit = 10,
    kRtLastEpi = 11, kRtEnd = 13, kRtATmem = 14, kRtASent = 15, kRtAReady = 16, kRtARead = 17,
    kRtAWritten = 18, kRtBSent = 21, kRtBReduced = 23, kRtFirstBMma = 24, kRtBRecv = 30, kRtSlots = 64
};
#define RS_TRACE(slot) \
    do { if (a.trace) a.trace[(size_t)blockIdx.x * kRtSlots + (slot)] = globaltimer_ns(); } while (0)
#define RS_TRACE_ONCE(slot)                                                            \
    do {                                                                               \
        if (a.trace && !(atomicOr(&sh.trace_once, 1u << (slot)) & (1u << (slot))))     \
            a.trace[(size_t)blockIdx.x * kRtSlots + (slot)] = globaltimer_ns();        \
    } while (0)

__device__ __forceinline__ float rs_swish(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

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

// The 8 MMAs of one pipeline stage: D (+)= W[128 x 128] * act[N x 128]^T, the
// weight tile at the stage's start and the activation tile after it, each as two
// 64-wide k-blocks in the 128-byte-swizzled K-major layout TMA writes.  ds is the
// descriptor of the stage's first byte; every operand's descriptor is ds plus a
// compile-time offset (computing each one from a run-time address made the
// issuing thread markedly slower per stage than the tensor core).
template <int N>
__device__ __forceinline__ void rs_stage_mma(uint32_t d, uint64_t ds, uint32_t idesc, bool acc) {
#pragma unroll
    for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_bf16(d, ds + (uint64_t)((kb * 16384 + kk * 32) >> 4),
                      ds + (uint64_t)((kRsWBytes + kb * N * 128 + kk * 32) >> 4), idesc,
                      (acc || kb > 0 || kk > 0) ? 1u : 0u);
}

// This block's expert-out tiles, in order: for each row tile rt = rt0, rt0 +
// step, ... of its cluster, the tiles j in [lo, hi) of that row tile, tile j
// being expert slot j / KPe and pair of 64-wide k-blocks kb = j % KPe (k-blocks
// 2kb and 2kb+1).  Stepped without divisions.
struct BCursor {
    int rt, j, s, kb;
    int lo, hi, s0, kb0, step, KPe;
    __device__ __forceinline__ void init(int rt0, int rtstep, int lo_, int hi_, int KPe_) {
        rt = rt0;
        step = rtstep;
        lo = lo_;
        hi = hi_;
        KPe = KPe_;
        s0 = lo / KPe;
        kb0 = lo - s0 * KPe;
        j = lo;
        s = s0;
        kb = kb0;
    }
    __device__ __forceinline__ void advance() {
        if (++j == hi) {
            j = lo;
            s = s0;
            kb = kb0;
            rt += step;
        } else if (++kb == KPe) {
            kb = 0;
            ++s;
        }
    }
};

// Where this block stands in the grid and what it computes.
struct RsWork {
    int cr, cid, ncl, pr, hk;   // cluster rank, cluster, #clusters, pair, k-half
    int nA, apos, npairs;       // expert-in units of the pair: v = apos + u * npairs, u < nA
    int nRT, rt0, rtstep;       // expert-out row tiles of the cluster: rt0, rt0 + rtstep, ...
    int bLo, bHi;               // this block's tiles of each of them
};

__device__ __forceinline__ RsWork rs_work(int G, int P, int MT, int KPe, int RT) {
    RsWork w;
    w.cr = (int)cluster_ctarank();
    w.cid = (int)blockIdx.x / kRsCluster;
    w.ncl = G / kRsCluster;
    w.pr = w.cid * 2 + (w.cr >> 1);
    w.hk = w.cr & 1;
    w.npairs = 2 * w.ncl;
    const int per_rt = P * KPe;
    w.nRT = w.cid < RT ? (RT - w.cid + w.ncl - 1) / w.ncl : 0;
    w.rt0 = w.cid;
    w.rtstep = w.ncl;
    w.bLo = per_rt * w.cr / kRsCluster;
    w.bHi = per_rt * (w.cr + 1) / kRsCluster;
    // the A order: pairs of clusters without a row tile first
    const int nBc = min(RT, w.ncl);
    w.apos = w.pr >= 2 * nBc ? w.pr - 2 * nBc : w.pr + 2 * (w.ncl - nBc);
    const int VA = P * MT;
    w.nA = w.apos < VA ? (VA - w.apos + w.npairs - 1) / w.npairs : 0;
    return w;
}

template <int N>
__global__ void __launch_bounds__(kRsThreads, 1)
union_expert_decode(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_win,
                    const __grid_constant__ CUtensorMap tm_wout, const __grid_constant__ CUtensorMap tm_h,
                    const __grid_constant__ CUtensorMap tm_y, const DcArgs a) {
    constexpr int NH = N / 2;   // tokens per k-half block in the expert-in epilogue
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned by pointer arithmetic on the shared array itself (an
    // integer round trip would make every access through it a generic one)
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float* recv = reinterpret_cast<float*>(smem + kRsStages * kRsStageBytes);
    __nv_bfloat16* hstage = reinterpret_cast<__nv_bfloat16*>(smem + kRsStages * kRsStageBytes + kRsRecvBytes);
    RsShared& sh = *reinterpret_cast<RsShared*>(smem + kRsStages * kRsStageBytes + kRsRecvBytes + kRsHStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x;
    const int KPe = a.d_e / 128;    // k-block pairs of one expert in the expert-out GEMM
    const int MT = a.d_e / 128;     // 128-row tiles of W_in_e
    const int KP = a.KB / 4;        // k-block pairs of one k-half in the expert-in GEMM
    const int nt = min(a.n, a.T);

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
            mbar_init(&sh.accB_full[s], 1);
            mbar_init(&sh.accB_empty[s], 4);
            mbar_init(&sh.recvA[s], 1);
            mbar_init(&sh.freeA[s], 1);
        }
        mbar_init(&sh.recvB, 1);
        mbar_init(&sh.freeB, 3);
        mbar_init(&sh.mma_done, 1);
        mbar_init(&sh.a_pub, 1);
        sh.trace_once = 0u;
        sh.pendA[0] = sh.pendA[1] = sh.pendB = -1;
        sh.h_last = -1;
        sh.mma_all = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_win);
        prefetch_tmap(&tm_wout);
        prefetch_tmap(&tm_h);
        prefetch_tmap(&tm_y);
    }
    if (warp == 2) {
        tmem_alloc(&sh.tmem_base, kRsTmemCols);
        tmem_relinquish();
    }
    // Launched as a programmatic dependent of the previous kernel in the stream,
    // this block may start before that kernel has finished.  The setup above
    // touches only this block's shared memory, TMEM and the kernel's own tensor
    // maps; everything below reads the inputs or the workspace, which that
    // kernel may still be writing (or, for the workspace, reading).
    griddep_wait();
    if (threadIdx.x == 0) {
        griddep_launch_dependents();
        // Three independent control-block accesses, issued back to back so their
        // round trips overlap: the sticky status, this block's launch ticket (the
        // launch index is ticket / grid) and the workspace's shape key.
        const int32_t st0 = __ldcg(&a.ctl->status);
        const unsigned long long tk = atomicAdd(&a.ctl->ticket, 1ull);
        const unsigned long long key0 = claim_shape_key(a.ctl, a.shape_key);
        const uint32_t ep0 = (uint32_t)(tk / gridDim.x);
        if (blockIdx.x == 0) a.ctl->issued[(ep0 & 1u) ^ 1u] = 0u;   // the next launch's counter
        sh.epoch = ep0;
        const bool key_ok = key0 == 0ull || key0 == a.shape_key;
        if (!key_ok) record_error(a.ctl, kErrWorkspace, kShapeKey);
        sh.abort = st0 != 0 || !key_ok;
        sh.abort0 = st0 != 0 || !key_ok;
    }
    if (warp >= 3) {
        // the chunk's union, ascending (warps 3-6 take 32-expert groups): from the
        // gates (all of a lane's gate loads are issued before their first use), or
        // from the caller's token masks
        const int ngroups = (a.E + 31) / 32;
        const uint32_t live = nt >= 32 ? 0xffffffffu : ((1u << nt) - 1u);
        for (int g = warp - 3; g < ngroups; g += 4) {
            const int e = g * 32 + lane;
            const int ec = min(e, a.E - 1);
            uint32_t bits = 0u;
            if (a.tmask_in != nullptr) {
                bits = e < a.E ? (__ldg(a.tmask_in + e) & live) : 0u;
            } else {
                float v[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = __ldg(a.gates + (size_t)min(j, nt - 1) * a.E + ec);
#pragma unroll
                for (int j = 0; j < 32; ++j) bits |= ((e < a.E && j < nt && v[j] != 0.f) ? 1u : 0u) << j;
            }
            if (e < a.E) sh.s_tmask[e] = bits;
            const uint32_t bal = __ballot_sync(0xffffffffu, bits != 0u);
            if (lane == 0) sh.s_bal[g] = bal;
        }
        named_bar_sync(1, 128);
        if (warp == 3) {
            int base = 0;
            bool bad = false;
            for (int g = 0; g < ngroups; ++g) {
                const uint32_t bal = sh.s_bal[g];
                const int slot = base + __popc(bal & ((1u << lane) - 1u));
                if ((bal >> lane) & 1u) {
                    sh.s_pair_e[slot] = g * 32 + lane;
                    // the caller's index list must name the same experts in the same order
                    if (a.idx_in != nullptr && __ldg(a.idx_in + slot) != g * 32 + lane) bad = true;
                }
                base += __popc(bal);
            }
            if (a.idx_in != nullptr) {
                for (int s2 = base + lane; s2 < a.E; s2 += 32)
                    if (__ldg(a.idx_in + s2) != -1) bad = true;
                if (lane == 0 && __ldg(a.counts_in) != base) bad = true;
            }
            bad = __any_sync(0xffffffffu, bad);
            if (lane == 0) {
                sh.P = base;
                sh.tab_bad = bad ? 1 : 0;
                if (bad) record_error(a.ctl, kErrInvalidArg, kUnionTables);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (sh.tab_bad) {
        // refused tables: nothing is computed (a uniform branch, so every thread
        // takes the second barrier)
        if (threadIdx.x == 0) sh.abort = 1;
        __syncthreads();
    }
    // Whether this launch computes at all, the same in every thread: both words
    // were written before the barrier above and are not written again.  (The
    // volatile abort flag itself may be raised by any role at any time.)
    const bool abort_at_start = sh.abort0 != 0 || sh.tab_bad != 0;
    const int P = sh.P;
    const RsWork wk = rs_work(G, P, MT, KPe, a.RT);
    const int nBt = wk.bHi - wk.bLo;                 // expert-out tiles per owned row tile
    const int totB = P > 0 ? wk.nRT * nBt : 0;        // this block's expert-out tiles
    const bool doB = P > 0 && wk.nRT > 0;             // this cluster sums expert-out row tiles
    // The expert-out stages' h' copies of the first two row tiles alternate
    // between the loader (even) and one epilogue lane (odd); later row tiles are
    // the loader's alone (their MMAs wait for an accumulator the epilogue frees,
    // which that lane, held at the epilogue's barrier, could not wait for).
    const int qsplit = min(totB, 2 * nBt);
    const long long iB0 = (long long)wk.nA * (a.KB / 4);   // ring index of the first expert-out stage
    long long ld_last = -1;                           // the loader's last issued ring index
    if (threadIdx.x == 0 && doB && !sh.abort) {
        // the first expert-out reduction: 3 quadrant partials of 32 rows x N tokens
        // (not armed by a launch that computes nothing, whose teardown would
        // otherwise wait for bytes nobody sends)
        mbar_arrive_expect_tx(&sh.recvB, 3u * 32u * N * 4u);
        sh.pendB = 0;
    }
    // Every block's barriers are initialised before any remote arrival: all
    // threads arrive here; only the epilogue warps, the one role that touches
    // a peer's shared memory, wait before their first remote access (the
    // other roles wait at teardown), so the loads start without the cluster's
    // slowest prologue.
    cluster_arrive_release();
    if (threadIdx.x == 0) RS_TRACE(kRtPrologue);

    const uint32_t tmem = sh.tmem_base;
    const int par = (int)(sh.epoch & 1u);
    uint32_t* const readyA = a.readyA + (size_t)par * a.E;
    const uint64_t limit_peer = a.wait_ns;
    const uint64_t limit = 2 * a.wait_ns;
    const uint32_t accA_col = 0, accB_col = 2 * N;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer --
        if (lane == 0 && !sh.abort) {
            const uint64_t pol_stream = policy_evict_first();
            long long i = 0;
            RingPos rp;
            bool stop = false;
            for (int ua = 0; ua < wk.nA && !stop; ++ua) {
                const int v = wk.apos + ua * wk.npairs;
                const int e = sh.s_pair_e[v / MT], mt = v % MT;
                for (int t = 0; t < KP; ++t, ++i, rp.advance()) {
                    const int kb = 2 * (wk.hk * KP + t);   // first of the stage's two k-blocks
                    if (!wait_bar(&sh.empty[rp.st], rp.ph ^ 1u, limit, &sh.abort, a.ctl, kWaitEmpty)) {
                        stop = true;
                        break;
                    }
                    uint8_t* w = smem + rp.st * kRsStageBytes;
                    mbar_arrive_expect_tx(&sh.full_w[rp.st], kRsWBytes);
                    tma_load_3d(w, &tm_win, &sh.full_w[rp.st], 0, e * a.d_e + mt * 128, kb, pol_stream);
                    if (i == 0) RS_TRACE(kRtFirstLoad);
                }
            }
            if (wk.nA > 0) red_relaxed_add_gpu(&a.ctl->issued[par], 1u);
            // Expert-out weights.  A block with expert-in units sends all of its
            // tiles towards L2 now and loads them into the ring only after its h'
            // is published: a release waits for the block's bulk loads in flight,
            // and no expert-out MMA can start before every h' is out anyway.
            // Other blocks first let every expert-in block issue its last load (a
            // scheduling hint, bounded and never an error: their requests then
            // queue behind the expert-in weights, which are on the critical path),
            // then load and prefetch what the ring cannot hold yet.
            if (totB > 0 && wk.nA == 0 && !stop) {
                const uint32_t nAblocks = 2u * (uint32_t)min(P * MT, wk.npairs);
                const uint64_t t0 = globaltimer_ns();
                while (ld_relaxed_gpu(&a.ctl->issued[par]) < nAblocks && globaltimer_ns() - t0 < 20000ull &&
                       !sh.abort)
                    __nanosleep(64);
            }
            if (totB > 0) {
                BCursor bc;
                bc.init(wk.rt0, wk.rtstep, wk.bLo, wk.bHi, KPe);
                for (int q = 0; q < totB; ++q, bc.advance())
                    if (wk.nA > 0 || q >= kRsStages)
                        tma_prefetch_l2_3d(&tm_wout, 0, sh.s_pair_e[bc.s] * a.d_h + bc.rt * 128, 2 * bc.kb);
                if (wk.nA > 0 && !stop && !wait_bar(&sh.a_pub, 0u, limit, &sh.abort, a.ctl, kWaitEmpty))
                    stop = true;
                bc.init(wk.rt0, wk.rtstep, wk.bLo, wk.bHi, KPe);
                for (int q = 0; q < totB && !stop; ++q, ++i, rp.advance(), bc.advance()) {
                    if (!wait_bar(&sh.empty[rp.st], rp.ph ^ 1u, limit, &sh.abort, a.ctl, kWaitEmpty)) {
                        stop = true;
                        break;
                    }
                    mbar_arrive_expect_tx(&sh.full_w[rp.st], kRsWBytes);
                    tma_load_3d(smem + rp.st * kRsStageBytes, &tm_wout, &sh.full_w[rp.st], 0,
                                sh.s_pair_e[bc.s] * a.d_h + bc.rt * 128, 2 * bc.kb, pol_stream);
                    if (i == 0) RS_TRACE(kRtFirstLoad);
                }
            }
            RS_TRACE(kRtLastLoad);
            for (long long q = i - kRsStages < 0 ? 0 : i - kRsStages; q < i; ++q)
                wait_bar_drain(&sh.full_w[q % kRsStages], (uint32_t)((q / kRsStages) & 1), limit, a.ctl);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer --
        // The whole warp runs the loops with warp-wide waits; one elected lane
        // issues the MMAs and commits.
        const bool leader = elect_one();
        const uint32_t idesc = idesc_bf16_f32(128, N);     // 128 weight rows x tokens
        // shared addresses are below 2^18, so stage offsets added to the
        // descriptor's start-address field never carry out of it
        const uint64_t desc0 = sw128_kmajor_desc(smem_u32(smem));
        long long i = 0;
        RingPos rp;
        bool stop = __shfl_sync(0xffffffffu, sh.abort, 0) != 0;
        // the current ring position's barriers as last tested (a stale "not yet"
        // only costs a blocking wait)
        uint32_t rw = 0u, rh = 0u;
        for (int ua = 0; ua < wk.nA && !stop; ++ua) {
            const int ab = ua & 1;
            if (!wait_bar_warp(&sh.accA_empty[ab], (uint32_t)(((ua >> 1) & 1) ^ 1), limit, &sh.abort, a.ctl,
                               kWaitAccEmpty))
                break;
            tc_fence_after();
            const uint32_t d = tmem + accA_col + (uint32_t)(ab * N);
            for (int t = 0; t < KP; ++t, ++i, rp.advance()) {
                const int st = rp.st;
                if (!__all_sync(0xffffffffu, rw & rh) &&
                    (!wait_bar_warp(&sh.full_w[st], rp.ph, limit, &sh.abort, a.ctl, kWaitFullW) ||
                     !wait_bar_warp(&sh.full_h[st], rp.ph, limit, &sh.abort, a.ctl, kWaitFullH))) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                {
                    // test the next ring position now: the two shared-memory round
                    // trips then overlap this stage's MMAs instead of preceding the next
                    RingPos nx = rp;
                    nx.advance();
                    rw = mbar_test_wait(&sh.full_w[nx.st], nx.ph);
                    rh = mbar_test_wait(&sh.full_h[nx.st], nx.ph);
                }
                if (leader) {
                    if (i == 0) RS_TRACE(kRtFirstFull);
                    rs_stage_mma<N>(d, desc0 + (uint64_t)(st * (kRsStageBytes >> 4)), idesc, t > 0);
                    umma_commit(&sh.empty[st]);
                }
                __syncwarp();
            }
            if (stop) break;
            if (leader) {
                umma_commit(&sh.accA_full[ab]);
                RS_TRACE(kRtLastACommit);
            }
            __syncwarp();
        }
        // one accumulator per owned row tile, alternating between two
        for (int k = 0; k < (totB > 0 ? wk.nRT : 0) && !stop; ++k) {
            const int ab = k & 1;
            if (!wait_bar_warp(&sh.accB_empty[ab], (uint32_t)(((k >> 1) & 1) ^ 1), limit, &sh.abort, a.ctl,
                               kWaitAccEmpty))
                break;
            tc_fence_after();
            const uint32_t d = tmem + accB_col + (uint32_t)(ab * N);
            for (int q = 0; q < nBt; ++q, ++i, rp.advance()) {
                const int st = rp.st;
                if (!__all_sync(0xffffffffu, rw & rh) &&
                    (!wait_bar_warp(&sh.full_w[st], rp.ph, limit, &sh.abort, a.ctl, kWaitFullW) ||
                     !wait_bar_warp(&sh.full_h[st], rp.ph, limit, &sh.abort, a.ctl, kWaitFullH))) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                {
                    RingPos nx = rp;
                    nx.advance();
                    rw = mbar_test_wait(&sh.full_w[nx.st], nx.ph);
                    rh = mbar_test_wait(&sh.full_h[nx.st], nx.ph);
                }
                if (leader) {
                    if (k == 0 && q == 0) RS_TRACE(kRtFirstBMma);
                    rs_stage_mma<N>(d, desc0 + (uint64_t)(st * (kRsStageBytes >> 4)), idesc, q > 0);
                    umma_commit(&sh.empty[st]);
                }
                __syncwarp();
            }
            if (stop) break;
            if (leader) {
                umma_commit(&sh.accB_full[ab]);
                RS_TRACE(kRtLastCommit);
            }
            __syncwarp();
        }
        if (leader) {
            // every stage read: each copy issued into the ring has landed
            if (i == (long long)wk.nA * KP + totB) sh.mma_all = 1;
            umma_commit(&sh.mma_done);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ------------------------------------------------- activation loader --
        // An expert-in stage's activations are the chunk's two x k-blocks of the
        // stage (lane 0 issues them, so the weight tiles and the activation tiles
        // come from two issuing threads: one thread issues bulk copies at a bounded
        // rate).  For an expert-out tile lane 0 waits (bounded) until the tile's
        // expert slot's h' is counted in, then moves the [N x 64] h' slice with
        // one TMA load, which lands in the same 128-byte-swizzled layout as the
        // weight tile's operand.
        long long i = 0;
        RingPos rp;
        int stop = sh.abort != 0;
        if (lane == 0) {
            const uint64_t pol_keep = policy_evict_last();
            for (int ua = 0; ua < wk.nA && !stop; ++ua) {
                for (int t = 0; t < KP; ++t, ++i, rp.advance()) {
                    if (!wait_bar(&sh.empty[rp.st], rp.ph ^ 1u, limit, &sh.abort, a.ctl, kWaitEmpty)) {
                        stop = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(&sh.full_h[rp.st], (uint32_t)(N * 256));
                    tma_load_3d(smem + rp.st * kRsStageBytes + kRsWBytes, &tm_x, &sh.full_h[rp.st], 0, 0,
                                2 * (wk.hk * KP + t), pol_keep);
                    ld_last = i;
                }
            }
        }
        stop = __shfl_sync(0xffffffffu, stop, 0);
        if (!stop && totB > 0 && lane == 0) {
            // Each expert-out tile waits (bounded) only for its own expert slot's h'
            // (both k-halves of every 128-row tile counted in), so tiles of experts
            // finished early start while later experts' expert-in units still run.
            // Of the first two row tiles this thread takes the even stages and an
            // epilogue lane (warp 6, or 5 in rank 2) the odd ones (one thread issues
            // bulk copies at a bounded rate, and the expert-out phase is one h'
            // copy per stage); later row tiles' stages are all this thread's.
            const uint64_t pol = policy_evict_first();
            BCursor bc;
            bc.init(wk.rt0, wk.rtstep, wk.bLo, wk.bHi, KPe);
            int ready_s = -1;
            for (int q = 0; q < totB; ++q, ++i, rp.advance(), bc.advance()) {
                if (q < qsplit && (q & 1)) continue;
                if (bc.s != ready_s) {
                    if (!wait_count(&readyA[bc.s], (uint32_t)(2 * MT), limit_peer, &sh.abort, a.ctl)) break;
                    // the h' stores were made visible to this thread by the acquire;
                    // the async proxy reads them next
                    fence_proxy_async_global();
                    if (ready_s < 0) RS_TRACE_ONCE(kRtFirstFlag);
                    RS_TRACE(kRtLastFlag);
                    ready_s = bc.s;
                }
                if (!wait_bar(&sh.empty[rp.st], rp.ph ^ 1u, limit, &sh.abort, a.ctl, kWaitEmpty)) break;
                mbar_arrive_expect_tx(&sh.full_h[rp.st], (uint32_t)(N * 256));
                tma_load_3d(smem + rp.st * kRsStageBytes + kRsWBytes, &tm_h, &sh.full_h[rp.st], 0, bc.s * N,
                            2 * bc.kb, pol);
                ld_last = i;
            }
        }
        __syncwarp();
        // (this warp's copies are drained at teardown, with the epilogue lane's)
    } else {
        // --------------------------------------------------------- epilogue --
        cluster_wait_acquire();
        const int qd = warp & 3;                     // TMEM lane quadrant of this warp
        const int row = qd * 32 + lane;              // TMEM lane = accumulator row
        const int et = threadIdx.x - 96;             // 0..127
        {
            // zero the other parity's counters for the next launch
            const int oth = par ^ 1;
            for (int k2 = (int)blockIdx.x * 128 + et; k2 < a.E; k2 += G * 128) a.readyA[(size_t)oth * a.E + k2] = 0u;
        }
        // Every decision below that ends a loop is taken from shared memory after a
        // named barrier (or, like this one, from values fixed before the block's
        // first barrier), so the four epilogue warps always take the same path and
        // meet the same named barriers.
        bool failed = abort_at_start;
        if (P == 0 && blockIdx.x == 0 && !failed) {
            // empty union: y is all zeros
            for (size_t k2 = et; k2 < (size_t)nt * a.d_h; k2 += 128) a.y[k2] = __float2bfloat16_rn(0.f);
        }
        // ---- A units: each block finishes its half of the tokens
        const uint32_t peer = (uint32_t)(wk.cr ^ 1);
        const uint32_t peer_recv = mapa_shared(smem_u32(recv), peer);
        const uint32_t peer_recvA = mapa_shared(smem_u32(&sh.recvA[0]), peer);
        const uint32_t peer_freeA = mapa_shared(smem_u32(&sh.freeA[0]), peer);
        const int tg = wk.hk * NH;                   // first token this block finishes
        for (int ua = 0; ua < wk.nA && !failed; ++ua) {
            const int b = ua & 1;
            const int v = wk.apos + ua * wk.npairs;
            const int s = v / MT, mt = v % MT;
            const int e = sh.s_pair_e[s];
            // stage the unit's gates now: the accumulator wait hides their latency,
            // and the activation loop below then reads shared memory only
            if (et < 32) sh.s_gate[b][et] = a.gates[(size_t)min(et, nt - 1) * a.E + e];
            // this accumulator row's fc1 bias (0 without biases)
            const float bin = a.b_in != nullptr ? __ldg(a.b_in + (size_t)e * a.d_e + mt * 128 + row) : 0.f;
            if (et == 0) {
                // the peer's partial for this block's half of unit ua lands in buffer b
                mbar_arrive_expect_tx(&sh.recvA[b], (uint32_t)(NH * 128 * 4));
                sh.pendA[b] = (ua >> 1) & 1;
                int ok = wait_bar(&sh.accA_full[b], (uint32_t)((ua >> 1) & 1), limit, &sh.abort, a.ctl,
                                  kWaitAccFull) ? 1 : 0;
                // before sending into the peer's buffer b again, the peer has read it
                if (ok && ua >= 2)
                    ok = wait_bar_cluster(&sh.freeA[b], (uint32_t)(((ua - 2) >> 1) & 1), limit_peer, &sh.abort,
                                          a.ctl, kWaitPeers) ? 1 : 0;
                sh.ep_okA[0] = ok;
            }
            named_bar_sync(1, 128);
            if (!sh.ep_okA[0]) { failed = true; break; }
            tc_fence_after();
            uint32_t r[32];
            const uint32_t taddr = tmem + ((uint32_t)(qd * 32) << 16) + accA_col + (uint32_t)(b * N);
            if constexpr (N == 32) tmem_ld_32x32b_x32(taddr, r);
            else tmem_ld_32x32b_x16(taddr, r);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.accA_empty[b]);
            if (et == 0) RS_TRACE_ONCE(kRtATmem);
            // the peer's half of the tokens goes to the peer: float4 of the half's
            // tokens 4k..4k+3 of a row at k*128 + row of its buffer b
            {
                const uint32_t dst = peer_recv + (uint32_t)(b * NH * 128 * 4 + row * 16);
                const uint32_t rbar = peer_recvA + (uint32_t)(b * 8);
#pragma unroll
                for (int k4 = 0; k4 < NH / 4; ++k4) {
                    float f[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        f[u] = __uint_as_float(wk.hk ? r[4 * k4 + u] : r[NH + 4 * k4 + u]);
                    st_async_v4(dst + (uint32_t)(k4 * 128 * 16), f[0], f[1], f[2], f[3], rbar);
                }
            }
            if (et == 0) RS_TRACE_ONCE(kRtASent);
            const uint32_t bits = sh.s_tmask[e] >> tg;   // this half's token bits
            if (et == 0) {
                sh.ep_okA[1] = wait_bar_cluster(&sh.recvA[b], (uint32_t)((ua >> 1) & 1), limit_peer, &sh.abort,
                                                a.ctl, kWaitPeers) ? 1 : 0;
                if (sh.ep_okA[1]) sh.pendA[b] = -1;
                RS_TRACE_ONCE(kRtAReady);
            }
            named_bar_sync(1, 128);
            if (!sh.ep_okA[1]) { failed = true; break; }
            // h = (k-half 0) + (k-half 1): two terms, and the sum does not depend on
            // which block of the pair forms it
            float z[NH];
            {
                const float4* rb = reinterpret_cast<const float4*>(recv + b * NH * 128) + row;
#pragma unroll
                for (int k4 = 0; k4 < NH / 4; ++k4) {
                    const float4 pv = rb[k4 * 128];
                    const float pw[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        z[4 * k4 + u] = __uint_as_float(wk.hk ? r[NH + 4 * k4 + u] : r[4 * k4 + u]) + pw[u];
                }
            }
            named_bar_sync(1, 128);
            if (et == 0) {
                RS_TRACE_ONCE(kRtARead);
                // the peer may send into buffer b again (its unit ua + 2)
                if (ua + 2 < wk.nA) mbar_arrive_relaxed_cluster(peer_freeA + (uint32_t)(b * 8));
            }
            // h' = bit ? g * Swish(h) : 0 (a select, so a masked token gives 0 even if
            // its h is not finite), staged token-major in shared memory, then written
            // with 16-byte stores: token t's 128 rows are 256 contiguous bytes
            {
                // gates into registers first (loads interleaved with the staging
                // stores would each wait for the store before them)
                float gv[NH];
#pragma unroll
                for (int tl = 0; tl < NH; ++tl) gv[tl] = sh.s_gate[b][tg + tl];
                __nv_bfloat16 hb[NH];
#pragma unroll
                for (int tl = 0; tl < NH; ++tl)
                    hb[tl] = __float2bfloat16_rn(((bits >> tl) & 1u) ? gv[tl] * rs_swish(z[tl] + bin) : 0.f);
                __nv_bfloat16* stg = hstage + row;
#pragma unroll
                for (int tl = 0; tl < NH; ++tl) stg[tl * 128] = hb[tl];
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
                if ((v * 2 + wk.hk) != a.skip_unit) red_release_add_gpu(&readyA[s], 1u);
                RS_TRACE_ONCE(kRtAWritten);
            }
        }
        if (et == 0) {
            RS_TRACE(kRtADone);
            if (wk.nA > 0) mbar_arrive(&sh.a_pub);   // the producer may load expert-out tiles now
        }
        // ---- expert-out row tiles: the cluster's 4 partials meet in shared memory
        // (failed is the same in the four warps here; the abort flag is read once,
        // by one thread, and shared)
        if (et == 0) {
            sh.b_go = (!failed && !sh.abort) ? 1 : 0;
            sh.b_fail = 0;
        }
        named_bar_sync(1, 128);
        failed = failed || !sh.b_go;
        // one lane of a warp that is neither the summing warp of this rank (whose
        // fc2 bias sums overlap the MMAs) nor warp 3 (whose lane 0 takes the
        // epilogue's waits)
        if (warp == (wk.cr == 2 ? 5 : 6) && lane == 0 && !failed && qsplit > 1) {
            // The odd expert-out stages' h' copies of the first two row tiles (the
            // loader issues the rest): the same per-expert readiness wait, then one
            // TMA copy into the stage; the last ring index issued goes to shared
            // memory for the teardown's drain.
            const uint64_t pol = policy_evict_first();
            long long ib = iB0;
            RingPos bp;
            bp.st = (int)(ib % kRsStages);
            bp.ph = (uint32_t)((ib / kRsStages) & 1);
            BCursor bc;
            bc.init(wk.rt0, wk.rtstep, wk.bLo, wk.bHi, KPe);
            int ready_s = -1;
            for (int q = 0; q < qsplit; ++q, ++ib, bp.advance(), bc.advance()) {
                if ((q & 1) == 0) continue;
                if (bc.s != ready_s) {
                    if (!wait_count(&readyA[bc.s], (uint32_t)(2 * MT), limit_peer, &sh.abort, a.ctl)) break;
                    fence_proxy_async_global();
                    ready_s = bc.s;
                }
                if (!wait_bar(&sh.empty[bp.st], bp.ph ^ 1u, limit, &sh.abort, a.ctl, kWaitEmpty)) break;
                mbar_arrive_expect_tx(&sh.full_h[bp.st], (uint32_t)(N * 256));
                tma_load_3d(smem + bp.st * kRsStageBytes + kRsWBytes, &tm_h, &sh.full_h[bp.st], 0, bc.s * N,
                            2 * bc.kb, pol);
                sh.h_last = ib;
            }
        }
        __syncwarp();
        if (doB) {
            const uint32_t recv_u32 = smem_u32(recv);
            for (int k = 0; k < wk.nRT && !failed; ++k) {
                const int rt = wk.rt0 + k * wk.rtstep;
                const int ab = k & 1;
                uint32_t r[32];
                // the summing warp's gated fc2 bias sums of its 32 rows, formed while
                // the expert-out MMAs run: lane = row, bacc[t] for token t
                float bacc[N];
#pragma unroll
                for (int t = 0; t < N; ++t) bacc[t] = 0.f;
                if (a.b_out != nullptr && qd == wk.cr) {
                    const float* bo = a.b_out + rt * 128 + wk.cr * 32 + lane;
                    // 8 union experts at a time: their loads are issued together
                    for (int s0 = 0; s0 < P; s0 += 8) {
                        float bv[8], gl[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            bv[u] = 0.f;
                            gl[u] = 0.f;
                            if (s0 + u < P) {
                                const int e = sh.s_pair_e[s0 + u];
                                bv[u] = __ldg(bo + (size_t)e * a.d_h);
                                if (lane < nt && ((sh.s_tmask[e] >> lane) & 1u))
                                    gl[u] = a.gates[(size_t)lane * a.E + e];
                            }
                        }
#pragma unroll
                        for (int u = 0; u < 8; ++u)
#pragma unroll
                            for (int t = 0; t < N; ++t)
                                bacc[t] = fmaf(__shfl_sync(0xffffffffu, gl[u], t), bv[u], bacc[t]);
                    }
                }
                if (nBt > 0) {
                    if (et == 0)
                        sh.ep_okB[0] = wait_bar(&sh.accB_full[ab], (uint32_t)((k >> 1) & 1), limit, &sh.abort, a.ctl,
                                            kWaitAccFull) ? 1 : 0;
                    named_bar_sync(1, 128);
                    if (!sh.ep_okB[0]) { failed = true; break; }
                    tc_fence_after();
                    const uint32_t taddr = tmem + ((uint32_t)(qd * 32) << 16) + accB_col + (uint32_t)(ab * N);
                    if constexpr (N == 32) tmem_ld_32x32b_x32(taddr, r);
                    else tmem_ld_32x32b_x16(taddr, r);
                    tmem_ld_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sh.accB_empty[ab]);
                } else {
#pragma unroll
                    for (int t = 0; t < 32; ++t) r[t] = 0u;   // no tiles here: a zero contribution
                }
                if (k > 0) {
                    // the receive area is reused: every other rank has summed the
                    // quadrants this block sent it for the previous row tile
                    if (et == 0)
                        sh.ep_okB[1] = wait_bar_cluster(&sh.freeB, (uint32_t)((k - 1) & 1), limit_peer, &sh.abort,
                                                    a.ctl, kWaitPeers) ? 1 : 0;
                    named_bar_sync(1, 128);
                    if (!sh.ep_okB[1]) { failed = true; break; }
                }
                if (qd != wk.cr) {
                    // rows of quadrant qd are summed by rank qd: slot cr of its receive
                    // area, float4 of tokens 4c..4c+3 of a row at [c][row] (consecutive
                    // lanes, consecutive 16 bytes: no bank conflicts on either side)
                    const uint32_t dst =
                        mapa_shared(recv_u32 + (uint32_t)((wk.cr * (N / 4) * 32 + lane) * 16), (uint32_t)qd);
                    const uint32_t rbar = mapa_shared(smem_u32(&sh.recvB), (uint32_t)qd);
#pragma unroll
                    for (int c4 = 0; c4 < N / 4; ++c4)
                        st_async_v4(dst + (uint32_t)(c4 * 32 * 16), __uint_as_float(r[4 * c4]),
                                    __uint_as_float(r[4 * c4 + 1]), __uint_as_float(r[4 * c4 + 2]),
                                    __uint_as_float(r[4 * c4 + 3]), rbar);
                    if (lane == 0) RS_TRACE_ONCE(kRtBSent);
                } else {
                    // this warp sums rows 32*cr .. 32*cr + 31 of the row tile over the 4
                    // ranks, in rank order
                    int ok = 1;
                    if (lane == 0) {
                        ok = wait_bar_cluster(&sh.recvB, (uint32_t)(k & 1), limit_peer, &sh.abort, a.ctl,
                                              kWaitPeers) ? 1 : 0;
                        if (ok) sh.pendB = -1;
                        RS_TRACE(kRtBRecv);
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    float acc[N];
                    if (ok) {
#pragma unroll
                        for (int t = 0; t < N; ++t) acc[t] = bacc[t];
#pragma unroll
                        for (int q = 0; q < kRsCluster; ++q) {
                            if (q == wk.cr) {
#pragma unroll
                                for (int t = 0; t < N; ++t) acc[t] += __uint_as_float(r[t]);
                            } else {
                                const float4* src = reinterpret_cast<const float4*>(recv) + q * (N / 4) * 32 + lane;
#pragma unroll
                                for (int c4 = 0; c4 < N / 4; ++c4) {
                                    const float4 pv = src[c4 * 32];
                                    acc[4 * c4] += pv.x;
                                    acc[4 * c4 + 1] += pv.y;
                                    acc[4 * c4 + 2] += pv.z;
                                    acc[4 * c4 + 3] += pv.w;
                                }
                            }
                        }
                    }
                    if (ok) {
                        // rows 32*cr.. of y for all tokens: staged [N tokens][32 rows]
                        // bf16, then one TMA store (rows past T are clipped)
                        if (k > 0 && lane == 0) bulk_wait_group_read0();   // staging free again
                        __syncwarp();
#pragma unroll
                        for (int t = 0; t < N; ++t) hstage[t * 32 + lane] = __float2bfloat16_rn(acc[t]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tm_y, hstage, rt * 128 + wk.cr * 32, 0);
                            bulk_commit_group();
                            RS_TRACE_ONCE(kRtBReduced);
                        }
                    } else if (lane == 0) {
                        sh.b_fail = 1;   // the other warps learn it after the barrier below
                    }
                }
                if (k + 1 < wk.nRT) {
                    // hand the receive area back: re-arm it for the next row tile and
                    // tell the other ranks this block has summed what they sent
                    named_bar_sync(1, 128);
                    failed = failed || sh.b_fail != 0;
                    if (et == 0 && !failed && !sh.abort) {
                        mbar_arrive_expect_tx(&sh.recvB, 3u * 32u * N * 4u);
                        sh.pendB = (k + 1) & 1;
                        for (int q = 1; q < kRsCluster; ++q)
                            mbar_arrive_relaxed_cluster(
                                mapa_shared(smem_u32(&sh.freeB), (uint32_t)((wk.cr + q) % kRsCluster)));
                    }
                }
            }
        }
        if (doB && qd == wk.cr && lane == 0) bulk_wait_group_read0();   // y's staging is read
        if (et == 0) RS_TRACE(kRtLastEpi);
    }

    // --------------------------------------------------------------- teardown --
    __syncwarp();
    __syncthreads();
    if (threadIdx.x == 0) {
        // a receive that was armed but never seen complete (a peer gave up or is
        // late): give its bytes a bounded chance to land before this block leaves
        for (int b = 0; b < 2; ++b)
            if (sh.pendA[b] >= 0) wait_bar_drain(&sh.recvA[b], (uint32_t)sh.pendA[b], limit, a.ctl);
        if (sh.pendB >= 0) wait_bar_drain(&sh.recvB, (uint32_t)sh.pendB, limit, a.ctl);
    }
    if (warp == 2) {
        if (lane == 0 && !sh.mma_all) {
            // No activation copy into this block's shared memory outlives it.  When
            // the MMAs read every stage, every copy landed; otherwise (a launch that
            // gave up), for every ring slot the last copy issued into it (by the
            // loader or the epilogue lane) is waited for: an earlier copy into a slot
            // was followed by a later one, issued only after the MMAs had read the
            // slot, so it had landed; and no copy followed the last one, so the
            // parity of its phase is not ambiguous.
            const long long h_last = sh.h_last;
            const long long last = ld_last > h_last ? ld_last : h_last;
            int found = 0;
            for (long long pos = last; pos >= 0 && found != (1 << kRsStages) - 1; --pos) {
                const int slot = (int)(pos % kRsStages);
                if (found & (1 << slot)) continue;
                const long long qb = pos - iB0;   // expert-out stage, or negative: expert-in
                const bool helper = qb >= 0 && qb < qsplit && (qb & 1);
                if (helper ? pos <= h_last : pos <= ld_last) {
                    found |= 1 << slot;
                    wait_bar_drain(&sh.full_h[slot], (uint32_t)((pos / kRsStages) & 1), limit, a.ctl);
                }
            }
        }
        if (lane == 0) wait_bar_drain(&sh.mma_done, 0, limit, a.ctl);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kRsTmemCols);
    }
    if (threadIdx.x == 0) RS_TRACE(kRtEnd);
    if (warp < 3) cluster_wait_acquire();   // the prologue's phase (the epilogue waited on it already)
    // no block leaves while a block of its cluster might still use its shared memory
    cluster_barrier_sync_relaxed();
}

size_t forward_decode_smem_bytes() {
    return 1024 + (size_t)kRsStages * kRsStageBytes + kRsRecvBytes + kRsHStageBytes + sizeof(RsShared);
}

template <int N>
static cudaError_t launch_decode_n(const DcArgs& a, const CUtensorMap* maps, int grid, cudaStream_t s) {
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
    attr[0].val.clusterDim.x = kRsCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // may start while the previous kernel in the stream finishes (the kernel
    // waits for it before touching any input or the workspace)
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, union_expert_decode<N>, maps[0], maps[1], maps[2], maps[3], maps[4], a);
}

cudaError_t launch_forward_decode(const DcArgs& a, const CUtensorMap* maps, int grid, cudaStream_t s) {
    if (grid % kRsCluster != 0 || grid > kRsMaxG || a.E > kRsMaxE) return cudaErrorInvalidValue;
    if (a.N == 32) return launch_decode_n<32>(a, maps, grid, s);
    if (a.N == 16) return launch_decode_n<16>(a, maps, grid, s);
    return cudaErrorInvalidValue;
}

// Clusters of 4 blocks (one block per SM) that can be resident at once, -1 on error.
int decode_max_clusters() {
    const size_t smem = forward_decode_smem_bytes();
    if (cudaFuncSetAttribute(union_expert_decode<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return -1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kRsCluster);
    cfg.blockDim = dim3(kRsThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kRsCluster;
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
