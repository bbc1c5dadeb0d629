// abi.cu -- the C ABI of libblockffn (include/blockffn.h): argument checks,
// workspace layout, TMA descriptors and kernel launches.  Nothing here computes
// on the host; every step of the layer runs in the kernels.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdarg>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/blockffn.h"
#include "common.cuh"
#include "launch.h"

namespace {

using namespace bffn;

std::atomic<unsigned long long> g_wait_ns{2000000000ull};
std::atomic<int> g_skip_flag{-1};
std::atomic<unsigned long long*> g_trace{nullptr};
thread_local char g_msg[512] = "";

blockffn_status fail(blockffn_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return st;
}

blockffn_status cuda_fail(cudaError_t e, const char* where) {
    return fail(BLOCKFFN_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms_current() {
    static int cache[64];
    static std::once_flag once[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    std::call_once(once[dev], [dev]() {
        int v = 0;
        cache[dev] = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? v : -1;
    });
    return cache[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, []() {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D bf16 tensor [outer, inner] (inner contiguous), box {64, box_outer}, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {64, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A bf16 matrix [rows, cols] (cols contiguous, row pitch cols*2 bytes) seen as a
// 3-D tensor {64-wide column block element, row, column block}: a box {64,
// box_rows, 2} fetches two consecutive 64-column blocks of box_rows rows and
// lands as two [box_rows x 128 B] 128-byte-swizzled tiles, one after the other.
// One TMA operation instead of two: the per-operation cost dominates below
// ~32 KB.  cols must be a multiple of 128.  map_kblocks is the same with nkb
// consecutive column blocks per box (cols a multiple of 64 * nkb).
bool map_kblocks(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows,
                 uint32_t nkb) {
    auto fn = encode_fn();
    if (fn == nullptr || cols % (64 * nkb) != 0) return false;
    cuuint64_t dims[3] = {64, rows, cols / 64};
    cuuint64_t strides[2] = {cols * 2, 128};
    cuuint32_t box[3] = {64, box_rows, nkb};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_kpair(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
    return map_kblocks(m, base, cols, rows, box_rows, 2);
}

// 2-D fp32 tensor [outer, inner], box {box_inner, box_outer}, no swizzle.
bool make_map_f32(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                  uint32_t box_outer) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * 4};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 tensor [outer, inner], box {box_inner, box_outer}, no swizzle (for
// tiled stores from a plain row-major shared-memory tile).
bool make_map_plain(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                    uint32_t box_outer) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Which kernel computes a forward call.
enum class Path { F32, Decode, Group };

// Workspace layout of one forward call (byte offsets; 0 = not used by the path).
struct Layout {
    Path path;
    size_t ctl, counts, offsets, idx, tmask, pair_ce, gcounts, goffsets, gpair, gates;
    size_t readyA, cntB, partB, hbuf;
    size_t ybias;        // group path with fc2 biases: [T, d_h] fp32 per-token bias sums
    size_t total;
    int C;               // chunks
    int N;               // tokens per MMA
    int NG, NT, NGr;     // group kernel: chunks and tokens per group, groups
    int MT, RT, KB, KBe;
    long long Pmax;      // pairs the tables can hold
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int decode_clusters_current() {
    static int cache[64];
    static std::once_flag once[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    std::call_once(once[dev], [dev]() { cache[dev] = decode_max_clusters(); });
    return cache[dev];
}

// The single-chunk kernel's grid (4 blocks per cluster), or 0 when it cannot run
// these shapes here.
int decode_grid(int C, int d_h, int E, int G) {
    if (C != 1 || (d_h / 64) % 4 != 0 || E > 256) return 0;
    int ncl = decode_clusters_current();
    if (ncl > G / 4) ncl = G / 4;
    if (ncl <= 0 || 4 * ncl > 160) return 0;
    return 4 * ncl;
}

void make_layout(int T, int d_h, int E, int d_e, int n, bool bf16, bool with_router, bool with_bias, int G,
                 Layout& L) {
    L.C = (T + n - 1) / n;
    L.MT = bf16 ? d_e / 128 : 1;
    L.RT = bf16 ? d_h / 128 : 1;
    L.KB = bf16 ? d_h / 64 : 1;
    L.KBe = bf16 ? d_e / 64 : 1;
    L.path = !bf16 ? Path::F32 : (decode_grid(L.C, d_h, E, G) > 0 ? Path::Decode : Path::Group);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + (bytes > 0 ? bytes : 1), 256);
        return o;
    };
    L.ctl = L.counts = L.offsets = L.idx = L.tmask = L.pair_ce = L.gcounts = L.goffsets = L.gpair = 0;
    L.gates = L.readyA = L.cntB = L.partB = L.hbuf = L.ybias = 0;
    L.NG = L.NT = L.NGr = 0;
    const size_t C = (size_t)L.C;
    L.ctl = take(sizeof(Ctl));
    if (with_router) L.gates = take((size_t)T * E * 4);
    if (L.path == Path::F32) {
        L.N = n;
        L.Pmax = (long long)L.C * E;
        L.counts = take(C * 4);
        L.offsets = take((C + 1) * 4);
        L.idx = take(C * E * 4);
        L.tmask = take(C * E * 4);
        L.pair_ce = take((size_t)L.Pmax * 4);
        L.hbuf = take((size_t)L.Pmax * n * d_e * 4);
    } else if (L.path == Path::Decode) {
        // the single-chunk kernel forms the union itself: counters and h' only
        L.N = n <= 16 ? 16 : 32;
        L.Pmax = E;
        L.readyA = take(2 * (size_t)E * 4);
        L.hbuf = take((size_t)E * L.N * d_e * 2);
    } else {
        // groups of whole chunks, N = 128 tokens per MMA for short inputs, else 256
        L.N = T <= 128 ? 128 : 256;
        L.NG = L.N / n;
        L.NT = L.NG * n;
        L.NGr = (L.C + L.NG - 1) / L.NG;
        L.Pmax = (long long)L.NGr * E;
        const size_t NGr = (size_t)L.NGr, Pm = (size_t)L.Pmax;
        L.counts = take(C * 4);
        L.idx = take(C * E * 4);
        L.tmask = take(C * E * 4);
        L.gcounts = take(NGr * 4);
        L.goffsets = take((NGr + 1) * 4);
        L.gpair = take(Pm * 4);
        L.readyA = take(2 * Pm * L.MT * 4);
        L.cntB = take(2 * NGr * L.RT * 4);
        L.partB = take((size_t)G * 2 * L.N * 128 * 4);
        L.hbuf = take(Pm * L.N * d_e * 2);
        // last, so that every other offset is the same with or without it
        if (with_bias) L.ybias = take((size_t)T * d_h * 4);
    }
    L.total = off;
}

blockffn_status check_shapes(int T, int d_h, int E, int d_e, int n, blockffn_dtype dt) {
    if (dt != BLOCKFFN_F32 && dt != BLOCKFFN_BF16) return fail(BLOCKFFN_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    if (T < 0) return fail(BLOCKFFN_ERR_INVALID_ARG, "T = %d < 0", T);
    if (n < 1 || n > 32) return fail(BLOCKFFN_ERR_INVALID_ARG, "chunk length n = %d outside [1, 32]", n);
    if (E < 1 || E > 256) return fail(BLOCKFFN_ERR_INVALID_ARG, "E = %d outside [1, 256]", E);
    if (d_h < 1 || d_e < 1) return fail(BLOCKFFN_ERR_INVALID_ARG, "d_h = %d, d_e = %d must be >= 1", d_h, d_e);
    const long long C = ((long long)T + n - 1) / n;
    if (C > (1LL << 22)) return fail(BLOCKFFN_ERR_UNSUPPORTED, "too many chunks (%lld)", C);
    if (dt == BLOCKFFN_BF16) {
        if (d_h % 128 != 0) return fail(BLOCKFFN_ERR_UNSUPPORTED, "bf16 needs d_h %% 128 == 0 (d_h = %d)", d_h);
        if (d_e % 128 != 0 || d_e > 512)
            return fail(BLOCKFFN_ERR_UNSUPPORTED, "bf16 needs d_e in {128, 256, 384, 512} (d_e = %d)", d_e);
    } else {
        if (C > 65535) return fail(BLOCKFFN_ERR_UNSUPPORTED, "fp32 path: at most 65535 chunks");
    }
    return BLOCKFFN_OK;
}

}  // namespace

// for the kernels' own launchers (launch.h)
bool bffn::make_map_kblocks(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows,
                            uint32_t nkb) {
    return map_kblocks(m, base, cols, rows, box_rows, nkb);
}

extern "C" {

const char* blockffn_status_string(blockffn_status s) {
    switch (s) {
        case BLOCKFFN_OK: return "ok";
        case BLOCKFFN_ERR_INVALID_ARG: return "invalid argument";
        case BLOCKFFN_ERR_UNSUPPORTED: return "unsupported shape or type";
        case BLOCKFFN_ERR_CUDA: return "CUDA error";
        case BLOCKFFN_ERR_TIMEOUT: return "device wait timed out";
        case BLOCKFFN_ERR_WORKSPACE: return "workspace too small or corrupted";
    }
    return "unknown status";
}

const char* blockffn_last_error_message(void) { return g_msg; }

int blockffn_version(void) { return 20000; }

void blockffn_set_wait_limit_ns(uint64_t ns) { g_wait_ns.store(ns > 0 ? ns : 1); }

int blockffn_num_sms(void) { return num_sms_current(); }

void blockffn_debug_skip_flag(int unit) { g_skip_flag.store(unit < 0 ? -1 : unit); }

void blockffn_debug_set_trace(void* device_buffer) {
    g_trace.store(static_cast<unsigned long long*>(device_buffer));
}

blockffn_status blockffn_route(const void* x, const void* W_r, const float* b_r,
                               const float* gamma, float eps, int T, int d_h, int E,
                               blockffn_dtype dt, float* gates, void* stream) {
    if (dt != BLOCKFFN_F32 && dt != BLOCKFFN_BF16) return fail(BLOCKFFN_ERR_INVALID_ARG, "unknown dtype");
    if (T < 0 || d_h < 1 || E < 1 || E > 256) return fail(BLOCKFFN_ERR_INVALID_ARG, "bad shape");
    if (!(eps >= 0.f) || !std::isfinite(eps)) return fail(BLOCKFFN_ERR_INVALID_ARG, "eps must be finite and >= 0");
    if (dt == BLOCKFFN_BF16 && (d_h % 64 != 0 || E % 16 != 0))
        return fail(BLOCKFFN_ERR_UNSUPPORTED, "bf16 router needs d_h %% 64 == 0 and E %% 16 == 0");
    if (T == 0) return BLOCKFFN_OK;
    if (!x || !W_r || !gamma || !gates) return fail(BLOCKFFN_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(x) || !aligned16(W_r) || !aligned16(gates) || !aligned16(gamma) || (b_r && !aligned16(b_r)))
        return fail(BLOCKFFN_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    cudaError_t e = launch_route(x, W_r, b_r, gamma, eps, T, d_h, E, dt == BLOCKFFN_BF16, gates,
                                 static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BLOCKFFN_OK : cuda_fail(e, "route launch");
}

blockffn_status blockffn_residual_layernorm(const void* y, const void* x, const float* ln_gamma,
                                           const float* ln_beta, float eps, int T, int d_h, blockffn_dtype dt,
                                           void* out, void* stream) {
    if (dt != BLOCKFFN_F32 && dt != BLOCKFFN_BF16) return fail(BLOCKFFN_ERR_INVALID_ARG, "unknown dtype");
    if (T < 0 || d_h < 1) return fail(BLOCKFFN_ERR_INVALID_ARG, "bad shape (T = %d, d_h = %d)", T, d_h);
    if (!(eps >= 0.f) || !std::isfinite(eps)) return fail(BLOCKFFN_ERR_INVALID_ARG, "eps must be finite and >= 0");
    if (T == 0) return BLOCKFFN_OK;
    if (!y || !x || !ln_gamma || !out) return fail(BLOCKFFN_ERR_INVALID_ARG, "null pointer");
    cudaError_t e = launch_residual_layernorm(y, x, ln_gamma, ln_beta, eps, T, d_h, dt == BLOCKFFN_BF16, out,
                                              static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BLOCKFFN_OK : cuda_fail(e, "residual layernorm launch");
}

blockffn_status blockffn_chunk_union(const float* gates, int T, int E, int n, int32_t* counts,
                                     int32_t* idx, uint32_t* tmask, void* stream) {
    if (T < 0 || E < 1 || E > 256 || n < 1 || n > 32) return fail(BLOCKFFN_ERR_INVALID_ARG, "bad shape");
    if (T == 0) return BLOCKFFN_OK;
    if (!gates || !counts || !idx || !tmask) return fail(BLOCKFFN_ERR_INVALID_ARG, "null pointer");
    cudaError_t e = launch_chunk_union(gates, T, E, n, counts, idx, tmask, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BLOCKFFN_OK : cuda_fail(e, "chunk_union launch");
}

size_t blockffn_forward_workspace_bytes(int T, int d_h, int E, int d_e, int n, blockffn_dtype dt, int flags) {
    if (check_shapes(T, d_h, E, d_e, n, dt) != BLOCKFFN_OK) return 0;
    if ((flags & ~(BLOCKFFN_WS_ROUTER | BLOCKFFN_WS_EXPERT_BIAS)) != 0) return 0;
    const int G = num_sms_current();
    if (G <= 0) return 0;
    Layout L;
    make_layout(T, d_h, E, d_e, n, dt == BLOCKFFN_BF16, (flags & BLOCKFFN_WS_ROUTER) != 0,
                (flags & BLOCKFFN_WS_EXPERT_BIAS) != 0, G, L);
    return L.total;
}

blockffn_status blockffn_workspace_reset(void* workspace, size_t ws_bytes, void* stream) {
    if (!workspace || ws_bytes == 0) return fail(BLOCKFFN_ERR_INVALID_ARG, "null workspace");
    cudaError_t e = cudaMemsetAsync(workspace, 0, ws_bytes, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BLOCKFFN_OK : cuda_fail(e, "workspace memset");
}

blockffn_status blockffn_forward(const void* x, const float* gates, const void* W_r,
                                 const float* b_r, const float* gamma, float eps,
                                 const int32_t* counts, const int32_t* idx, const uint32_t* tmask,
                                 const void* W_in, const void* W_out, int T, int d_h, int E,
                                 int d_e, int n, blockffn_dtype dt, const blockffn_layer_opts* opts,
                                 void* y, void* workspace, size_t ws_bytes, void* stream) {
    blockffn_status st = check_shapes(T, d_h, E, d_e, n, dt);
    if (st != BLOCKFFN_OK) return st;
    if (T == 0) return BLOCKFFN_OK;   // nothing to compute (empty tensors may be NULL)
    const bool routed = gates == nullptr;
    const int ntab = (counts != nullptr) + (idx != nullptr) + (tmask != nullptr);
    if (ntab != 0 && ntab != 3)
        return fail(BLOCKFFN_ERR_INVALID_ARG, "pass all of counts, idx and tmask, or none of them");
    const bool tables = ntab == 3;
    if (routed) {
        if (!W_r || !gamma) return fail(BLOCKFFN_ERR_INVALID_ARG, "no gates: W_r and gamma are required");
        if (!(eps >= 0.f) || !std::isfinite(eps)) return fail(BLOCKFFN_ERR_INVALID_ARG, "eps must be finite and >= 0");
        if (dt == BLOCKFFN_BF16 && E % 16 != 0)
            return fail(BLOCKFFN_ERR_UNSUPPORTED, "bf16 router needs E %% 16 == 0");
        if (tables)
            return fail(BLOCKFFN_ERR_INVALID_ARG, "union tables can only come with injected gates");
    } else if (W_r || b_r || gamma) {
        return fail(BLOCKFFN_ERR_INVALID_ARG, "pass either gates or router weights, not both");
    }
    if (!x || !W_in || !W_out || !y || !workspace) return fail(BLOCKFFN_ERR_INVALID_ARG, "null pointer");
    const float* b_in = opts ? opts->b_in : nullptr;
    const float* b_out = opts ? opts->b_out : nullptr;
    const float* ln_w = opts ? opts->ln_weight : nullptr;
    const float* ln_b = (opts && ln_w) ? opts->ln_bias : nullptr;
    const float ln_eps = opts ? opts->ln_eps : 0.f;
    if (ln_w && (!(ln_eps >= 0.f) || !std::isfinite(ln_eps)))
        return fail(BLOCKFFN_ERR_INVALID_ARG, "ln_eps must be finite and >= 0");
    if ((b_in && !aligned16(b_in)) || (b_out && !aligned16(b_out)) || (ln_w && !aligned16(ln_w)) ||
        (ln_b && !aligned16(ln_b)))
        return fail(BLOCKFFN_ERR_INVALID_ARG, "bias and LayerNorm pointers must be 16-byte aligned");
    if (!aligned16(x) || !aligned16(W_in) || !aligned16(W_out) || !aligned16(y) ||
        !aligned16(workspace) || (gates && !aligned16(gates)) || (W_r && !aligned16(W_r)) ||
        (gamma && !aligned16(gamma)) || (b_r && !aligned16(b_r)) || (counts && !aligned16(counts)) ||
        (idx && !aligned16(idx)) || (tmask && !aligned16(tmask)))
        return fail(BLOCKFFN_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    const int G = num_sms_current();
    if (G <= 0) return fail(BLOCKFFN_ERR_CUDA, "no current CUDA device");
    const bool bf16 = dt == BLOCKFFN_BF16;
    const bool with_bias = b_out != nullptr;
    Layout L;
    make_layout(T, d_h, E, d_e, n, bf16, routed, with_bias, G, L);
    if (ws_bytes < L.total)
        return fail(BLOCKFFN_ERR_WORKSPACE, "workspace of %zu bytes < %zu needed%s", ws_bytes, L.total,
                    with_bias ? " (fc2 biases: size it with BLOCKFFN_WS_EXPERT_BIAS)" : "");
    // the LayerNorm as its own kernel after the forward (a programmatic dependent
    // of it), rewriting y in place
    auto closing_layernorm = [&]() -> blockffn_status {
        if (!ln_w) return BLOCKFFN_OK;
        cudaError_t e2 = launch_residual_layernorm(y, x, ln_w, ln_b, ln_eps, T, d_h, bf16, y,
                                                   static_cast<cudaStream_t>(stream));
        return e2 == cudaSuccess ? BLOCKFFN_OK : cuda_fail(e2, "residual layernorm launch");
    };
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    Ctl* ctl = reinterpret_cast<Ctl*>(ws + L.ctl);
    cudaError_t e;

    const float* g = gates;
    if (routed) {
        float* gw = reinterpret_cast<float*>(ws + L.gates);
        e = launch_route(x, W_r, b_r, gamma, eps, T, d_h, E, bf16, gw, s);
        if (e != cudaSuccess) return cuda_fail(e, "route launch");
        g = gw;
    }
    // the union tables: the caller's (checked on the device against its token
    // masks), or the workspace's, computed from the gates
    int32_t* t_counts = tables ? const_cast<int32_t*>(counts) : reinterpret_cast<int32_t*>(ws + L.counts);
    int32_t* t_idx = tables ? const_cast<int32_t*>(idx) : reinterpret_cast<int32_t*>(ws + L.idx);
    uint32_t* t_tmask = tables ? const_cast<uint32_t*>(tmask) : reinterpret_cast<uint32_t*>(ws + L.tmask);

    if (L.path == Path::F32) {
        int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
        int32_t* pair_ce = reinterpret_cast<int32_t*>(ws + L.pair_ce);
        e = launch_chunk_union_plan(g, T, E, n, t_counts, t_idx, t_tmask, !tables, ctl, offsets, pair_ce, y,
                                    d_h, 4, s);
        if (e != cudaSuccess) return cuda_fail(e, "union launch");
        e = launch_forward_f32(static_cast<const float*>(x), g, static_cast<const float*>(W_in),
                               static_cast<const float*>(W_out), b_in, b_out, t_counts, offsets, pair_ce,
                               t_tmask, ctl, reinterpret_cast<float*>(ws + L.hbuf), T, d_h, E, d_e, n,
                               static_cast<float*>(y), G, s);
        if (e != cudaSuccess) return cuda_fail(e, "fp32 forward launch");
        return closing_layernorm();
    }

    if (L.path == Path::Decode) {
        // one chunk: clusters of 4 blocks, expert-in in k-half pairs, expert-out
        // row tiles summed inside the cluster (forward_decode.cu)
        const int Gd = decode_grid(L.C, d_h, E, G);
        CUtensorMap dmaps[5];
        if (!make_map_kpair(&dmaps[0], x, (uint64_t)d_h, (uint64_t)T, (uint32_t)L.N) ||
            !make_map_kpair(&dmaps[1], W_in, (uint64_t)d_h, (uint64_t)E * d_e, 128) ||
            !make_map_kpair(&dmaps[2], W_out, (uint64_t)d_e, (uint64_t)E * d_h, 128) ||
            !make_map_kpair(&dmaps[3], ws + L.hbuf, (uint64_t)d_e, (uint64_t)E * L.N, (uint32_t)L.N) ||
            !make_map_plain(&dmaps[4], y, (uint64_t)d_h, (uint64_t)T, 32, (uint32_t)L.N))
            return fail(BLOCKFFN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
        DcArgs da;
        da.gates = g;
        da.counts_in = tables ? counts : nullptr;
        da.idx_in = tables ? idx : nullptr;
        da.tmask_in = tables ? tmask : nullptr;
        da.y = static_cast<__nv_bfloat16*>(y);
        da.hbuf = reinterpret_cast<__nv_bfloat16*>(ws + L.hbuf);
        da.readyA = reinterpret_cast<uint32_t*>(ws + L.readyA);
        da.ctl = ctl;
        da.b_in = b_in;
        da.b_out = b_out;
        da.T = T;
        da.d_h = d_h;
        da.E = E;
        da.d_e = d_e;
        da.n = n;
        da.N = L.N;
        da.KB = L.KB;
        da.RT = L.RT;
        da.skip_unit = g_skip_flag.load();
        da.wait_ns = g_wait_ns.load();
        da.trace = g_trace.load();
        da.shape_key = shape_key({T, d_h, E, d_e, n, (long long)dt, routed ? 1 : 0, 1, Gd});
        // A cluster launch cannot also be cooperative; the grid is sized to the
        // clusters that can be resident at once, and every wait is bounded.
        e = launch_forward_decode(da, dmaps, Gd, s);
        if (e != cudaSuccess) return cuda_fail(e, "single-chunk forward launch");
        return closing_layernorm();
    }

    // several chunks (or one the single-chunk kernel cannot take): group tables,
    // then the group-major kernel (forward_group.cu)
    int32_t* gcounts = reinterpret_cast<int32_t*>(ws + L.gcounts);
    int32_t* goffsets = reinterpret_cast<int32_t*>(ws + L.goffsets);
    int32_t* gpair = reinterpret_cast<int32_t*>(ws + L.gpair);
    e = launch_group_plan(g, T, E, n, t_counts, t_idx, t_tmask, !tables, ctl, L.NG, L.NGr, gcounts, goffsets,
                          gpair, static_cast<__nv_bfloat16*>(y), d_h, s);
    if (e != cudaSuccess) return cuda_fail(e, "group plan launch");
    float* ybias = with_bias ? reinterpret_cast<float*>(ws + L.ybias) : nullptr;
    if (with_bias) {
        e = launch_expert_bias_sum(g, t_counts, t_idx, t_tmask, ctl, b_out, T, d_h, E, n, ybias, s);
        if (e != cudaSuccess) return cuda_fail(e, "expert bias launch");
    }
    CUtensorMap maps[5];
    // expert-out partial tiles [blocks][2 slots][N/4 token quads][128 rows x 4 tokens]
    // fp32, seen as lines of 512 floats; a box is 32 rows of every token quad
    if (!make_map(&maps[0], x, (uint64_t)d_h, (uint64_t)T, (uint32_t)L.N) ||
        !make_map(&maps[1], W_in, (uint64_t)d_h, (uint64_t)E * d_e, 128) ||
        !make_map(&maps[2], W_out, (uint64_t)d_e, (uint64_t)E * d_h, 128) ||
        !make_map(&maps[3], ws + L.hbuf, (uint64_t)d_e, (uint64_t)L.Pmax * L.N, (uint32_t)L.N) ||
        !make_map_f32(&maps[4], ws + L.partB, 512, (uint64_t)G * 2 * (L.N / 4), 128, (uint32_t)(L.N / 4)))
        return fail(BLOCKFFN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    GrArgs a;
    a.gates = g;
    a.tmask = t_tmask;
    a.gcounts = gcounts;
    a.goffsets = goffsets;
    a.gpair = gpair;
    a.hbuf = reinterpret_cast<__nv_bfloat16*>(ws + L.hbuf);
    a.partB = reinterpret_cast<float*>(ws + L.partB);
    a.readyA = reinterpret_cast<uint32_t*>(ws + L.readyA);
    a.cntB = reinterpret_cast<uint32_t*>(ws + L.cntB);
    a.cnt_a_len = L.Pmax * L.MT;
    a.cnt_b_len = (long long)L.NGr * L.RT;
    a.ctl = ctl;
    a.y = static_cast<__nv_bfloat16*>(y);
    a.b_in = b_in;
    a.ybias = ybias;
    a.T = T;
    a.d_h = d_h;
    a.E = E;
    a.d_e = d_e;
    a.n = n;
    a.N = L.N;
    a.NT = L.NT;
    a.NGr = L.NGr;
    a.KB = L.KB;
    a.MT = L.MT;
    a.RT = L.RT;
    a.KBe = L.KBe;
    a.skip_flag_unit = g_skip_flag.load();
    a.wait_ns = g_wait_ns.load();
    a.shape_key = shape_key({T, d_h, E, d_e, n, (long long)dt, routed ? 1 : 0, 2, G});
    a.trace = g_trace.load();
    e = launch_forward_group(a, maps, G, s);
    if (e != cudaSuccess) return cuda_fail(e, "group forward launch");
    return closing_layernorm();
}

// ------------------------------------------------------------------------
// blockffn_forward_noalloc: the single-chunk forward without a caller-provided
// workspace.  Its scratch is the file-scope device array below, which every GPU
// that loads this library holds until the process exits.  Host code must not
// pass g_noalloc_scratch itself to a kernel (on the host it names a host-side
// stand-in); the device address comes from cudaGetSymbolAddress, taken once per
// device on the first call with that device current.
// ------------------------------------------------------------------------
}  // extern "C"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void* noalloc_scratch_ptr(int dev, cudaError_t* err) {
    static void* ptrs[64];
    static cudaError_t errs[64];
    static std::once_flag once[64];
    std::call_once(once[dev], [dev]() {
        void* p = nullptr;
        errs[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);   // the current device is `dev`
        ptrs[dev] = errs[dev] == cudaSuccess ? p : nullptr;
    });
    *err = errs[dev];
    return ptrs[dev];
}

}  // namespace

extern "C" {

blockffn_status blockffn_forward_noalloc(const void* x, const float* gates, const void* W_in,
                                         const void* W_out, int T, int d_h, int E, int d_e, int n,
                                         void* y, void* stream) {
    blockffn_status st = check_shapes(T, d_h, E, d_e, n, BLOCKFFN_BF16);
    if (st != BLOCKFFN_OK) return st;
    if (T > n) return fail(BLOCKFFN_ERR_UNSUPPORTED, "no-allocation forward: one chunk only (T = %d > n = %d)", T, n);
    if (T == 0) return BLOCKFFN_OK;
    if (!x || !gates || !W_in || !W_out || !y) return fail(BLOCKFFN_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(x) || !aligned16(gates) || !aligned16(W_in) || !aligned16(W_out) || !aligned16(y))
        return fail(BLOCKFFN_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return fail(BLOCKFFN_ERR_CUDA, "no current CUDA device");
    const int G = num_sms_current();
    const int Gd = decode_grid(1, d_h, E, G);
    if (Gd <= 0)
        return fail(BLOCKFFN_ERR_UNSUPPORTED, "no-allocation forward: single-chunk kernel unavailable here");
    const int N = n <= 16 ? 16 : 32;
    const int RT = d_h / 128;
    // scratch layout: control block and readiness counters (the part that must
    // start at zero), then h'
    const size_t off_ready = 256;
    const size_t zero_bytes = align_up(off_ready + 2 * (size_t)E * 4, 256);
    const size_t off_h = zero_bytes;
    const size_t need = off_h + (size_t)E * N * d_e * 2;
    if (need > kNoAllocScratchBytes)
        return fail(BLOCKFFN_ERR_UNSUPPORTED,
                    "no-allocation forward: these shapes need %zu bytes of scratch, more than the %zu "
                    "reserved (E * d_e too large)", need, kNoAllocScratchBytes);
    cudaError_t e = cudaSuccess;
    char* scratch = static_cast<char*>(noalloc_scratch_ptr(dev, &e));
    if (scratch == nullptr) return cuda_fail(e, "cudaGetSymbolAddress(no-allocation scratch)");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // every call starts from a clean control block and counters
    e = cudaMemsetAsync(scratch, 0, zero_bytes, s);
    if (e != cudaSuccess) return cuda_fail(e, "no-allocation scratch clear");
    CUtensorMap dmaps[5];
    if (!make_map_kpair(&dmaps[0], x, (uint64_t)d_h, (uint64_t)T, (uint32_t)N) ||
        !make_map_kpair(&dmaps[1], W_in, (uint64_t)d_h, (uint64_t)E * d_e, 128) ||
        !make_map_kpair(&dmaps[2], W_out, (uint64_t)d_e, (uint64_t)E * d_h, 128) ||
        !make_map_kpair(&dmaps[3], scratch + off_h, (uint64_t)d_e, (uint64_t)E * N, (uint32_t)N) ||
        !make_map_plain(&dmaps[4], y, (uint64_t)d_h, (uint64_t)T, 32, (uint32_t)N))
        return fail(BLOCKFFN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    DcArgs da;
    da.gates = gates;
    da.counts_in = nullptr;
    da.idx_in = nullptr;
    da.tmask_in = nullptr;
    da.y = static_cast<__nv_bfloat16*>(y);
    da.hbuf = reinterpret_cast<__nv_bfloat16*>(scratch + off_h);
    da.readyA = reinterpret_cast<uint32_t*>(scratch + off_ready);
    da.ctl = reinterpret_cast<Ctl*>(scratch);
    da.b_in = nullptr;
    da.b_out = nullptr;
    da.T = T;
    da.d_h = d_h;
    da.E = E;
    da.d_e = d_e;
    da.n = n;
    da.N = N;
    da.KB = d_h / 64;
    da.RT = RT;
    da.skip_unit = -1;
    da.wait_ns = g_wait_ns.load();
    da.trace = nullptr;
    da.shape_key = shape_key({T, d_h, E, d_e, n, (long long)BLOCKFFN_BF16, 0, 3, Gd});
    e = launch_forward_decode(da, dmaps, Gd, s);
    return e == cudaSuccess ? BLOCKFFN_OK : cuda_fail(e, "no-allocation forward launch");
}

blockffn_status blockffn_get_device_status(const void* workspace, void* stream, int32_t* detail) {
    if (!workspace) return fail(BLOCKFFN_ERR_INVALID_ARG, "null workspace");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t h[2] = {0, 0};
    cudaError_t e = cudaMemcpyAsync(h, workspace, sizeof(h), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "device status read");
    if (detail) *detail = h[1];
    return static_cast<blockffn_status>(h[0]);
}

}  // extern "C"
