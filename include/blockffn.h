/*
 * blockffn.h -- C ABI of the BlockFFN chunk-union layer forward on B200 (sm_100a).
 *
 * The layer (pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device
 * Deployment", sections Core Concept and Architecture Overview; "BlockFFN: Towards
 * End-Side Acceleration-Friendly Mixture-of-Experts with Chunk-Level Activation
 * Sparsity", Abstract):
 *
 *   route:  g[t,:] = RMSNorm(ReLU(W_r x_t + b_r))          over the E experts
 *   union:  U_c    = { e : g[t,e] != 0 for some t in chunk c }, chunks of n tokens
 *   expert: o_e(x) = W_out_e Swish(W_in_e x + b_in_e) + b_out_e   non-gated, d_e << d_h
 *                    (the biases are optional)
 *   output: y[t,:] = sum_{e in U_c, ascending} [g[t,e] != 0] g[t,e] o_e(x_t)
 *           optionally followed by y <- LayerNorm(y + x) over d_h
 *
 * Only the union experts run, each over every token of the chunk as one small
 * dense GEMM pair; tokens whose own gate is zero are masked after computing.
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller, contiguous,
 *   row-major, 16-byte aligned.  The library allocates no device memory; scratch
 *   space comes from the caller's workspace (blockffn_forward_workspace_bytes).
 * - Weights follow the nn.Linear convention weight[out, in]:
 *     x [T, d_h]; W_r [E, d_h]; b_r [E] fp32; gamma [E] fp32; gates [T, E] fp32;
 *     W_in [E, d_e, d_h]; W_out [E, d_h, d_e]; y [T, d_h].
 *   x, W_r, W_in, W_out and y share one element type (blockffn_dtype).
 * - Chunks are n consecutive tokens starting at token 0; C = ceil(T / n); the
 *   last chunk may be short (its missing tokens count as inactive).  n in [1, 32].
 * - stream is a cudaStream_t (NULL = the legacy default stream).  Every call is
 *   asynchronous on it, except blockffn_get_device_status, which synchronizes it.
 * - Arguments are validated on the host before anything is launched; a call that
 *   returns an error other than BLOCKFFN_ERR_CUDA has launched nothing.
 * - Device-side failures (a bounded wait that ran out, a corrupted workspace) are
 *   recorded in the workspace status word and read by blockffn_get_device_status.
 *   After one, reset the workspace before the next call.
 * - Results are deterministic: two calls with the same inputs, shapes and device
 *   give bit-identical outputs (every sum runs in a fixed order).
 */
#ifndef BLOCKFFN_H
#define BLOCKFFN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BLOCKFFN_OK = 0,
    BLOCKFFN_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer      */
    BLOCKFFN_ERR_UNSUPPORTED = 2, /* valid but outside what the kernels implement   */
    BLOCKFFN_ERR_CUDA = 3,        /* a CUDA runtime/driver call or launch failed     */
    BLOCKFFN_ERR_TIMEOUT = 4,     /* device: a bounded wait ran out (status word)    */
    BLOCKFFN_ERR_WORKSPACE = 5    /* workspace too small, or found corrupted         */
} blockffn_status;

typedef enum {
    BLOCKFFN_F32 = 0,  /* fp32 values, fp32 arithmetic (CUDA-core FFMA)               */
    BLOCKFFN_BF16 = 1  /* bf16 values, fp32 accumulation (tcgen05 tensor cores)       */
} blockffn_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* blockffn_status_string(blockffn_status s);

/* Text of the last host-side error of the calling thread ("" when none):
 * which check failed, or the CUDA error string.  Valid until the next call. */
const char* blockffn_last_error_message(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int blockffn_version(void);

/*
 * blockffn_route -- the router.
 * Pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device Deployment",
 * Architecture Overview (Router Module: linear map, ReLU, RMSNorm) and Router
 * Architecture Setup (nn.Linear without bias, nn.RMSNorm over the experts).
 *
 *   logit[t,e] = sum_k W_r[e,k] x[t,k] + (b_r ? b_r[e] : 0)      (fp32 accumulation)
 *   r          = max(logit, 0)
 *   gates[t,e] = r > 0 ? gamma[e] * r / sqrt(mean_e' r[t,e']^2 + eps) : 0
 *
 * x [T, d_h] and W_r [E, d_h] in dtype dt; b_r [E] fp32 or NULL; gamma [E] fp32;
 * eps >= 0.  gates [T, E] fp32 output.  Requirements: T >= 0, 1 <= E <= 256,
 * d_h >= 1; bf16 additionally d_h % 64 == 0 and E % 16 == 0.
 * Arithmetic: every sum in a fixed order, so repeated calls give the same bits;
 * bf16 with d_h % 256 == 0 multiplies on the tensor cores, other shapes on the
 * CUDA cores (the two orders differ in rounding, not in what they compute).
 * Stream-ordered; a forward launched right after it may be scheduled early and
 * waits for it before reading the gates.
 */
blockffn_status blockffn_route(const void* x, const void* W_r, const float* b_r,
                               const float* gamma, float eps, int T, int d_h, int E,
                               blockffn_dtype dt, float* gates, void* stream);

/*
 * blockffn_chunk_union -- the union of active experts of each n-token chunk.
 * Pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device Deployment",
 * Core Concept and Architecture Overview (the kernel computes only the union of
 * the experts activated across n tokens).
 *
 *   tmask[c,e]  bit j set  <=>  t = c*n + j < T and gates[t,e] != 0  (IEEE !=)
 *   counts[c]   = number of e with tmask[c,e] != 0
 *   idx[c,s]    = the s-th such e in ascending order for s < counts[c], else -1
 *
 * gates [T, E] fp32 (finite); outputs counts [C] int32, idx [C, E] int32,
 * tmask [C, E] uint32.  Requirements: T >= 0, 1 <= E <= 256, 1 <= n <= 32.
 * Integer results, bit-exact.
 */
blockffn_status blockffn_chunk_union(const float* gates, int T, int E, int n,
                                     int32_t* counts, int32_t* idx, uint32_t* tmask,
                                     void* stream);

/*
 * blockffn_residual_layernorm -- the layer's closing step, out = LayerNorm(y + x)
 * over the hidden dimension:
 *   v = y + x;  mu = mean_k v;  var = mean_k (v - mu)^2  (population variance);
 *   out[t,k] = ln_gamma[k] * (v[t,k] - mu) / sqrt(var + eps) + ln_beta[k].
 * Pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device Deployment",
 * Full BlockFFN Layer with Combined Losses (the expert sum plus the input, through
 * nn.LayerNorm(hidden_dim); its default eps is 1e-5).
 * y, x, out [T, d_h] in dtype dt (out may alias y or x: every element is read
 * before it is written); ln_gamma [d_h] fp32; ln_beta [d_h] fp32 or NULL (no
 * shift); eps finite and >= 0.
 * Arithmetic: fp32 from the dt inputs, the sums in a fixed order, out rounded once
 * to dt.  Stream-ordered; launched as a programmatic dependent of the preceding
 * kernel (it reads nothing before that kernel has completed).
 */
blockffn_status blockffn_residual_layernorm(const void* y, const void* x, const float* ln_gamma,
                                           const float* ln_beta, float eps, int T, int d_h,
                                           blockffn_dtype dt, void* out, void* stream);

/*
 * blockffn_layer_opts -- the optional parts of the layer around the expert sum,
 * passed to blockffn_forward (a NULL pointer there means none of them).
 * Pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device Deployment",
 * Router Architecture Setup (each expert's fc1 and fc2 are nn.Linear layers, which
 * carry a bias unless told otherwise) and Full BlockFFN Layer with Combined Losses
 * (the expert sum plus the layer's input goes through nn.LayerNorm(hidden_dim)).
 *
 *   b_in  [E, d_e] fp32 or NULL    fc1 biases:  h = Swish(W_in_e x + b_in_e)
 *   b_out [E, d_h] fp32 or NULL    fc2 biases:  o_e = W_out_e h' + b_out_e; the gate
 *                                  multiplies the whole o_e, so a token adds
 *                                  g[t,e] b_out_e only for experts it activates
 *   ln_weight [d_h] fp32 or NULL   when given, y = LayerNorm(sum + x): population
 *                                  variance over d_h, scale ln_weight, shift ln_bias
 *   ln_bias   [d_h] fp32 or NULL   (NULL: no shift; ignored without ln_weight)
 *   ln_eps    finite, >= 0         (nn.LayerNorm's default is 1e-5)
 * All pointers are device pointers, 16-byte aligned, owned by the caller.
 */
typedef struct blockffn_layer_opts {
    const float* b_in;
    const float* b_out;
    const float* ln_weight;
    const float* ln_bias;
    float ln_eps;
} blockffn_layer_opts;

/* Flags of blockffn_forward_workspace_bytes. */
#define BLOCKFFN_WS_ROUTER 1      /* the gates will come from the router           */
#define BLOCKFFN_WS_EXPERT_BIAS 2 /* the calls will pass fc2 biases (opts->b_out)  */

/*
 * blockffn_forward_workspace_bytes -- size of the scratch buffer blockffn_forward
 * needs for these shapes (0 when the shapes are invalid).  flags: an OR of
 * BLOCKFFN_WS_ROUTER (the gates come from the router; the workspace then also
 * holds them) and BLOCKFFN_WS_EXPERT_BIAS (fc2 biases are given; the multi-chunk
 * kernels then stage the per-token bias sums, T * d_h fp32, in the workspace).
 * The value 1 means BLOCKFFN_WS_ROUTER, as the flag argument always has.
 */
size_t blockffn_forward_workspace_bytes(int T, int d_h, int E, int d_e, int n,
                                        blockffn_dtype dt, int flags);

/*
 * blockffn_workspace_reset -- zero a workspace (asynchronous memset on stream).
 * Required once before a workspace's first use and after any device-side error.
 */
blockffn_status blockffn_workspace_reset(void* workspace, size_t ws_bytes, void* stream);

/*
 * blockffn_forward -- the layer output y over all chunks.
 * Pages: "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device Deployment",
 * Core Concept (union of activated experts over n tokens, unneeded activations
 * masked after computation), Architecture Overview (non-gated Swish experts),
 * Full BlockFFN Layer with Combined Losses (gate times expert output, summed over
 * experts).
 *
 * Gating source, exactly one of:
 *   gates != NULL : injected gates [T, E] fp32 (W_r, b_r, gamma ignored, must be NULL);
 *   gates == NULL : the router runs first (W_r, gamma required, b_r optional, eps).
 * Union tables (counts [C] int32, idx [C, E] int32, tmask [C, E] uint32, C =
 * ceil(T / n)), either all NULL -- the union is formed from the gates -- or all
 * given, exactly as blockffn_chunk_union returns them for these gates and n
 * (injected gates only).  Given tables replace the union step: the token masks
 * decide which experts run and which tokens are kept; counts and idx are checked
 * against the masks on the device, and a mismatch records
 * BLOCKFFN_ERR_INVALID_ARG in the status word (detail 11) and computes nothing.
 * W_in [E, d_e, d_h] and W_out [E, d_h, d_e] in dtype dt; y [T, d_h] in dtype dt is
 * fully overwritten (without LayerNorm, rows of tokens with no active expert are
 * exact zeros).  opts: NULL, or the optional biases and LayerNorm
 * (blockffn_layer_opts); fc2 biases need a workspace sized with
 * BLOCKFFN_WS_EXPERT_BIAS.  The LayerNorm is a kernel of its own that follows
 * the forward on the stream (a programmatic dependent of it) and rewrites y in
 * place.
 * workspace: ws_bytes >= blockffn_forward_workspace_bytes(...), reset once with
 * blockffn_workspace_reset; it carries state between calls (never share one
 * workspace between calls that may overlap on the GPU).  The first call after a
 * reset binds the workspace to its (T, d_h, E, d_e, n, dt, gating mode); a later
 * call with any of these different records BLOCKFFN_ERR_WORKSPACE in the status
 * word (blockffn_get_device_status, detail 10) and computes nothing.  Reset the
 * workspace, or use another one, to change them.  Calls with and without the
 * optional parts may share a workspace (one sized for fc2 biases serves both).
 * Requirements: T >= 0, 1 <= n <= 32, 1 <= E <= 256;
 *   bf16: d_h % 128 == 0, d_e % 128 == 0, d_e <= 512, E % 16 == 0 when routed;
 *   fp32: any d_h, d_e >= 1.
 * Arithmetic: bf16 inputs, fp32 accumulation; the gated Swish activations are
 * rounded to bf16 between the two GEMMs; the biases and the LayerNorm are fp32;
 * the expert sum is rounded once to dt, and the LayerNorm reads it as stored and
 * rounds its result once more.
 * Kernels: one chunk (T <= n, bf16, d_h % 256 == 0) runs the single-chunk
 * cluster kernel; several chunks run the group kernel, which takes whole chunks
 * 256 tokens at a time (128 when T <= 128) and runs each expert of the group's
 * union once over all of them, masking every token by its own chunk's mask.
 * Ordering: stream-ordered like any kernel launch.  The single-chunk bf16 kernel
 * is launched as a programmatic dependent of the preceding kernel on the
 * stream: its blocks may start while that kernel finishes, but they set up
 * only their own on-chip state before waiting for it to complete, so inputs
 * produced by the preceding kernel (x, gates, tables, weights) are read only
 * after it.
 */
blockffn_status blockffn_forward(const void* x, const float* gates, const void* W_r,
                                 const float* b_r, const float* gamma, float eps,
                                 const int32_t* counts, const int32_t* idx, const uint32_t* tmask,
                                 const void* W_in, const void* W_out, int T, int d_h,
                                 int E, int d_e, int n, blockffn_dtype dt,
                                 const blockffn_layer_opts* opts, void* y,
                                 void* workspace, size_t ws_bytes, void* stream);

/*
 * blockffn_forward_noalloc -- the same layer output as blockffn_forward for ONE
 * chunk with injected gates (T <= n, bf16), for callers that cannot allocate
 * device memory: code running where cudaMalloc is not allowed or not wanted,
 * such as a runtime that plans every device byte ahead of time, a caller inside
 * a region that must not synchronize the device (cudaMalloc can), or a plug-in
 * that receives only input and output buffers from its host.  No counterpart in
 * the paper: this is a calling convention of this library.
 *
 * Arguments as in blockffn_forward (x [T, d_h], gates [T, E] fp32, W_in, W_out,
 * y [T, d_h], device pointers owned by the caller); there is no workspace.  The
 * scratch is a fixed 8 MiB device array inside the library, which every GPU that
 * loads the library holds until the process exits.  Shapes whose scratch would
 * exceed it (roughly E * d_e * 64 bytes) are rejected with
 * BLOCKFFN_ERR_UNSUPPORTED; so are T > n and non-bf16 data.  Nothing is
 * allocated: no cudaMalloc, cudaFree or allocating library call.
 * The first call on a device looks up the scratch's device address (with that
 * device current); make that first call before capturing any CUDA graph.  Every
 * call clears the scratch's counters on `stream` and then launches the forward.
 * All calls share the one scratch array and it keeps the last call's contents:
 * calls that can overlap on the GPU (different streams, or concurrent host
 * threads) race and must not be issued.  Device-side timeouts are not reported
 * back (there is no workspace to read); use blockffn_forward for that.
 */
blockffn_status blockffn_forward_noalloc(const void* x, const float* gates, const void* W_in,
                                         const void* W_out, int T, int d_h, int E, int d_e, int n,
                                         void* y, void* stream);

/*
 * blockffn_get_device_status -- synchronize stream, then read the device status
 * word of a workspace: BLOCKFFN_OK, or the first device-side error recorded
 * (BLOCKFFN_ERR_TIMEOUT, BLOCKFFN_ERR_WORKSPACE).  detail (may be NULL) receives
 * a code naming the wait that ran out (1-9), 10 for a workspace bound to
 * other shapes or another gating mode, or 11 for union tables whose counts or
 * index lists disagree with their token masks.  Returns BLOCKFFN_ERR_CUDA if the
 * synchronization itself failed.
 */
blockffn_status blockffn_get_device_status(const void* workspace, void* stream,
                                           int32_t* detail);

/*
 * blockffn_set_wait_limit_ns -- upper bound, in nanoseconds, of every spin-wait
 * inside the kernels (waits on another thread block's result or on a copy).  A
 * wait that runs out records BLOCKFFN_ERR_TIMEOUT and the kernel returns.  The
 * default is 2e9 (2 s), far above any legitimate wait.  Applies to later launches.
 */
void blockffn_set_wait_limit_ns(uint64_t ns);

/*
 * blockffn_debug_skip_flag -- failure-detection test support.  For later forward
 * launches (bf16 path), the thread blocks that finish expert-in unit `unit`
 * (the unit index is pair * (d_e / 128) + m-tile) write its activations but never
 * count them as ready; the expert-out tiles that need them then wait until the
 * bounded-wait limit runs out, and the launch records BLOCKFFN_ERR_TIMEOUT in the
 * workspace.  -1 (the default) turns it off.
 */
void blockffn_debug_skip_flag(int unit);

/*
 * blockffn_debug_set_trace -- timeline tracing of later bf16 forward launches.
 * device_buffer (device memory, zeroed by the caller, blockffn_num_sms() * 64
 * uint64 entries) receives globaltimer stamps in nanoseconds, 64 entries per
 * thread block.
 * Multi-chunk (group) launches: 0 start, 1 prologue done, 2 first weight load
 * issued, 3 last expert-in weight load issued, 4 last expert-in accumulator
 * committed, 5 expert-in results announced, 6 first expert-out activation tile
 * ready, 7 last expert-out accumulator committed, 8 epilogue done, 9 end,
 * 10 first accumulator drained, 12 last load issued, 13 first expert-in
 * accumulator written out, 14 expert-in announcement begun, 15 first 32-token
 * slice staged; for the first unit's slices s = 0..7, 16 + 4s + {0: TMEM read,
 * 1: staged, 2: barrier passed, 3: stores issued}; 48 expert-out partials
 * written, 49 announced, and for pending split unit k = 0, 1: 50 + 3k
 * contributors counted, 51 + 3k first batch of partials landed, 52 + 3k rows of
 * y stored.
 * Single-chunk launches: 0 start, 1 prologue done,
 * 2 first weight load issued, 3 last load issued, 4 first expert-in tile landed,
 * 5 last expert-in accumulator committed, 7 expert-in units finished, 8 first and
 * 9 last expert slot seen ready, 10 last expert-out accumulator
 * committed, 11 last epilogue step, 13 end; for the block's first expert-in unit:
 * 14 accumulator read, 15 partial sent to the peer, 16 peer's partial received,
 * 17 peer's partial read, 18 h' published; 21 first expert-out quadrant sent,
 * 23 first 32 rows of y summed and stored, 24 first expert-out MMA issued,
 * 30 the other ranks' expert-out partials received (summing warp).
 * Unset stamps stay 0.  NULL (the default) turns tracing off.
 */
void blockffn_debug_set_trace(void* device_buffer);

/*
 * blockffn_num_sms -- streaming multiprocessors of the current device (the grid
 * size of the persistent forward kernel), or -1 on error.
 */
int blockffn_num_sms(void);

#ifdef __cplusplus
}
#endif

#endif /* BLOCKFFN_H */
