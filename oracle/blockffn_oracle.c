/*
 * blockffn_oracle.c -- plain, slow, fp64 CPU oracle of the BlockFFN layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load
 * this file or the library built from it: only the tests, the smoke check and the
 * CPU-baseline leg of the benchmark use it.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * Sources (the method as the pages state it):
 *   [SKILL]  "BlockFFN: Sparse Mixture-of-Experts Optimized for End-Device Deployment"
 *            (skill page), sections "Core Concept", "Architecture Overview",
 *            "Router Architecture Setup", "Full BlockFFN Layer with Combined Losses",
 *            "Chunk Sparsification Loss", "Key Hyperparameters".
 *   [ABS]    "BlockFFN: Towards End-Side Acceleration-Friendly Mixture-of-Experts with
 *            Chunk-Level Activation Sparsity", Abstract.
 *
 * All arithmetic is IEEE fp64, in the order the definitions are written: plain
 * loops, no blocking, no reassociation (build without -ffast-math).  Inputs are
 * the values the GPU sees (bf16- or fp32-representable), widened to fp64 exactly.
 *
 * Layouts (row-major, nn.Linear convention weight = [out, in]):
 *   x      [T, d_h]          tokens
 *   W_r    [E, d_h]          router weight;  b_r [E] optional router bias
 *   gamma  [E]               RMSNorm scale
 *   gates  [T, E]
 *   W_in   [E, d_e, d_h]     expert fc1 weights;  b_in  [E, d_e] optional fc1 biases
 *   W_out  [E, d_h, d_e]     expert fc2 weights;  b_out [E, d_h] optional fc2 biases
 *   y      [T, d_h]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Router.  [SKILL] "Architecture Overview" (Router Module) and [ABS]: a linear map
 * of the token, then ReLU, then RMSNorm over the expert axis with a learnable
 * per-expert scale.  "Router Architecture Setup" gives nn.Linear(hidden, E, bias
 * off) and nn.RMSNorm(E).
 *
 *   logits[t,e] = sum_k W_r[e,k] x[t,k]  (+ b_r[e] when b_r != NULL)
 *   r[t,e]      = max(logits[t,e], 0)
 *   g[t,e]      = gamma[e] * r[t,e] / sqrt( (1/E) sum_e' r[t,e']^2 + eps )
 *
 * Reading: RMSNorm rescales each token's row; entries that ReLU zeroed stay
 * exactly zero (they are selected to 0, so eps = 0 with an all-zero row gives 0,
 * not 0/0).  logits may be NULL.
 */
void oracle_route(const double* x, const double* W_r, const double* b_r,
                  const double* gamma, double eps, int T, int d_h, int E,
                  double* logits, double* gates)
{
    int t;
#pragma omp parallel for schedule(static)
    for (t = 0; t < T; ++t) {
        double* r = (double*)malloc(sizeof(double) * (size_t)E);
        double ms = 0.0;
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int k = 0; k < d_h; ++k)
                s += W_r[(size_t)e * d_h + k] * x[(size_t)t * d_h + k];
            if (b_r) s += b_r[e];
            if (logits) logits[(size_t)t * E + e] = s;
            r[e] = s > 0.0 ? s : 0.0;
        }
        for (int e = 0; e < E; ++e) ms += r[e] * r[e];
        ms /= (double)E;
        for (int e = 0; e < E; ++e)
            gates[(size_t)t * E + e] = r[e] > 0.0 ? gamma[e] * r[e] / sqrt(ms + eps) : 0.0;
        free(r);
    }
}

/*
 * Chunk union.  [SKILL] "Core Concept" / "Architecture Overview" (CUTLASS
 * acceleration kernel): the accelerator runs, for a chunk of n consecutive
 * tokens, the union of the experts any of them activates.  Chunks do not overlap
 * and start at token 0; the last one may be short ([SKILL] "Chunk
 * Sparsification Loss" splits the sequence the same way).
 *
 *   C            = ceil(T / n)
 *   tmask[c,e]   bit j set  <=>  t = c*n + j < T  and  gates[t,e] != 0
 *   U_c          = { e : tmask[c,e] != 0 }, ascending
 *   counts[c]    = |U_c|;  idx[c, 0..counts[c]-1] = U_c;  idx[c, counts[c]..E-1] = -1
 *
 * A token is active for an expert when its gate is non-zero (IEEE !=, so -0.0
 * counts as zero).  n must be in [1, 32].
 */
void oracle_chunk_union(const double* gates, int T, int E, int n,
                        int32_t* counts, int32_t* idx, uint32_t* tmask)
{
    int C = (T + n - 1) / n;
    for (int c = 0; c < C; ++c) {
        int cnt = 0;
        for (int e = 0; e < E; ++e) {
            uint32_t bits = 0u;
            for (int j = 0; j < n; ++j) {
                int t = c * n + j;
                if (t < T && gates[(size_t)t * E + e] != 0.0) bits |= (1u << j);
            }
            tmask[(size_t)c * E + e] = bits;
            if (bits != 0u) idx[(size_t)c * E + cnt++] = e;
        }
        counts[c] = cnt;
        for (int s = cnt; s < E; ++s) idx[(size_t)c * E + s] = -1;
    }
}

/* Swish / SiLU, [SKILL] "Architecture Overview" (Expert Modules): z * sigmoid(z). */
static double silu(double z) { return z / (1.0 + exp(-z)); }

/*
 * One expert on one token.  [SKILL] "Router Architecture Setup" (expert module:
 * fc1 -> SiLU -> dropout -> fc2, both nn.Linear) and "Architecture Overview"
 * (non-gated MLP with Swish, d_e << d_h).  Inference: dropout is the identity.
 * nn.Linear carries a bias by default; the biases are optional here (NULL = the
 * expert is W_out_e Swish(W_in_e x), the form the layer's sparse computation is
 * stated in):
 *   h[j] = silu( sum_k W_in[e,j,k] x[k] + b_in[e,j] ),
 *   o[i] = sum_j W_out[e,i,j] h[j] + b_out[e,i]
 */
static void expert_apply(const double* xt, const double* W_in, const double* W_out,
                         const double* b_in, const double* b_out,
                         int d_h, int d_e, int e, double* h, double* o)
{
    const double* Wi = W_in + (size_t)e * d_e * d_h;
    const double* Wo = W_out + (size_t)e * d_h * d_e;
    for (int j = 0; j < d_e; ++j) {
        double s = 0.0;
        for (int k = 0; k < d_h; ++k) s += Wi[(size_t)j * d_h + k] * xt[k];
        if (b_in) s += b_in[(size_t)e * d_e + j];
        h[j] = silu(s);
    }
    for (int i = 0; i < d_h; ++i) {
        double s = 0.0;
        for (int j = 0; j < d_e; ++j) s += Wo[(size_t)i * d_e + j] * h[j];
        if (b_out) s += b_out[(size_t)e * d_h + i];
        o[i] = s;
    }
}

/*
 * Dense layer output, the definition.  [SKILL] "Full BlockFFN Layer with
 * Combined Losses" (BlockFFNLayer.forward): every expert is applied to every
 * token, each output is multiplied by that token's gate, and the products are
 * summed over the experts.  The gate is g = RMSNorm(ReLU(W_r x)) ([ABS]), not the
 * sigmoid training probabilities; the LayerNorm + residual that follows the sum
 * on that page is outside the FFN output y.  The gate multiplies the whole
 * expert output, its fc2 bias included.
 *
 *   y[t,:] = sum_{e=0}^{E-1} gates[t,e] * ( W_out_e Swish(W_in_e x_t + b_in_e) + b_out_e )
 */
void oracle_forward_dense(const double* x, const double* gates, const double* W_in,
                          const double* W_out, const double* b_in, const double* b_out,
                          int T, int d_h, int E, int d_e, double* y)
{
    int t;
#pragma omp parallel for schedule(dynamic, 1)
    for (t = 0; t < T; ++t) {
        double* h = (double*)malloc(sizeof(double) * (size_t)d_e);
        double* o = (double*)malloc(sizeof(double) * (size_t)d_h);
        double* yt = y + (size_t)t * d_h;
        for (int i = 0; i < d_h; ++i) yt[i] = 0.0;
        for (int e = 0; e < E; ++e) {
            double g = gates[(size_t)t * E + e];
            expert_apply(x + (size_t)t * d_h, W_in, W_out, b_in, b_out, d_h, d_e, e, h, o);
            for (int i = 0; i < d_h; ++i) yt[i] += g * o[i];
        }
        free(h);
        free(o);
    }
}

/*
 * The method's own schedule: chunk union, then mask after computing.  [SKILL]
 * "Core Concept": compute the union of the experts activated across the n
 * tokens, run each of them on all n tokens, and mask the activations that were
 * not needed after the computation.  For every chunk c and every e in U_c
 * (ascending) the expert runs on every token of the chunk; a token keeps the
 * gated output only where its own bit in tmask[c,e] is set:
 *
 *   y[t,:] = sum_{e in U_c, ascending} ( bit_t(tmask[c,e]) ? gates[t,e] * o_e(x_t) : 0 )
 *
 * with o_e the expert's output as above (its biases included when given).
 * Masked terms are selected to exactly zero.  Same summation order as the dense
 * definition restricted to the active experts.
 */
void oracle_forward_chunk_union(const double* x, const double* gates, const double* W_in,
                                const double* W_out, const double* b_in, const double* b_out,
                                int T, int d_h, int E, int d_e, int n, double* y)
{
    int C = (T + n - 1) / n;
    int32_t* counts = (int32_t*)malloc(sizeof(int32_t) * (size_t)C);
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)C * E);
    uint32_t* tmask = (uint32_t*)malloc(sizeof(uint32_t) * (size_t)C * E);
    oracle_chunk_union(gates, T, E, n, counts, idx, tmask);
    memset(y, 0, sizeof(double) * (size_t)T * d_h);
    int t;
#pragma omp parallel for schedule(dynamic, 1)
    for (t = 0; t < T; ++t) {
        int c = t / n, j = t % n;
        double* h = (double*)malloc(sizeof(double) * (size_t)d_e);
        double* o = (double*)malloc(sizeof(double) * (size_t)d_h);
        for (int s = 0; s < counts[c]; ++s) {
            int e = idx[(size_t)c * E + s];
            uint32_t bits = tmask[(size_t)c * E + e];
            expert_apply(x + (size_t)t * d_h, W_in, W_out, b_in, b_out, d_h, d_e, e, h, o);
            int keep = (int)((bits >> j) & 1u);
            double g = gates[(size_t)t * E + e];
            for (int i = 0; i < d_h; ++i)
                y[(size_t)t * d_h + i] += keep ? g * o[i] : 0.0;
        }
        free(h);
        free(o);
    }
    free(counts);
    free(idx);
    free(tmask);
}

/*
 * Sparsity statistics, [ABS] (TLS and 8-token CLS) and [SKILL] "Key
 * Hyperparameters" (token-level and chunk-level sparsity targets).
 *   TLS     = fraction of (token, expert) pairs whose gate is zero.
 *   CLS_L   = fraction of (L-token chunk, expert) pairs in which the expert is
 *             inactive on every token of the chunk; chunks as in the union above,
 *             the last one possibly short.  ([SKILL] "Chunk Sparsification Loss":
 *             the expert is active in a chunk with probability 1 - prod_k(1 - p_k);
 *             with 0/1 activations that is the OR over the chunk.)
 * out[0] = TLS, out[1] = CLS_L.
 */
void oracle_sparsity(const double* gates, int T, int E, int L, double* out)
{
    long long zero = 0, inactive = 0;
    int C = (T + L - 1) / L;
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e)
            if (gates[(size_t)t * E + e] == 0.0) ++zero;
    for (int c = 0; c < C; ++c)
        for (int e = 0; e < E; ++e) {
            int any = 0;
            for (int j = 0; j < L && c * L + j < T; ++j)
                if (gates[(size_t)(c * L + j) * E + e] != 0.0) any = 1;
            if (!any) ++inactive;
        }
    out[0] = (double)zero / ((double)T * E);
    out[1] = (double)inactive / ((double)C * E);
}

/*
 * Residual and LayerNorm after the layer.  [SKILL] "Full BlockFFN Layer with
 * Combined Losses": the layer's output is its expert sum plus its input, put
 * through a LayerNorm over the hidden dimension (nn.LayerNorm(hidden_dim): a
 * learnable per-feature scale and shift, population variance).
 *
 *   v[t,k]   = y[t,k] + x[t,k]
 *   mu[t]    = (1/d_h) sum_k v[t,k]
 *   var[t]   = (1/d_h) sum_k (v[t,k] - mu[t])^2
 *   out[t,k] = ln_gamma[k] * (v[t,k] - mu[t]) / sqrt(var[t] + eps) + ln_beta[k]
 *
 * Reading: eps is an argument (nn.LayerNorm's default is 1e-5); the variance is
 * taken around the mean in a second pass.
 */
void oracle_residual_layernorm(const double* y, const double* x, const double* ln_gamma,
                               const double* ln_beta, double eps, int T, int d_h, double* out)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        const double* yr = y + (size_t)t * d_h;
        const double* xr = x + (size_t)t * d_h;
        double* o = out + (size_t)t * d_h;
        double mu = 0.0;
        for (int k = 0; k < d_h; ++k) mu += yr[k] + xr[k];
        mu /= (double)d_h;
        double var = 0.0;
        for (int k = 0; k < d_h; ++k) {
            const double dv = (yr[k] + xr[k]) - mu;
            var += dv * dv;
        }
        var /= (double)d_h;
        const double rstd = 1.0 / sqrt(var + eps);
        for (int k = 0; k < d_h; ++k) o[k] = ln_gamma[k] * ((yr[k] + xr[k]) - mu) * rstd + ln_beta[k];
    }
}
