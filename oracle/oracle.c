/*
 * Plain, slow, obviously-correct CPU oracle for the event-tensor hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant with the CUDA path and includes no CUDA header.
 *
 * Sources (web pages, cited by title and section):
 *   [ETN]  "Event Tensor：用“事件张量”编译动态 Megakernel" (reading notes on
 *          "Event Tensor: A Unified Abstraction for Compiling Dynamic
 *          Megakernel", MLSys 2026)
 *   [ETS]  hyper.ai summary of the same paper (§方法 / method)
 *
 * Floating point: every sum is accumulated in double, in index order.  A
 * value is rounded to fp32 or bf16 only where the method hands a tensor of
 * that type to the next step (xn, h and y are bf16 tensors; router logits
 * and routing weights are fp32 tensors).  bf16 rounding is round-to-nearest-
 * even, written out below from the IEEE definition.
 *
 * Threads: loops whose iterations compute disjoint outputs (tokens, rows,
 * routed pairs) may run on several OpenMP threads (orc_set_threads).  Each
 * output is still computed by one thread with the same sums in the same
 * order, so every result is bit-identical for any thread count.
 *
 * Parity status of each entry point is stated in its comment.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- bf16 -- */

/* IEEE binary32 -> bfloat16 (upper 16 bits), round to nearest, ties to even.
 * Inputs here are finite; NaN is kept quiet by forcing a mantissa bit. */
static uint16_t orc_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x40u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

static float orc_bf16_to_f32(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* double -> bf16: first to the nearest fp32 (the value the GPU holds in a
 * register), then RNE to bf16.  Double rounding is the GPU's own path. */
static uint16_t orc_d_to_bf16(double d) { return orc_f32_to_bf16((float)d); }

uint16_t orc_bf16_round_bits(float f) { return orc_f32_to_bf16(f); }

/* Number of OpenMP threads used by the parallel loops below (default 1). */
static int orc_threads = 1;
void orc_set_threads(int n) { orc_threads = n > 0 ? n : 1; }
int orc_get_threads(void) { return orc_threads; }
int orc_max_threads(void) { return omp_get_num_procs(); }
float orc_bf16_value(uint16_t h) { return orc_bf16_to_f32(h); }

/* ------------------------------------------------------------- split-K -- */

/* [ETN] §Split-K reduction 示例 (two-stage reduction):
 *   B[i,j] = sum_{k=chunk*j}^{chunk*j+chunk-1} A[i,k]
 *   C[i]   = sum_j B[i,j]
 * A is fp32 [rows, cols], row-major.  B is [rows, nchunk] with
 * nchunk = ceil(cols/chunk) (the last chunk may be short), C is [rows].
 * Parity pin: C[i] equals the full row sum of A (closed form). */
void orc_splitk(const float* A, int rows, int cols, int chunk, double* B, double* C) {
    int nchunk = (cols + chunk - 1) / chunk;
    for (int i = 0; i < rows; ++i) {
        double c = 0.0;
        for (int j = 0; j < nchunk; ++j) {
            double b = 0.0;
            int k0 = j * chunk, k1 = k0 + chunk;
            if (k1 > cols) k1 = cols;
            for (int k = k0; k < k1; ++k) b += (double)A[(size_t)i * cols + k];
            B[(size_t)i * nchunk + j] = b;
            c += b;
        }
        C[i] = c;
    }
}

/* ------------------------------------------------------------- RMSNorm -- */

/* RMSNorm of the decode pipeline ([ETN] §端到端低 batch serving lists Norm
 * among the fused operators; the formula is the standard one):
 *   xn[r,:] = bf16( x[r,:] / sqrt(mean(x[r,:]^2) + eps) * gamma )
 * x, gamma, xn are bf16 bit patterns. */
void orc_rmsnorm(const uint16_t* X, const uint16_t* gamma, int rows, int hidden, double eps,
                 uint16_t* xn) {
    for (int r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int k = 0; k < hidden; ++k) {
            double v = orc_bf16_to_f32(X[(size_t)r * hidden + k]);
            ss += v * v;
        }
        double inv = 1.0 / sqrt(ss / (double)hidden + eps);
        for (int k = 0; k < hidden; ++k) {
            double v = orc_bf16_to_f32(X[(size_t)r * hidden + k]);
            double g = orc_bf16_to_f32(gamma[k]);
            xn[(size_t)r * hidden + k] = orc_d_to_bf16(v * inv * g);
        }
    }
}

static double orc_silu(double g) { return g / (1.0 + exp(-g)); }

/* One row through a SwiGLU block:
 *   g = x . Wg^T, u = x . Wu^T (double accumulation, index order)
 *   h = bf16( silu(g) * u )
 * W is [2*inter, hidden]: gate rows 0..inter-1, then up rows. */
static void orc_swiglu_row(const uint16_t* x, const uint16_t* W, int hidden, int inter,
                           uint16_t* h) {
    for (int n = 0; n < inter; ++n) {
        const uint16_t* wg = W + (size_t)n * hidden;
        const uint16_t* wu = W + (size_t)(inter + n) * hidden;
        double g = 0.0, u = 0.0;
        for (int k = 0; k < hidden; ++k) {
            double xv = orc_bf16_to_f32(x[k]);
            g += xv * (double)orc_bf16_to_f32(wg[k]);
            u += xv * (double)orc_bf16_to_f32(wu[k]);
        }
        h[n] = orc_d_to_bf16(orc_silu(g) * u);
    }
}

/* o[n] = sum_k h[k] * Wd[n,k], Wd [out, in] (double accumulation). */
static void orc_linear_row(const uint16_t* h, const uint16_t* W, int in, int out, double* o) {
    for (int n = 0; n < out; ++n) {
        const uint16_t* w = W + (size_t)n * in;
        double acc = 0.0;
        for (int k = 0; k < in; ++k) acc += (double)orc_bf16_to_f32(h[k]) * (double)orc_bf16_to_f32(w[k]);
        o[n] = acc;
    }
}

/* Fused decode MLP: RMSNorm -> gate/up -> SiLU*mul -> down.
 *   y = bf16( h . Wd^T ),  h as in orc_swiglu_row on xn = rmsnorm(x).
 * xn_out [B,hidden] and h_out [B,inter] are optional (NULL to skip). */
void orc_mlp(const uint16_t* X, const uint16_t* gamma, const uint16_t* Wgu, const uint16_t* Wd,
             int B, int hidden, int inter, double eps, uint16_t* Y, uint16_t* xn_out,
             uint16_t* h_out) {
    uint16_t* xn = (uint16_t*)malloc((size_t)B * hidden * 2);
    uint16_t* h = (uint16_t*)malloc((size_t)inter * 2);
    double* o = (double*)malloc((size_t)hidden * sizeof(double));
    orc_rmsnorm(X, gamma, B, hidden, eps, xn);
    for (int r = 0; r < B; ++r) {
        orc_swiglu_row(xn + (size_t)r * hidden, Wgu, hidden, inter, h);
        if (h_out) memcpy(h_out + (size_t)r * inter, h, (size_t)inter * 2);
        orc_linear_row(h, Wd, inter, hidden, o);
        for (int n = 0; n < hidden; ++n) Y[(size_t)r * hidden + n] = orc_d_to_bf16(o[n]);
    }
    if (xn_out) memcpy(xn_out, xn, (size_t)B * hidden * 2);
    free(xn);
    free(h);
    free(o);
}

/* ----------------------------------------------------------------- MoE -- */

/* Router logits: l[t,e] = sum_k x[t,k] * Wr[e,k] + bias[e], double
 * accumulation, rounded to fp32 (the logits tensor is fp32). */
void orc_router_logits(const uint16_t* X, const uint16_t* Wr, const float* bias, int T, int hidden,
                       int E, float* logits) {
#pragma omp parallel for num_threads(orc_threads) schedule(dynamic, 1) if (T > 1)
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int k = 0; k < hidden; ++k)
                acc += (double)orc_bf16_to_f32(X[(size_t)t * hidden + k]) *
                       (double)orc_bf16_to_f32(Wr[(size_t)e * hidden + k]);
            logits[(size_t)t * E + e] = (float)(acc + (double)bias[e]);
        }
}

/* Top-k routing ([ETN] §Data-dependent event update: topk[i,:] is the
 * runtime tensor that picks a token's experts).  Selection order: larger
 * fp32 logit first, equal logits -> lower expert index first (a strict
 * total order, so the result is unique).  Weights: softmax over the k
 * selected logits, max-subtracted, in double, rounded to fp32.
 * Written as k passes of "take the best remaining", the definition. */
void orc_topk_softmax(const float* logits, int T, int E, int k, int32_t* idx, float* w) {
    char* taken = (char*)malloc((size_t)E);
    double* ex = (double*)malloc((size_t)k * sizeof(double));
    for (int t = 0; t < T; ++t) {
        const float* l = logits + (size_t)t * E;
        memset(taken, 0, (size_t)E);
        for (int s = 0; s < k; ++s) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e; /* ties keep the lower index */
            }
            taken[best] = 1;
            idx[(size_t)t * k + s] = best;
        }
        double m = (double)l[idx[(size_t)t * k]];
        double z = 0.0;
        for (int s = 0; s < k; ++s) {
            ex[s] = exp((double)l[idx[(size_t)t * k + s]] - m);
            z += ex[s];
        }
        for (int s = 0; s < k; ++s) w[(size_t)t * k + s] = (float)(ex[s] / z);
    }
    free(taken);
    free(ex);
}

/* Token grouping ([ETN] §Data-dependent event update and §Data-dependent
 * task triggering):
 *   counts[e]        number of (token, slot) pairs routed to expert e
 *                    (= the initial counter of expert event E[e])
 *   indptr[e]        exclusive prefix of counts (CSR over pairs), E+1 long
 *   perm[p]          pairs grouped by expert, ascending token inside a
 *                    group, encoded t*k + s
 *   task_indptr[e]   exclusive prefix of ceil(counts[e]/bm): the CSR
 *                    range tasks[task_indptr[e] : task_indptr[e+1]]
 *   pos[t*k+s]       inverse of perm (row of pair (t,s) in grouped order)
 * Written as a plain scan over experts, then over tokens in order. */
void orc_group(const int32_t* topk, int T, int k, int E, int bm, int32_t* counts, int32_t* indptr,
               int32_t* perm, int32_t* task_indptr, int32_t* pos) {
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int p = 0; p < T * k; ++p) counts[topk[p]] += 1;
    indptr[0] = 0;
    task_indptr[0] = 0;
    for (int e = 0; e < E; ++e) {
        indptr[e + 1] = indptr[e] + counts[e];
        task_indptr[e + 1] = task_indptr[e] + (counts[e] + bm - 1) / bm;
    }
    int at = 0;
    for (int e = 0; e < E; ++e)
        for (int t = 0; t < T; ++t)
            for (int s = 0; s < k; ++s)
                if (topk[(size_t)t * k + s] == e) {
                    perm[at] = t * k + s;
                    pos[t * k + s] = at;
                    ++at;
                }
}

/* One routed pair through expert e:
 *   h = bf16( silu(x . W1g_e^T) * (x . W1u_e^T) ),  o = h . W2_e^T (double)
 * W1 [E, 2*inter, hidden] (gate rows first), W2 [E, hidden, inter]. */
static void orc_expert(const uint16_t* x, const uint16_t* W1, const uint16_t* W2, int hidden,
                       int inter, int e, uint16_t* h, double* o) {
    orc_swiglu_row(x, W1 + (size_t)e * 2 * inter * hidden, hidden, inter, h);
    orc_linear_row(h, W2 + (size_t)e * hidden * inter, inter, hidden, o);
}

/* MoE layer, grouped evaluation: experts in order, each over its group of
 * pairs (perm order), then the weighted combine per token in slot order:
 *   y[t] = bf16( sum_{s<k} w[t,s] * o[t,s] )  (double sum, slots 0..k-1).
 * topk/w/indptr/perm come from orc_topk_softmax and orc_group.
 * h_out [T*k, inter] in grouped (perm) order is optional.
 * Returns 0, or -1 (and computes nothing) when the grouping is malformed:
 * indptr not a non-decreasing CSR over T*k pairs, a perm entry out of
 * range or listed twice, or a pair listed under an expert its topk entry
 * does not name. */
int orc_moe_grouped(const uint16_t* X, const uint16_t* W1, const uint16_t* W2,
                    const int32_t* topk, const float* w, const int32_t* indptr,
                    const int32_t* perm, int T, int hidden, int inter, int E, int k,
                    uint16_t* Y, uint16_t* h_out) {
    const int P = T * k;
    if (indptr[0] != 0 || indptr[E] != P) return -1;
    int32_t* row_expert = (int32_t*)malloc((size_t)(P > 0 ? P : 1) * sizeof(int32_t));
    char* seen = (char*)calloc((size_t)(P > 0 ? P : 1), 1);
    int bad = 0;
    for (int e = 0; e < E && !bad; ++e) {
        if (indptr[e + 1] < indptr[e]) bad = 1;
        for (int r = indptr[e]; r < indptr[e + 1] && !bad; ++r) {
            int p = perm[r];
            if (p < 0 || p >= P || seen[p] || topk[p] != e) bad = 1;
            else {
                seen[p] = 1;
                row_expert[r] = e;
            }
        }
    }
    free(seen);
    if (bad) {
        free(row_expert);
        return -1;
    }
    double* o_all = (double*)malloc((size_t)(P > 0 ? P : 1) * hidden * sizeof(double));
#pragma omp parallel num_threads(orc_threads) if (P > 1)
    {
        uint16_t* h = (uint16_t*)malloc((size_t)inter * 2);
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < P; ++r) {
            int p = perm[r];
            int t = p / k;
            orc_expert(X + (size_t)t * hidden, W1, W2, hidden, inter, row_expert[r], h,
                       o_all + (size_t)p * hidden);
            if (h_out) memcpy(h_out + (size_t)r * inter, h, (size_t)inter * 2);
        }
        free(h);
    }
    free(row_expert);
    for (int t = 0; t < T; ++t)
        for (int n = 0; n < hidden; ++n) {
            double acc = 0.0;
            for (int s = 0; s < k; ++s)
                acc += (double)w[(size_t)t * k + s] * o_all[((size_t)t * k + s) * hidden + n];
            Y[(size_t)t * hidden + n] = orc_d_to_bf16(acc);
        }
    free(o_all);
    return 0;
}

/* MoE layer, per-token evaluation of the same definition: for each token,
 * route it (logits, top-k, softmax) and run its k experts one by one, then
 * combine.  No grouping at all; used to pin the grouped evaluation.
 * Only the tokens listed in `tokens` (n_tokens of them) are evaluated; row
 * i of Y_rows belongs to tokens[i].  Router outputs for those tokens are
 * written to topk_rows/w_rows when non-NULL. */
void orc_moe_per_token(const uint16_t* X, const uint16_t* Wr, const float* bias,
                       const uint16_t* W1, const uint16_t* W2, const int32_t* tokens,
                       int n_tokens, int hidden, int inter, int E, int k, uint16_t* Y_rows,
                       int32_t* topk_rows, float* w_rows) {
#pragma omp parallel num_threads(orc_threads) if (n_tokens > 1)
    {
    float* l = (float*)malloc((size_t)E * sizeof(float));
    int32_t* idx = (int32_t*)malloc((size_t)k * sizeof(int32_t));
    float* wt = (float*)malloc((size_t)k * sizeof(float));
    uint16_t* h = (uint16_t*)malloc((size_t)inter * 2);
    double* o = (double*)malloc((size_t)k * hidden * sizeof(double));
#pragma omp for schedule(dynamic, 1)
    for (int i = 0; i < n_tokens; ++i) {
        const uint16_t* x = X + (size_t)tokens[i] * hidden;
        orc_router_logits(x, Wr, bias, 1, hidden, E, l);
        orc_topk_softmax(l, 1, E, k, idx, wt);
        for (int s = 0; s < k; ++s) orc_expert(x, W1, W2, hidden, inter, idx[s], h, o + (size_t)s * hidden);
        for (int n = 0; n < hidden; ++n) {
            double acc = 0.0;
            for (int s = 0; s < k; ++s) acc += (double)wt[s] * o[(size_t)s * hidden + n];
            Y_rows[(size_t)i * hidden + n] = orc_d_to_bf16(acc);
        }
        if (topk_rows) memcpy(topk_rows + (size_t)i * k, idx, (size_t)k * sizeof(int32_t));
        if (w_rows) memcpy(w_rows + (size_t)i * k, wt, (size_t)k * sizeof(float));
    }
    free(l);
    free(idx);
    free(wt);
    free(h);
    free(o);
    }
}

/* Same per-token evaluation, but with the routing given (topk, w for each
 * listed token) instead of recomputed: used where a near-tie in the logits
 * lets the device legitimately pick a different 8th expert. */
void orc_moe_rows_given_routing(const uint16_t* X, const uint16_t* W1, const uint16_t* W2,
                                const int32_t* tokens, const int32_t* topk_rows,
                                const float* w_rows, int n_tokens, int hidden, int inter, int k,
                                uint16_t* Y_rows) {
#pragma omp parallel num_threads(orc_threads) if (n_tokens > 1)
    {
    uint16_t* h = (uint16_t*)malloc((size_t)inter * 2);
    double* o = (double*)malloc((size_t)k * hidden * sizeof(double));
#pragma omp for schedule(dynamic, 1)
    for (int i = 0; i < n_tokens; ++i) {
        const uint16_t* x = X + (size_t)tokens[i] * hidden;
        for (int s = 0; s < k; ++s)
            orc_expert(x, W1, W2, hidden, inter, topk_rows[(size_t)i * k + s], h, o + (size_t)s * hidden);
        for (int n = 0; n < hidden; ++n) {
            double acc = 0.0;
            for (int s = 0; s < k; ++s) acc += (double)w_rows[(size_t)i * k + s] * o[(size_t)s * hidden + n];
            Y_rows[(size_t)i * hidden + n] = orc_d_to_bf16(acc);
        }
    }
    free(h);
    free(o);
    }
}

/* MLP rows: the decode MLP evaluated for the listed rows only (sampled
 * checks at full size). */
void orc_mlp_rows(const uint16_t* X, const uint16_t* gamma, const uint16_t* Wgu, const uint16_t* Wd,
                  const int32_t* rows, int n_rows, int hidden, int inter, double eps,
                  uint16_t* Y_rows) {
#pragma omp parallel num_threads(orc_threads) if (n_rows > 1)
    {
        uint16_t* x1 = (uint16_t*)malloc((size_t)hidden * 2);
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < n_rows; ++i) {
            memcpy(x1, X + (size_t)rows[i] * hidden, (size_t)hidden * 2);
            orc_mlp(x1, gamma, Wgu, Wd, 1, hidden, inter, eps, Y_rows + (size_t)i * hidden, NULL, NULL);
        }
        free(x1);
    }
}

/* --------------------------------------------------------- decode layer -- */

/* Rotary position embedding of one head vector at position `pos`
 * (rotate-half pairing: element i is rotated with element i + dim/2 by the
 * angle pos * base^(-2i/dim), i < dim/2).  In place, double precision. */
static void orc_rope(double* v, int dim, int pos, double base) {
    int half = dim / 2;
    for (int i = 0; i < half; ++i) {
        double ang = (double)pos * pow(base, -2.0 * (double)i / (double)dim);
        double c = cos(ang), s = sin(ang);
        double a = v[i], b = v[i + half];
        v[i] = a * c - b * s;
        v[i + half] = b * c + a * s;
    }
}

void orc_rope_bf16(const uint16_t* x, int dim, int pos, double base, uint16_t* out) {
    double* v = (double*)malloc((size_t)dim * sizeof(double));
    for (int i = 0; i < dim; ++i) v[i] = orc_bf16_to_f32(x[i]);
    orc_rope(v, dim, pos, base);
    for (int i = 0; i < dim; ++i) out[i] = orc_d_to_bf16(v[i]);
    free(v);
}

/* One decode step of a transformer layer for B requests, each adding one
 * token ([ETN] §端到端低 batch serving: the decoding pipeline fuses
 * Attention, RoPE, KV-cache, Norm and MLP; the Q branch runs Norm + RoPE,
 * the K branch Norm + RoPE + cache append).  Per request b, at position
 * p = pos[b] (the number of tokens already in its cache):
 *   xn  = bf16(rmsnorm(x) * g1)
 *   qkv = bf16(xn . Wqkv^T)                 rows: n_q query heads, then
 *                                           n_kv key heads, then n_kv value heads
 *   q_h = bf16(rope(rmsnorm(q_h) * gq, p))  every query head (per-head norm)
 *   k_g = bf16(rope(rmsnorm(k_g) * gk, p))  every key head
 *   cache: K[b,g,p] = k_g, V[b,g,p] = v_g   (written in place)
 *   o_h = sum_{j<=p} softmax_j(q_h . K[b,g,j] / sqrt(hd)) V[b,g,j],  g = h / (n_q / n_kv)
 *   a   = bf16(o)                            heads concatenated [n_q * hd]
 *   h1  = bf16(x + a . Wo^T)                 residual, one rounding
 *   y   = bf16(h1 + mlp(h1))                 mlp = the decode MLP above
 *                                           (rmsnorm with g2, SwiGLU, down)
 * Caches are [B, n_kv, max_ctx, hd] bf16.  All sums in double, in index
 * order; softmax max-subtracted.  Optional outputs (NULL to skip): q_out
 * [B, n_q*hd], k_out [B, n_kv*hd], a_out [B, n_q*hd], h1_out [B, hidden].
 * Returns 0, or -1 when a position is outside the cache. */
int orc_decode_layer(const uint16_t* X, const int32_t* pos, int B, int hidden, int n_q, int n_kv,
                     int hd, int inter, const uint16_t* g1, const uint16_t* Wqkv, const uint16_t* gq,
                     const uint16_t* gk, const uint16_t* Wo, const uint16_t* g2,
                     const uint16_t* Wgu, const uint16_t* Wd, uint16_t* Kc, uint16_t* Vc,
                     int max_ctx, double eps, double rope_base, uint16_t* Y, uint16_t* q_out,
                     uint16_t* k_out, uint16_t* a_out, uint16_t* h1_out) {
    for (int b = 0; b < B; ++b)
        if (pos[b] < 0 || pos[b] >= max_ctx) return -1;
    const int nqkv = (n_q + 2 * n_kv) * hd;
    const int group = n_q / n_kv;
    const double scale = 1.0 / sqrt((double)hd);
#pragma omp parallel num_threads(orc_threads) if (B > 1)
    {
        uint16_t* xn = (uint16_t*)malloc((size_t)hidden * 2);
        uint16_t* qkv = (uint16_t*)malloc((size_t)nqkv * 2);
        uint16_t* q = (uint16_t*)malloc((size_t)n_q * hd * 2);
        uint16_t* a = (uint16_t*)malloc((size_t)n_q * hd * 2);
        uint16_t* h1 = (uint16_t*)malloc((size_t)hidden * 2);
        double* o = (double*)malloc((size_t)(hidden > nqkv ? hidden : nqkv) * sizeof(double));
        double* v = (double*)malloc((size_t)hd * sizeof(double));
        double* s = (double*)malloc((size_t)max_ctx * sizeof(double));
        double* acc = (double*)malloc((size_t)hd * sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int b = 0; b < B; ++b) {
            const uint16_t* x = X + (size_t)b * hidden;
            const int p = pos[b];
            orc_rmsnorm(x, g1, 1, hidden, eps, xn);
            orc_linear_row(xn, Wqkv, hidden, nqkv, o);
            for (int i = 0; i < nqkv; ++i) qkv[i] = orc_d_to_bf16(o[i]);
            /* Q branch: per-head norm + rope */
            for (int h = 0; h < n_q; ++h) {
                const uint16_t* qh = qkv + (size_t)h * hd;
                double ss = 0.0;
                for (int i = 0; i < hd; ++i) {
                    double t = orc_bf16_to_f32(qh[i]);
                    ss += t * t;
                }
                double inv = 1.0 / sqrt(ss / (double)hd + eps);
                for (int i = 0; i < hd; ++i) v[i] = orc_bf16_to_f32(qh[i]) * inv * orc_bf16_to_f32(gq[i]);
                orc_rope(v, hd, p, rope_base);
                for (int i = 0; i < hd; ++i) q[(size_t)h * hd + i] = orc_d_to_bf16(v[i]);
            }
            /* K branch: per-head norm + rope + cache append; V appended as is */
            for (int g = 0; g < n_kv; ++g) {
                const uint16_t* kh = qkv + (size_t)(n_q + g) * hd;
                const uint16_t* vh = qkv + (size_t)(n_q + n_kv + g) * hd;
                double ss = 0.0;
                for (int i = 0; i < hd; ++i) {
                    double t = orc_bf16_to_f32(kh[i]);
                    ss += t * t;
                }
                double inv = 1.0 / sqrt(ss / (double)hd + eps);
                for (int i = 0; i < hd; ++i) v[i] = orc_bf16_to_f32(kh[i]) * inv * orc_bf16_to_f32(gk[i]);
                orc_rope(v, hd, p, rope_base);
                uint16_t* kd = Kc + (((size_t)b * n_kv + g) * max_ctx + p) * hd;
                uint16_t* vd = Vc + (((size_t)b * n_kv + g) * max_ctx + p) * hd;
                for (int i = 0; i < hd; ++i) {
                    kd[i] = orc_d_to_bf16(v[i]);
                    vd[i] = vh[i];
                }
                if (k_out) memcpy(k_out + ((size_t)b * n_kv + g) * hd, kd, (size_t)hd * 2);
            }
            /* attention over positions 0..p (the appended token included) */
            for (int h = 0; h < n_q; ++h) {
                const int g = h / group;
                const uint16_t* K = Kc + ((size_t)b * n_kv + g) * max_ctx * hd;
                const uint16_t* V = Vc + ((size_t)b * n_kv + g) * max_ctx * hd;
                const uint16_t* qh = q + (size_t)h * hd;
                double m = -INFINITY;
                for (int j = 0; j <= p; ++j) {
                    double d = 0.0;
                    for (int i = 0; i < hd; ++i)
                        d += (double)orc_bf16_to_f32(qh[i]) * (double)orc_bf16_to_f32(K[(size_t)j * hd + i]);
                    s[j] = d * scale;
                    if (s[j] > m) m = s[j];
                }
                double z = 0.0;
                for (int j = 0; j <= p; ++j) {
                    s[j] = exp(s[j] - m);
                    z += s[j];
                }
                for (int i = 0; i < hd; ++i) acc[i] = 0.0;
                for (int j = 0; j <= p; ++j)
                    for (int i = 0; i < hd; ++i) acc[i] += s[j] * (double)orc_bf16_to_f32(V[(size_t)j * hd + i]);
                for (int i = 0; i < hd; ++i) a[(size_t)h * hd + i] = orc_d_to_bf16(acc[i] / z);
            }
            /* o-proj + residual */
            orc_linear_row(a, Wo, n_q * hd, hidden, o);
            for (int n = 0; n < hidden; ++n) h1[n] = orc_d_to_bf16((double)orc_bf16_to_f32(x[n]) + o[n]);
            /* MLP + residual: y = bf16(h1 + down(silu(gate(xn2)) * up(xn2))), one rounding */
            {
                uint16_t* xn2 = (uint16_t*)malloc((size_t)hidden * 2);
                uint16_t* hm = (uint16_t*)malloc((size_t)inter * 2);
                orc_rmsnorm(h1, g2, 1, hidden, eps, xn2);
                orc_swiglu_row(xn2, Wgu, hidden, inter, hm);
                orc_linear_row(hm, Wd, inter, hidden, o);
                for (int n = 0; n < hidden; ++n)
                    Y[(size_t)b * hidden + n] = orc_d_to_bf16((double)orc_bf16_to_f32(h1[n]) + o[n]);
                free(xn2);
                free(hm);
            }
            if (q_out) memcpy(q_out + (size_t)b * n_q * hd, q, (size_t)n_q * hd * 2);
            if (a_out) memcpy(a_out + (size_t)b * n_q * hd, a, (size_t)n_q * hd * 2);
            if (h1_out) memcpy(h1_out + (size_t)b * hidden, h1, (size_t)hidden * 2);
        }
        free(xn); free(qkv); free(q); free(a); free(h1); free(o); free(v); free(s); free(acc);
    }
    return 0;
}
