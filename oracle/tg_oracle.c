/*
 * TokenGate gated-prefill hot path -- plain CPU oracle (test infrastructure).
 *
 * This file is the slow, obviously-correct definition that the CUDA kernels are
 * checked against.  It is test infrastructure only: the tests, the smoke check
 * and the bench's CPU-baseline leg may call it; the product path never does.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * Every floating-point step is carried out in double precision from the same
 * stored input values the GPU receives (bf16 inputs arrive here widened to
 * float, which is exact).  Loops follow the definitions literally: no tiling,
 * no fusion, no reordering beyond what the definition states.
 *
 * Method (TokenGate, "Adapting LLMs for Fast and Memory-Efficient Prefill with
 * Learned Token Pruning"; abstract page and the news write-ups' "how it works"
 * sections):
 *   1. At gate layer L a small MLP scores every token from its post-attention
 *      residual                                   -> tgo_gate_score
 *   2. A top-K selector keeps the K highest-scoring document tokens; question
 *      tokens are never pruned                    -> tgo_topk_select
 *      (random-K ablation: caller-drawn keys)    -> tgo_select_by_keys
 *   3. Layers above L see only the kept tokens; no KV exists for dropped ones
 *                                                 -> tgo_compact_gather
 *   4. Token-gated attention: each kept token's score is added, scaled by a
 *      per-head learned gain, as a bias on the attention logits above the gate,
 *      and a per-head learned temperature divides q.k  -> tgo_gated_attention
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - bias_hj = g_h * log(sigmoid(z_j)) for kept document keys, 0 for question
 *     keys; logits = q.k / (sqrt(d_h) * tau_h) + bias (tau does not divide the bias)
 *   - gate MLP: z = w2 . GELU(W1 h + b1) + b2 with the exact erf GELU, no norm
 *   - top-K total order: larger score first, equal scores (+0 == -0) by lower
 *     index, NaN below every number; K counts document tokens only
 *   - kept tokens stay in ascending original order; RoPE uses original
 *     positions within the prompt (rotate-half pairing, angle pos*theta^(-2i/d))
 *
 * Parity pins: see tests/test_oracle_*.py (brute-force top-K, closed forms,
 * library reductions).  Nothing here is "parity unpinned" except the link to
 * TokenGate's released weights, which the pages do not print.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int tgo_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* GELU with the exact Gaussian CDF: u = a * Phi(a) = a/2 * (1 + erf(a/sqrt(2))). */
static double gelu_exact(double a) { return 0.5 * a * (1.0 + erf(a / sqrt(2.0))); }

/*
 * Gate MLP score (pages: "at layer L a small MLP scores each token from its
 * post-attention residual").
 *   h  [n, d]       residual rows (row-major)
 *   W1 [dg, d]      first layer weight, b1 [dg]
 *   w2 [dg], b2     second layer (one output)
 *   rows            list of n_rows row ids to score, or NULL for all n rows
 *   z_out           [n_rows] (or [n]) scores in double
 */
int tgo_gate_score(const float* h, int64_t n, int32_t d, const float* W1, const float* b1,
                   int32_t dg, const float* w2, double b2, const int64_t* rows, int64_t n_rows,
                   double* z_out) {
    if (!h || !W1 || !b1 || !w2 || !z_out || n < 0 || d <= 0 || dg <= 0) return 1;
    int64_t count = rows ? n_rows : n;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < count; ++t) {
        int64_t j = rows ? rows[t] : t;
        const float* hj = h + j * (int64_t)d;
        double z = b2;
        for (int32_t u = 0; u < dg; ++u) {
            double a = b1[u];
            const float* wu = W1 + (int64_t)u * d;
            for (int32_t c = 0; c < d; ++c) a += (double)wu[c] * (double)hj[c];
            z += (double)w2[u] * gelu_exact(a);
        }
        z_out[t] = z;
    }
    return 0;
}

/* ---- top-K ---------------------------------------------------------------- */

typedef struct {
    float z;
    int32_t idx;
} scored_token;

/*
 * Total order used for selection: a ranks before b when a's score is larger;
 * +0.0 and -0.0 are the same score; equal scores rank by lower index; NaN ranks
 * after every number (and NaNs among themselves by index).
 */
static int rank_before(const scored_token* a, const scored_token* b) {
    int a_nan = isnan(a->z), b_nan = isnan(b->z);
    if (a_nan || b_nan) {
        if (a_nan && b_nan) return a->idx < b->idx;
        return b_nan; /* the number ranks first */
    }
    if (a->z > b->z) return 1;
    if (a->z < b->z) return 0;
    return a->idx < b->idx;
}

static int cmp_rank(const void* pa, const void* pb) {
    const scored_token* a = (const scored_token*)pa;
    const scored_token* b = (const scored_token*)pb;
    if (rank_before(a, b)) return -1;
    if (rank_before(b, a)) return 1;
    return 0;
}

static int cmp_int32(const void* pa, const void* pb) {
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a > b) - (a < b);
}

/*
 * Top-K over each prompt's document span, question protected (pages: "a top-K
 * selector keeps the highest-scoring tokens ... only the document part of the
 * prompt is pruned, the question is never touched"; the user budget is
 * max_kept_prefill_tokens).
 *   z            [total] fp32 scores (selection is decided in fp32)
 *   cu_seqlens   [B+1] prompt offsets
 *   doc_begin/doc_end [B] document span relative to each prompt's start
 *   budget       [B] document tokens to keep (K >= n_doc keeps the whole document)
 *   kept_idx     [sum M_b] global row ids, ascending within each prompt
 *   cu_kept      [B+1] offsets of each prompt's kept rows
 * Returns 0, or 1 on invalid arguments.
 */
int tgo_topk_select(const float* z, int32_t B, const int32_t* cu_seqlens, const int32_t* doc_begin,
                    const int32_t* doc_end, const int32_t* budget, int32_t* kept_idx,
                    int32_t* cu_kept) {
    if (!z || !cu_seqlens || !doc_begin || !doc_end || !budget || !cu_kept || B < 0) return 1;
    cu_kept[0] = 0;
    for (int32_t b = 0; b < B; ++b) {
        int32_t start = cu_seqlens[b];
        int32_t n = cu_seqlens[b + 1] - start;
        int32_t s = doc_begin[b], e = doc_end[b], K = budget[b];
        if (n < 0 || s < 0 || e < s || e > n || K < 0) return 1;
        int32_t n_doc = e - s;
        int32_t k_keep = K < n_doc ? K : n_doc;

        scored_token* doc = (scored_token*)malloc(sizeof(scored_token) * (n_doc > 0 ? n_doc : 1));
        int32_t* kept = (int32_t*)malloc(sizeof(int32_t) * (n > 0 ? n : 1));
        for (int32_t i = 0; i < n_doc; ++i) {
            doc[i].idx = s + i;
            doc[i].z = z[start + s + i];
        }
        qsort(doc, (size_t)n_doc, sizeof(scored_token), cmp_rank);

        int32_t m = 0;
        for (int32_t i = 0; i < k_keep; ++i) kept[m++] = doc[i].idx;       /* top-K of the document */
        for (int32_t p = 0; p < s; ++p) kept[m++] = p;                     /* protected before the span */
        for (int32_t p = e; p < n; ++p) kept[m++] = p;                     /* protected after the span */
        qsort(kept, (size_t)m, sizeof(int32_t), cmp_int32);                /* keep original order */

        for (int32_t i = 0; i < m; ++i) kept_idx[cu_kept[b] + i] = start + kept[i];
        cu_kept[b + 1] = cu_kept[b] + m;
        free(doc);
        free(kept);
    }
    return 0;
}

/*
 * Random-K selection (pages: the random-K selector ablation, a selector that
 * keeps K document tokens at random instead of by gate score).  The random
 * numbers are the caller's: one uint32 key per token; the K document tokens
 * with the largest keys are kept (equal keys: lower index first), with the
 * question protected and the kept rows in ascending order, exactly as in
 * tgo_topk_select.  With i.i.d. uniform keys every K-subset of the document is
 * equally likely.
 */
typedef struct {
    int32_t idx;
    uint32_t key;
} keyed_token;

static int cmp_key_rank(const void* pa, const void* pb) {
    const keyed_token* a = (const keyed_token*)pa;
    const keyed_token* b = (const keyed_token*)pb;
    if (a->key != b->key) return a->key > b->key ? -1 : 1;
    return (a->idx > b->idx) - (a->idx < b->idx);
}

int tgo_select_by_keys(const uint32_t* keys, int32_t B, const int32_t* cu_seqlens,
                       const int32_t* doc_begin, const int32_t* doc_end, const int32_t* budget,
                       int32_t* kept_idx, int32_t* cu_kept) {
    if (!keys || !cu_seqlens || !doc_begin || !doc_end || !budget || !cu_kept || B < 0) return 1;
    cu_kept[0] = 0;
    for (int32_t b = 0; b < B; ++b) {
        int32_t start = cu_seqlens[b];
        int32_t n = cu_seqlens[b + 1] - start;
        int32_t s = doc_begin[b], e = doc_end[b], K = budget[b];
        if (n < 0 || s < 0 || e < s || e > n || K < 0) return 1;
        int32_t n_doc = e - s;
        int32_t k_keep = K < n_doc ? K : n_doc;

        keyed_token* doc = (keyed_token*)malloc(sizeof(keyed_token) * (n_doc > 0 ? n_doc : 1));
        int32_t* kept = (int32_t*)malloc(sizeof(int32_t) * (n > 0 ? n : 1));
        for (int32_t i = 0; i < n_doc; ++i) {
            doc[i].idx = s + i;
            doc[i].key = keys[start + s + i];
        }
        qsort(doc, (size_t)n_doc, sizeof(keyed_token), cmp_key_rank);

        int32_t m = 0;
        for (int32_t i = 0; i < k_keep; ++i) kept[m++] = doc[i].idx;
        for (int32_t p = 0; p < s; ++p) kept[m++] = p;
        for (int32_t p = e; p < n; ++p) kept[m++] = p;
        qsort(kept, (size_t)m, sizeof(int32_t), cmp_int32);

        for (int32_t i = 0; i < m; ++i) kept_idx[cu_kept[b] + i] = start + kept[i];
        cu_kept[b + 1] = cu_kept[b] + m;
        free(doc);
        free(kept);
    }
    return 0;
}

/* ---- compaction + RoPE + log-sigmoid ------------------------------------- */

/* log(sigmoid(x)) = -log(1 + exp(-x)), written to stay finite for large |x|. */
static double log_sigmoid(double x) { return (x < 0.0 ? x : 0.0) - log1p(exp(-fabs(x))); }

/*
 * Rotary embedding of one head vector x[dh] at position pos (rotate-half
 * pairing: element i pairs with i + dh/2, angle pos * theta^(-2i/dh)).
 */
static void rope_head(const float* x, int32_t dh, double pos, double theta, double* out) {
    int32_t half = dh / 2;
    for (int32_t i = 0; i < half; ++i) {
        double ang = pos * pow(theta, -2.0 * (double)i / (double)dh);
        double c = cos(ang), s = sin(ang);
        double x0 = x[i], x1 = x[i + half];
        out[i] = x0 * c - x1 * s;
        out[i + half] = x1 * c + x0 * s;
    }
}

/*
 * Compaction of the kept rows (pages: "layers above L process only the kept
 * tokens and create no KV entry for the others") plus the per-key bias term.
 *   kept_idx [M] global row ids; cu_seqlens/doc_begin/doc_end describe prompts
 *   src      [total, width] source rows
 *   rope_heads: 0 = plain copy, else the row holds rope_heads heads of dh that
 *               are rotated at their original in-prompt position
 *   dst      [M, width] double
 */
int tgo_gather_rows(const int32_t* kept_idx, int64_t M, int32_t B, const int32_t* cu_seqlens,
                    const float* src, int32_t width, int32_t rope_heads, int32_t dh, double theta,
                    double* dst) {
    if (!kept_idx || !cu_seqlens || !src || !dst || M < 0 || width <= 0) return 1;
    if (rope_heads > 0 && (dh <= 0 || dh % 2 != 0 || rope_heads * dh > width)) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M; ++i) {
        int32_t row = kept_idx[i];
        int32_t b = 0;
        while (b + 1 < B && cu_seqlens[b + 1] <= row) ++b;
        double pos = (double)(row - cu_seqlens[b]);
        const float* x = src + (int64_t)row * width;
        double* y = dst + i * (int64_t)width;
        for (int32_t c = 0; c < width; ++c) y[c] = x[c];
        for (int32_t hh = 0; hh < rope_heads; ++hh) rope_head(x + hh * dh, dh, pos, theta, y + hh * dh);
    }
    return 0;
}

/*
 * Per-key bias term l_i = log sigmoid(z[kept_i]) for document tokens, 0 for
 * protected (question) tokens.
 */
int tgo_logsig(const int32_t* kept_idx, int64_t M, int32_t B, const int32_t* cu_seqlens,
               const int32_t* doc_begin, const int32_t* doc_end, const float* z, double* out) {
    if (!kept_idx || !cu_seqlens || !doc_begin || !doc_end || !z || !out) return 1;
    for (int64_t i = 0; i < M; ++i) {
        int32_t row = kept_idx[i];
        int32_t b = 0;
        while (b + 1 < B && cu_seqlens[b + 1] <= row) ++b;
        int32_t pos = row - cu_seqlens[b];
        int is_doc = pos >= doc_begin[b] && pos < doc_end[b];
        out[i] = is_doc ? log_sigmoid((double)z[row]) : 0.0;
    }
    return 0;
}

/* ---- token-gated causal GQA attention ------------------------------------ */

/*
 * For every listed query row i (global kept row) and query head h:
 *   logit_j = (q_i . k_j) / (sqrt(dh) * tau_h) + g_h * l_j,  j = prompt start .. i
 *   o_i     = sum_j softmax_j(logit) v_j,  lse_i = log sum_j exp(logit_j)
 * with kv head = h / (Hq / Hkv).  (Pages: the kept tokens' scores become a bias
 * on the attention logits above the gate, with a per-head learned gain, and a
 * per-head learned temperature compensates for each query seeing fewer keys.)
 *   q [M, Hq, dh], k/v [M, Hkv, dh]; logsig [M] or NULL (no bias)
 *   rows [n_rows] query rows, or NULL for all M
 *   out [count, Hq, dh] double; lse [count, Hq] double (may be NULL)
 */
int tgo_gated_attention(const float* q, const float* k, const float* v, int32_t B,
                        const int32_t* cu_kept, int32_t Hq, int32_t Hkv, int32_t dh,
                        const float* logsig, const float* gain, const float* temp,
                        const int64_t* rows, int64_t n_rows, double* out, double* lse) {
    if (!q || !k || !v || !cu_kept || !gain || !temp || !out) return 1;
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || dh <= 0) return 1;
    int64_t M = cu_kept[B];
    int64_t count = rows ? n_rows : M;
    int32_t group = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < count; ++t) {
        int64_t i = rows ? rows[t] : t;
        int32_t b = 0;
        while (b + 1 < B && cu_kept[b + 1] <= i) ++b;
        int64_t j0 = cu_kept[b];
        int64_t nk = i - j0 + 1;
        double* logit = (double*)malloc(sizeof(double) * (size_t)nk);
        for (int32_t h = 0; h < Hq; ++h) {
            int32_t hk = h / group;
            const float* qi = q + (i * Hq + h) * (int64_t)dh;
            double scale = 1.0 / (sqrt((double)dh) * (double)temp[h]);
            double mx = -INFINITY;
            for (int64_t j = j0; j <= i; ++j) {
                const float* kj = k + (j * Hkv + hk) * (int64_t)dh;
                double dot = 0.0;
                for (int32_t c = 0; c < dh; ++c) dot += (double)qi[c] * (double)kj[c];
                double lg = dot * scale + (logsig ? (double)gain[h] * (double)logsig[j] : 0.0);
                logit[j - j0] = lg;
                if (lg > mx) mx = lg;
            }
            double denom = 0.0;
            double* o = out + (t * Hq + h) * (int64_t)dh;
            for (int32_t c = 0; c < dh; ++c) o[c] = 0.0;
            for (int64_t j = j0; j <= i; ++j) {
                double p = exp(logit[j - j0] - mx);
                denom += p;
                const float* vj = v + (j * Hkv + hk) * (int64_t)dh;
                for (int32_t c = 0; c < dh; ++c) o[c] += p * (double)vj[c];
            }
            for (int32_t c = 0; c < dh; ++c) o[c] /= denom;
            if (lse) lse[t * Hq + h] = mx + log(denom);
        }
        free(logit);
    }
    return 0;
}

/* ---- backward of the gated attention --------------------------------------
 *
 * The gate is trained through the attention bias (pages: the gate's scores
 * enter the attention logits above the gate as a bias, the "MoE router trick",
 * which is what carries a gradient back to the scorer).  For a scalar loss
 * L = sum over rows i, heads h, dims c of dout[i,h,c] * out[i,h,c] these
 * functions give L itself and its exact gradient with respect to the kept
 * rows' log-gates l_j, the per-head gains g_h and temperatures tau_h, all in
 * fp64 from double parameters (so that finite differences can check them).
 *
 * Per prompt, head h and query row i (keys j <= i of the same prompt):
 *   logit_ij = (q_i . k_j) / (sqrt(d_h) tau_h) + g_h l_j,  P_ij = softmax_j(logit_ij)
 *   dP_ij = dout_i . v_j,   D_i = sum_j P_ij dP_ij,   dlogit_ij = P_ij (dP_ij - D_i)
 *   dL/dl_j  += g_h dlogit_ij
 *   dL/dg_h  += l_j dlogit_ij
 *   dL/dtau_h += dlogit_ij * (-(q_i . k_j) / (sqrt(d_h) tau_h^2))
 * (the derivative of the softmax-weighted sum out_i = sum_j P_ij v_j through
 * the logits; D_i equals dout_i . out_i).
 */
static void attn_row_f64(const float* q, const float* k, int64_t i, int64_t j0,
                         int32_t h, int32_t hk, int32_t Hq, int32_t Hkv, int32_t dh,
                         const double* logsig, const double* gain, const double* temp,
                         double* s, double* P) {
    const float* qi = q + (i * Hq + h) * (int64_t)dh;
    double scale = 1.0 / (sqrt((double)dh) * temp[h]);
    double mx = -INFINITY;
    for (int64_t j = j0; j <= i; ++j) {
        const float* kj = k + (j * Hkv + hk) * (int64_t)dh;
        double dot = 0.0;
        for (int32_t c = 0; c < dh; ++c) dot += (double)qi[c] * (double)kj[c];
        s[j - j0] = dot;
        double lg = dot * scale + gain[h] * logsig[j];
        P[j - j0] = lg;
        if (lg > mx) mx = lg;
    }
    double denom = 0.0;
    for (int64_t j = j0; j <= i; ++j) {
        P[j - j0] = exp(P[j - j0] - mx);
        denom += P[j - j0];
    }
    for (int64_t j = j0; j <= i; ++j) P[j - j0] /= denom;
}

static int32_t prompt_of(const int32_t* cu, int32_t B, int64_t i) {
    int32_t b = 0;
    while (b + 1 < B && cu[b + 1] <= i) ++b;
    return b;
}

int tgo_attention_loss(const float* q, const float* k, const float* v, int32_t B,
                       const int32_t* cu_kept, int32_t Hq, int32_t Hkv, int32_t dh,
                       const double* logsig, const double* gain, const double* temp,
                       const float* dout, double* loss_out) {
    if (!q || !k || !v || !cu_kept || !logsig || !gain || !temp || !dout || !loss_out) return 1;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || dh <= 0) return 1;
    int64_t M = cu_kept[B];
    int32_t group = Hq / Hkv;
    double total = 0.0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : total)
    for (int64_t i = 0; i < M; ++i) {
        int64_t j0 = cu_kept[prompt_of(cu_kept, B, i)];
        int64_t nk = i - j0 + 1;
        double* s = (double*)malloc(sizeof(double) * (size_t)nk);
        double* P = (double*)malloc(sizeof(double) * (size_t)nk);
        for (int32_t h = 0; h < Hq; ++h) {
            int32_t hk = h / group;
            attn_row_f64(q, k, i, j0, h, hk, Hq, Hkv, dh, logsig, gain, temp, s, P);
            const float* di = dout + (i * Hq + h) * (int64_t)dh;
            for (int64_t j = j0; j <= i; ++j) {
                const float* vj = v + (j * Hkv + hk) * (int64_t)dh;
                double dp = 0.0;
                for (int32_t c = 0; c < dh; ++c) dp += (double)di[c] * (double)vj[c];
                total += P[j - j0] * dp;
            }
        }
        free(s);
        free(P);
    }
    *loss_out = total;
    return 0;
}

int tgo_gated_attention_backward(const float* q, const float* k, const float* v, int32_t B,
                                 const int32_t* cu_kept, int32_t Hq, int32_t Hkv, int32_t dh,
                                 const double* logsig, const double* gain, const double* temp,
                                 const float* dout, double* d_logsig, double* d_gain,
                                 double* d_temp) {
    if (!q || !k || !v || !cu_kept || !logsig || !gain || !temp || !dout || !d_logsig || !d_gain ||
        !d_temp)
        return 1;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || dh <= 0) return 1;
    int64_t M = cu_kept[B];
    int32_t group = Hq / Hkv;
    for (int64_t j = 0; j < M; ++j) d_logsig[j] = 0.0;
    for (int32_t h = 0; h < Hq; ++h) d_gain[h] = d_temp[h] = 0.0;
#pragma omp parallel
    {
        /* each thread sums into its own buffers; they are added up at the end */
        double* dl = (double*)calloc((size_t)(M > 0 ? M : 1), sizeof(double));
        double* dg = (double*)calloc((size_t)Hq, sizeof(double));
        double* dtau = (double*)calloc((size_t)Hq, sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < M; ++i) {
            int64_t j0 = cu_kept[prompt_of(cu_kept, B, i)];
            int64_t nk = i - j0 + 1;
            double* s = (double*)malloc(sizeof(double) * (size_t)nk);
            double* P = (double*)malloc(sizeof(double) * (size_t)nk);
            double* dP = (double*)malloc(sizeof(double) * (size_t)nk);
            for (int32_t h = 0; h < Hq; ++h) {
                int32_t hk = h / group;
                attn_row_f64(q, k, i, j0, h, hk, Hq, Hkv, dh, logsig, gain, temp, s, P);
                const float* di = dout + (i * Hq + h) * (int64_t)dh;
                double D = 0.0;
                for (int64_t j = j0; j <= i; ++j) {
                    const float* vj = v + (j * Hkv + hk) * (int64_t)dh;
                    double dp = 0.0;
                    for (int32_t c = 0; c < dh; ++c) dp += (double)di[c] * (double)vj[c];
                    dP[j - j0] = dp;
                    D += P[j - j0] * dp;
                }
                double scale = 1.0 / (sqrt((double)dh) * temp[h]);
                for (int64_t j = j0; j <= i; ++j) {
                    double dlogit = P[j - j0] * (dP[j - j0] - D);
                    dl[j] += gain[h] * dlogit;
                    dg[h] += logsig[j] * dlogit;
                    dtau[h] += dlogit * (-s[j - j0] * scale / temp[h]);
                }
            }
            free(s);
            free(P);
            free(dP);
        }
#pragma omp critical
        {
            for (int64_t j = 0; j < M; ++j) d_logsig[j] += dl[j];
            for (int32_t h = 0; h < Hq; ++h) {
                d_gain[h] += dg[h];
                d_temp[h] += dtau[h];
            }
        }
        free(dl);
        free(dg);
        free(dtau);
    }
    return 0;
}
