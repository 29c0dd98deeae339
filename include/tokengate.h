/*
 * tokengate.h -- C ABI of libtokengate.so, the B200 (sm_100a) gated-prefill hot
 * path of TokenGate ("Adapting LLMs for Fast and Memory-Efficient Prefill with
 * Learned Token Pruning").
 *
 * The method (abstract page; news write-ups, "how it works"): below a gate layer
 * L every token is processed; at layer L a small MLP scores each token from its
 * post-attention residual, a top-K selector keeps the highest-scoring document
 * tokens while the question is never pruned, and the layers above L process only
 * the kept tokens -- no KV entry exists for a dropped token.  To make the
 * selection trainable, each kept token's score enters the attention logits above
 * the gate as a bias (the Mixture-of-Experts router trick) with a per-head
 * learned gain, and a per-head learned temperature corrects for each query
 * seeing fewer keys.  Four calls are that forward pass, one call per step:
 *
 *     tg_gate_score -> tg_topk_select -> tg_compact_gather -> tg_gated_attention
 *
 * Further calls serve the layers around it: budget sweeps and random-K selection,
 * the backward of the gated attention (gradients of the log-gates, gains and
 * temperatures), the element-wise steps of a stack of gated upper layers that
 * emits a compacted KV cache, and a Gated DeltaNet layer over the kept rows.
 *
 * Conventions shared by every call
 *   - Device pointers point to memory on the current CUDA device; "host" arrays
 *     are ordinary host memory read synchronously during the call.
 *   - The caller owns and allocates every buffer.  The library allocates no
 *     device memory, keeps no state between calls and never synchronises the
 *     stream: each call validates its arguments, enqueues kernels on `stream`
 *     and returns.
 *   - A prompt batch is packed row-major ("varlen"): prompt b owns rows
 *     [cu_seqlens[b], cu_seqlens[b+1]) of every per-token tensor.  Each prompt
 *     is [document | question] in any arrangement: doc_begin/doc_end give the
 *     prunable document span relative to the prompt's first row (the `{state}`
 *     span of the reference prompt template); every token outside it is
 *     protected (always kept).  At most TG_MAX_BATCH prompts per call.
 *   - Errors: a call that returns anything but TG_OK has enqueued no work.
 *     TG_ERR_CUDA means a launch failed; tg_last_error_message() describes the
 *     most recent error on the calling host thread.
 *   - Kept rows: with n_doc = doc_end - doc_begin and K = budget, prompt b keeps
 *     M_b = min(K, n_doc) + (N_b - n_doc) rows, in ascending original order.
 */
#ifndef TOKENGATE_H_
#define TOKENGATE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TG_API __attribute__((visibility("default")))
#else
#define TG_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* tg_stream_t; /* same type as cudaStream_t; NULL = legacy default */

typedef enum {
    TG_OK = 0,
    TG_ERR_INVALID_ARG = 1,  /* null pointer, negative size or budget, bad span */
    TG_ERR_SHAPE = 2,        /* inconsistent sizes between arguments */
    TG_ERR_DTYPE = 3,        /* unknown tg_dtype */
    TG_ERR_ALIGNMENT = 4,    /* a pointer or row pitch is not 16-byte aligned */
    TG_ERR_UNSUPPORTED = 5,  /* valid but outside what the kernels implement */
    TG_ERR_CUDA = 6,         /* a CUDA runtime/driver call or launch failed */
    TG_ERR_DEVICE_CHECK = 7, /* a kernel reported a failure (see tg_device_status) */
    TG_ERR_WORKSPACE = 8     /* the workspace given is smaller than the call needs */
} tg_status;

typedef enum { TG_BF16 = 0, TG_FP32 = 1 } tg_dtype;

/* Kernel selection for the two contraction steps. */
typedef enum {
    TG_ALGO_AUTO = 0,    /* tensor-core kernel when the shape allows it, else CUDA cores */
    TG_ALGO_SIMT = 1,    /* CUDA-core (FFMA) kernel; every dtype and shape it accepts */
    TG_ALGO_TCGEN05 = 2  /* tcgen05/TMEM tensor-core kernel; TG_ERR_UNSUPPORTED if the shape
                            or dtype does not allow it (bf16 only) */
} tg_algo;

#define TG_MAX_BATCH 128

/* Human-readable name of a status code (static string). */
TG_API const char* tg_status_string(tg_status status);

/* Description of the most recent failed call on this host thread (static buffer). */
TG_API const char* tg_last_error_message(void);

/* Library version string, e.g. "0.1.0 sm_100a". */
TG_API const char* tg_version(void);

/*
 * Device-side status word: kernels never trap; a bounded wait that gives up
 * (a pipeline barrier that did not complete within ~2 s) sets a bit here and
 * the kernel exits early with its outputs undefined.  Synchronises `stream`,
 * writes the accumulated bits to *bits_out (0 = no failure) and clears them.
 * Returns TG_ERR_DEVICE_CHECK when bits were set.
 */
TG_API tg_status tg_device_status(tg_stream_t stream, uint32_t* bits_out);

/*
 * The same read-and-clear of the device status word with the bits as a signed
 * code (0 = no kernel reported a failure).  Synchronises `stream`; returns
 * TG_ERR_DEVICE_CHECK when bits were set, TG_ERR_INVALID_ARG for a NULL
 * code_out.  Bits: 1 a gate pipeline wait gave up, 2 an attention wait gave
 * up (forward or backward), 4 the top-K selection produced more rows than M_b (extra rows skipped),
 * 8 a kept index outside the prompt batch reached the gather (row skipped),
 * 16 a gather pipeline wait gave up, 32 a chunk load of the chunked delta-rule
 * scan did not land.
 */
TG_API tg_status tg_last_device_error(tg_stream_t stream, int32_t* code_out);

/*
 * Host-only helper: validates a prompt batch and writes the kept-row offsets
 * cu_kept_h[0..batch] (cu_kept_h[b+1] - cu_kept_h[b] = M_b) so the caller can
 * size the outputs of the later calls.  All arrays are host memory.
 */
TG_API tg_status tg_kept_offsets(int32_t batch, const int32_t* cu_seqlens_h, const int32_t* doc_begin_h,
                          const int32_t* doc_end_h, const int32_t* budget_h, int32_t* cu_kept_h);

/*
 * Step 1 -- gate score (pages: "at layer L a small MLP scores each token from
 * its post-attention residual").  For every token j:
 *     z[j] = sum_u w2[u] * GELU(sum_c W1[u,c] h[j,c] + b1[u]) + b2
 * with the exact (erf) GELU, products accumulated in fp32.
 *   h        device [n_tokens, d_model], dtype, row-major, 16-byte aligned
 *   W1       device [d_hidden, d_model], same dtype, row-major (K-major)
 *   b1, w2   device [d_hidden] fp32;  b2 host scalar
 *   z_out    device [n_tokens] fp32
 *   algo     tg_algo.  The tcgen05 kernel needs bf16, d_model % 64 == 0 and
 *            d_hidden a multiple of 32 in [32, 256].
 */
TG_API tg_status tg_gate_score(const void* h, tg_dtype dtype, int64_t n_tokens, int32_t d_model,
                        const void* W1, const float* b1, int32_t d_hidden, const float* w2,
                        float b2, float* z_out, int32_t algo, tg_stream_t stream);

/*
 * Step 2 -- top-K over each prompt's document span, question protected
 * (pages: "a top-K selector keeps the highest-scoring tokens"; "only the
 * document part of the prompt is pruned, the question is never touched"; the
 * user budget is max_kept_prefill_tokens).  Selection order: larger fp32 score
 * first; +0.0 and -0.0 are equal; equal scores by lower index; NaN after every
 * number.  Exactly min(K, n_doc) document tokens are kept, so the result is
 * unique.
 *   z             device [total_tokens] fp32 scores
 *   batch, cu_seqlens_h[batch+1], doc_begin_h/doc_end_h/budget_h[batch]: host
 *   kept_idx_out  device [M] int32 global row ids, ascending within a prompt,
 *                 prompts in order (M = sum M_b, see tg_kept_offsets)
 *   cu_kept_out   device [batch+1] int32 kept-row offsets (may be NULL)
 * Limits: N_b <= 360448 tokens per prompt (TG_ERR_UNSUPPORTED beyond).
 */
TG_API tg_status tg_topk_select(const float* z, int32_t batch, const int32_t* cu_seqlens_h,
                         const int32_t* doc_begin_h, const int32_t* doc_end_h,
                         const int32_t* budget_h, int32_t* kept_idx_out, int32_t* cu_kept_out,
                         tg_stream_t stream);

/*
 * Bytes of the top-K workspace for a batch of `batch` prompts (0 outside
 * 1..TG_MAX_BATCH): per prompt, the first radix pass's 2048-bin histogram of
 * its document scores and a tag (8448 bytes).  total_tokens does not change
 * the size.  The workspace carries the histograms from tg_gate_score_hist to
 * tg_topk_select_ws; the caller zeroes it once after allocating it (for
 * example cudaMemsetAsync), and every tg_topk_select_ws leaves it zeroed
 * again.  Host-only.
 */
TG_API size_t tg_topk_workspace_bytes(int32_t batch, int64_t total_tokens);

/*
 * Step 1 with the selection's first radix pass folded into the gate's epilogue
 * (the scores are in registers there): as tg_gate_score, and each document
 * token's score is also counted into its prompt's first-pass histogram in the
 * top-K workspace, so tg_topk_select_ws starts at the second pass.
 *   batch, cu_seqlens_h[batch+1], doc_begin_h/doc_end_h[batch]: host, as for
 *       tg_topk_select (cu_seqlens_h[batch] must equal n_tokens; 1..TG_MAX_BATCH
 *       prompts)
 *   topk_workspace, topk_workspace_bytes: device, >= tg_topk_workspace_bytes,
 *       16-byte aligned, zero on entry (it is after allocation plus a memset
 *       and after every tg_topk_select_ws); TG_ERR_WORKSPACE when smaller
 * Other arguments and errors as tg_gate_score.  The histograms name the
 * scores they were counted from (z_out): a tg_topk_select_ws on other scores,
 * or on a workspace counted twice, finds the name or the counts wrong and
 * counts the first pass itself.
 */
TG_API tg_status tg_gate_score_hist(const void* h, tg_dtype dtype, int64_t n_tokens,
                                    int32_t d_model, const void* W1, const float* b1,
                                    int32_t d_hidden, const float* w2, float b2, float* z_out,
                                    int32_t batch, const int32_t* cu_seqlens_h,
                                    const int32_t* doc_begin_h, const int32_t* doc_end_h,
                                    void* topk_workspace, size_t topk_workspace_bytes,
                                    int32_t algo, tg_stream_t stream);

/*
 * Step 2 on a top-K workspace: the selection of tg_topk_select, exactly (the
 * same rows), taking the first pass's histograms from the workspace when
 * tg_gate_score_hist counted them from these scores z (otherwise counting
 * them itself), and leaving the workspace zeroed for the next gate.
 *   workspace, workspace_bytes: device, >= tg_topk_workspace_bytes(batch, .),
 *       16-byte aligned (TG_ERR_WORKSPACE when smaller); calls that share a
 *       workspace must not overlap on the GPU.
 * Other arguments, order, limits and errors as tg_topk_select.
 */
TG_API tg_status tg_topk_select_ws(const float* z, int32_t batch, const int32_t* cu_seqlens_h,
                                   const int32_t* doc_begin_h, const int32_t* doc_end_h,
                                   const int32_t* budget_h, int32_t* kept_idx_out,
                                   int32_t* cu_kept_out, void* workspace, size_t workspace_bytes,
                                   tg_stream_t stream);

#define TG_MAX_BUDGETS 8

/*
 * Step 2 for a budget sweep: one scoring pass, several budgets (pages: the
 * budget max_kept_prefill_tokens is a user choice; sweeping it reuses the
 * gate's scores).  Budget q keeps, per prompt, exactly what tg_topk_select
 * with budgets_h[q * batch .. q * batch + batch - 1] keeps; all budgets are
 * selected in one launch from the same scores.
 *   n_budgets     1 .. TG_MAX_BUDGETS
 *   budgets_h     host [n_budgets][batch] document tokens to keep
 *   kept_idx_out  host array of n_budgets device pointers, budget q's rows
 *                 [M_q] (M_q = sum over prompts of its kept rows)
 *   cu_kept_out   host array of n_budgets device pointers [batch+1] (entries
 *                 may be NULL), or NULL
 * Other arguments, order and limits as for tg_topk_select.
 */
TG_API tg_status tg_topk_select_multi(const float* z, int32_t batch, const int32_t* cu_seqlens_h,
                               const int32_t* doc_begin_h, const int32_t* doc_end_h,
                               int32_t n_budgets, const int32_t* budgets_h,
                               int32_t* const* kept_idx_out, int32_t* const* cu_kept_out,
                               tg_stream_t stream);

/*
 * The budget sweep on a top-K workspace: the selections of tg_topk_select_multi
 * (the same rows for every budget), with every budget's first radix pass taken
 * from the one histogram tg_gate_score_hist counted from these scores -- the
 * scores' histogram is computed once and each budget takes its threshold from
 * it -- and the workspace left zeroed once the last budget has read it.
 * Arguments as tg_topk_select_multi plus the workspace of tg_topk_select_ws.
 */
TG_API tg_status tg_topk_select_multi_ws(const float* z, int32_t batch,
                                         const int32_t* cu_seqlens_h, const int32_t* doc_begin_h,
                                         const int32_t* doc_end_h, int32_t n_budgets,
                                         const int32_t* budgets_h, int32_t* const* kept_idx_out,
                                         int32_t* const* cu_kept_out, void* workspace,
                                         size_t workspace_bytes, tg_stream_t stream);

/*
 * Random-K selection (pages: the random-K selector ablation, which keeps K
 * document tokens at random instead of by gate score).  The random numbers are
 * the caller's: keys[total_tokens] uint32, one per token (for example i.i.d.
 * uniform from a counter-based generator); the K document tokens with the
 * largest keys are kept, equal keys by lower index, question protected, rows
 * ascending -- the selection of tg_topk_select with the keys as scores.  With
 * i.i.d. uniform keys every K-subset of the document is equally likely.
 */
TG_API tg_status tg_random_select(const uint32_t* keys, int32_t batch, const int32_t* cu_seqlens_h,
                           const int32_t* doc_begin_h, const int32_t* doc_end_h,
                           const int32_t* budget_h, int32_t* kept_idx_out, int32_t* cu_kept_out,
                           tg_stream_t stream);

/* One tensor to compact: rows of `row_elems` elements, pitch = row_elems. */
typedef struct {
    const void* src;     /* device [total_tokens, row_elems] */
    void* dst;           /* device [M, row_elems] */
    int32_t row_elems;   /* elements per row; row bytes must be a multiple of 16 */
    int32_t rope_heads;  /* 0 = plain copy; else the first rope_heads*head_dim elements
                            are rope_heads heads rotated by RoPE (rotate-half pairing,
                            angle pos * theta^(-2i/head_dim), pos = original position
                            within the prompt, angles evaluated in fp64) */
} tg_gather_tensor;

#define TG_MAX_GATHER_TENSORS 8

/*
 * Step 3 -- compaction (pages: "layers above L process only the kept K tokens
 * and create no KV cache for the removed ones").  For each kept row i:
 *     dst_t[i] = src_t[kept_idx[i]]            (RoPE applied where requested)
 *     logsig_out[i] = log sigmoid(z[kept_idx[i]]) for document tokens, 0 for
 *                     question tokens (the per-key bias term of step 4)
 *   kept_idx      device [m_total] from tg_topk_select
 *   prompt arrays host, as for tg_topk_select (m_total must equal sum M_b)
 *   tensors       host array of n_tensors (<= TG_MAX_GATHER_TENSORS) entries
 *   head_dim      RoPE head size (even, <= 256) when any rope_heads > 0
 *   z             device [total_tokens] fp32 (may be NULL when logsig_out is NULL)
 *   logsig_out    device [m_total] fp32 or NULL
 */
TG_API tg_status tg_compact_gather(const int32_t* kept_idx, int64_t m_total, int32_t batch,
                            const int32_t* cu_seqlens_h, const int32_t* doc_begin_h,
                            const int32_t* doc_end_h, const int32_t* budget_h, tg_dtype dtype,
                            const tg_gather_tensor* tensors, int32_t n_tensors, int32_t head_dim,
                            double rope_theta, const float* z, float* logsig_out,
                            tg_stream_t stream);

/*
 * Step 4 -- token-gated causal GQA attention over the kept rows (pages: the
 * kept tokens' scores become a bias on the attention logits above the gate,
 * scaled by a per-head learned gain; a per-head learned temperature corrects
 * for each query seeing fewer keys).  For prompt b, query row i, head h:
 *     logit_j = (q_i . k_j) / (sqrt(head_dim) * temp[h]) + gain[h] * logsig[j]
 *     out_i   = sum_{j <= i in prompt b} softmax_j(logit) v_j
 *     lse[h, i] = log sum_j exp(logit_j)            (natural log)
 * with kv head = h / (n_q_heads / n_kv_heads).  logsig == NULL means no bias.
 *   q    device [M, n_q_heads, head_dim];  k, v device [M, n_kv_heads, head_dim]
 *   cu_kept_h  host [batch+1] kept-row offsets (M = cu_kept_h[batch])
 *   gain, temp device [n_q_heads] fp32 (temp > 0)
 *   out  device [M, n_q_heads, head_dim], dtype;  lse device [n_q_heads, M] or NULL
 *   workspace, workspace_bytes
 *        device scratch owned by the caller, or NULL.  With a workspace the
 *        tensor-core kernel may split the key range of long query tiles over
 *        several SMs when the batch is too small to fill the GPU; each chunk's
 *        partial output is merged in a fixed order, so results do not depend on
 *        scheduling.  Size it with tg_attention_workspace_bytes (same arguments,
 *        same device); a smaller non-NULL workspace returns TG_ERR_WORKSPACE.
 *        16-byte aligned.  Calls that share a workspace must not overlap on the
 *        GPU (the call clears its counters with an asynchronous memset on stream).
 *   algo tg_algo; the tcgen05 kernel needs bf16 and head_dim in {64, 128}.
 */
TG_API tg_status tg_gated_attention(const void* q, const void* k, const void* v, tg_dtype dtype,
                             int32_t batch, const int32_t* cu_kept_h, int32_t n_q_heads,
                             int32_t n_kv_heads, int32_t head_dim, const float* logsig,
                             const float* gain, const float* temp, void* out, float* lse,
                             void* workspace, size_t workspace_bytes, int32_t algo,
                             tg_stream_t stream);

/*
 * Bytes of workspace tg_gated_attention can use for this batch and head shape
 * on the current device (0 when it would not split, e.g. large batches, fp32,
 * or TG_ALGO_SIMT).  Host-only: reads cu_kept_h, launches nothing.
 */
TG_API tg_status tg_attention_workspace_bytes(tg_dtype dtype, int32_t batch, const int32_t* cu_kept_h,
                                       int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                       int32_t algo, size_t* bytes_out);

/* The attention kernels tg_gated_attention chooses between. */
typedef enum {
    TG_ATTN_SIMT = 0,      /* CUDA-core kernel */
    TG_ATTN_TC = 1,        /* tcgen05 kernel, one SM per (query tile, head pair) */
    TG_ATTN_TC_SPLIT = 2,  /* same, long query tiles split by key range (uses the workspace) */
    TG_ATTN_TC_PAIR = 3    /* tcgen05 kernel on CTA pairs, two SMs per (query tile, head pair) */
} tg_attn_kernel;

/*
 * Which kernel tg_gated_attention launches for this batch and head shape on
 * the current device (a tg_attn_kernel in *kernel_out).  with_workspace: the
 * call will receive a workspace of tg_attention_workspace_bytes.  Host-only.
 */
TG_API tg_status tg_attention_kernel(tg_dtype dtype, int32_t batch, const int32_t* cu_kept_h,
                              int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                              int32_t algo, int32_t with_workspace, int32_t* kernel_out);

/*
 * tg_gated_attention for callers that cannot allocate device memory (the
 * pages have no counterpart: this is a deployment convenience).  A serving
 * process whose allocator reserved the whole GPU up front, or code that must
 * not allocate around CUDA-graph capture, cannot provide the attention
 * workspace; this call takes the scratch from a fixed array built into the
 * library instead: 32 MiB of device memory, held by every GPU that loads the
 * library until the process exits.
 *   Arguments, results and errors are those of tg_gated_attention without the
 *   workspace.  A batch whose split plan needs more scratch than the array
 *   holds runs the unsplit plan (each query tile on one SM), which needs none:
 *   the results are the same up to rounding, only the schedule differs.
 *   The first call on a device looks up the array's address (a runtime call,
 *   no allocation): make it before any stream capture on that device.  The
 *   address is looked up again when the device's context has changed (after a
 *   cudaDeviceReset), so it never outlives the context it belongs to.
 *   All calls share the array: calls that run on the GPU at the same time race
 *   on it, so issue them in order on one stream.  The call allocates nothing.
 */
TG_API tg_status tg_gated_attention_noalloc(const void* q, const void* k, const void* v, tg_dtype dtype,
                                     int32_t batch, const int32_t* cu_kept_h, int32_t n_q_heads,
                                     int32_t n_kv_heads, int32_t head_dim, const float* logsig,
                                     const float* gain, const float* temp, void* out, float* lse,
                                     int32_t algo, tg_stream_t stream);

/*
 * Backward of tg_gated_attention: the gradient that trains the gate.  The
 * gate's score enters every attention layer above the gate as a bias on the
 * logits scaled by a per-head gain (TokenGate, "How it works": the Mixture-of-
 * Experts router trick), so a loss on the attention output reaches the scorer
 * through it; the per-head gains and temperatures are learned the same way.
 *
 * For a scalar loss L and dout = dL/dout [M, Hq, head_dim] (dtype of q), with
 * out and lse the forward's outputs for the same inputs, the call writes (fp32,
 * overwritten, device):
 *   d_logsig [M]  dL/dl_j for every kept row j (l = logsig, the bias input)
 *   d_z_kept [M]  dL/dz of the kept rows' gate scores, d_logsig * (1 - exp(l)):
 *                 l = log sigmoid(z) for document rows; question rows (l fixed
 *                 at 0) get 0
 *   d_gain [Hq]   dL/dg_h
 *   d_temp [Hq]   dL/dtau_h
 * Per prompt, head h and query row i, with P the attention weights,
 * dP_ij = dout_i . v_j, D_i = dout_i . out_i and dlogit_ij = P_ij (dP_ij - D_i):
 * dL/dl_j = sum g_h dlogit_ij, dL/dg_h = sum l_j dlogit_ij, dL/dtau_h =
 * -sum dlogit_ij (q_i . k_j) / (sqrt(head_dim) tau_h^2).  Gradients with respect
 * to q, k and v are not computed.
 *   lse        [Hq, M] natural-log LSE from tg_gated_attention (required)
 *   logsig     [M] (required: without the bias there is no gate gradient)
 *   workspace  device scratch of tg_attention_backward_workspace_bytes bytes,
 *              16-byte aligned (TG_ERR_WORKSPACE when smaller)
 *   algo       tg_algo (TG_ALGO_TCGEN05 needs bf16)
 * Other arguments, layouts and errors as tg_gated_attention.  Results are summed
 * with floating-point atomics, so the last bits may differ between calls.
 */
TG_API tg_status tg_gated_attention_backward(const void* q, const void* k, const void* v,
                                             tg_dtype dtype, int32_t batch,
                                             const int32_t* cu_kept_h, int32_t n_q_heads,
                                             int32_t n_kv_heads, int32_t head_dim,
                                             const float* logsig, const float* gain,
                                             const float* temp, const void* out, const float* lse,
                                             const void* dout, float* d_logsig, float* d_z_kept,
                                             float* d_gain, float* d_temp, void* workspace,
                                             size_t workspace_bytes, int32_t algo,
                                             tg_stream_t stream);

/*
 * Steps of a stack of gated upper layers.  Every attention layer above the gate
 * keeps working on the same kept rows and creates KV only for them (TokenGate,
 * "How it works"), each with its own gain and temperature on the shared
 * log-gates.  The layers are Qwen3-shaped: RMSNorm, a fused QKV projection,
 * per-head RMSNorm of q and k, RoPE at the kept rows' original positions,
 * tg_gated_attention, an output projection, RMSNorm and a SwiGLU MLP.  The
 * projections are plain GEMMs left to the caller (cuBLAS); these calls do the
 * rest.  Row-major, contiguous, device pointers; dtype TG_BF16 or TG_FP32 with
 * fp32 arithmetic.
 *
 * tg_rmsnorm: out[r, c] = x[r, c] / sqrt(mean_c x[r, c]^2 + eps) * weight[c].
 *   x, out [rows, dim] (out may equal x), weight [dim].
 */
TG_API tg_status tg_rmsnorm(const void* x, const void* weight, void* out, tg_dtype dtype,
                            int64_t rows, int32_t dim, float eps, tg_stream_t stream);

/*
 * tg_qkv_rope_emit: split of a fused QKV projection of the kept rows.
 *   qkv      [M, (n_q_heads + 2 n_kv_heads) * head_dim]: q heads, then k heads, then v
 *   q_out    [M, n_q_heads, head_dim]    RMSNorm(q_h) * q_norm_w, then RoPE
 *   k_out    [M, n_kv_heads, head_dim]   RMSNorm(k_h) * k_norm_w, then RoPE (the KV cache
 *                                        slot of this layer, compacted)
 *   v_out    [M, n_kv_heads, head_dim]   v as it is (the cache slot)
 *   RoPE: rotate-half pairs (i, i + head_dim/2), angle pos * rope_theta^(-2i/head_dim)
 *   with pos = kept_idx[i] - cu_seqlens_h[b] the row's original position in its
 *   prompt b (cu_kept_h gives the kept rows of each prompt, host arrays as in
 *   tg_compact_gather).  head_dim 64 or 128.
 */
TG_API tg_status tg_qkv_rope_emit(const void* qkv, tg_dtype dtype, int32_t batch,
                                  const int32_t* cu_seqlens_h, const int32_t* cu_kept_h,
                                  const int32_t* kept_idx, int32_t n_q_heads, int32_t n_kv_heads,
                                  int32_t head_dim, const void* q_norm_w, const void* k_norm_w,
                                  float eps, double rope_theta, void* q_out, void* k_out,
                                  void* v_out, tg_stream_t stream);

/*
 * tg_swiglu: out[r, c] = SiLU(gate_up[r, c]) * gate_up[r, inter + c], SiLU(g) = g / (1 + e^-g).
 *   gate_up [rows, 2 inter] (the fused gate and up projections), out [rows, inter].
 */
TG_API tg_status tg_swiglu(const void* gate_up, void* out, tg_dtype dtype, int64_t rows,
                           int32_t inter, tg_stream_t stream);

/*
 * tg_gated_delta_scan: a Gated DeltaNet (linear-attention) layer of a hybrid
 * backbone above the gate, over each prompt's kept rows only.  TokenGate prunes
 * these layers as well as the attention layers (lucasainews.com, "성능 결과",
 * with its comparison table; lefilia.fr, body; the abstract's "hybrid-attention
 * models").  The pages do not write the layer out; this is the published gated
 * delta rule (Gated DeltaNet), with no gate bias (the bias acts on attention
 * logits) and a zero initial state.  Per prompt b and head h, over the kept rows
 * t of b in order:
 *   k^_t = k_t / sqrt(|k_t|^2 + eps),   q^_t = q_t / sqrt(|q_t|^2 + eps) / sqrt(head_dim)
 *   S_t  = alpha_t S_{t-1} + beta_t (v_t - alpha_t S_{t-1} k^_t) k^_t^T,  alpha_t = exp(log_alpha_t)
 *   out_t = S_t q^_t
 *   q, k, v        [M, n_heads, head_dim] (device, dtype, 16-byte aligned), M = cu_kept_h[batch]
 *   log_alpha,beta [M, n_heads] fp32 (log_alpha <= 0 keeps the state bounded; -inf is alpha = 0)
 *   cu_kept_h      [batch + 1] host array (prefix sums of the kept rows per prompt)
 *   out            [M, n_heads, head_dim] (dtype)
 *   state_out      [batch, n_heads, head_dim (v), head_dim (k)] fp32: S after each prompt's
 *                  last row (zero for a prompt with no rows); NULL to skip
 *   head_dim 64 or 128 (else TG_ERR_UNSUPPORTED); state kept in fp32.  One CTA per 32 state
 *   rows of a (prompt, head): batch x n_heads x head_dim / 32 above INT32_MAX is
 *   TG_ERR_UNSUPPORTED.  Errors: TG_ERR_DTYPE, TG_ERR_SHAPE (n_heads <= 0),
 *   TG_ERR_INVALID_ARG (cu_kept_h, eps < 0, null pointers with rows to process),
 *   TG_ERR_ALIGNMENT; nothing is launched on an error.
 */
TG_API tg_status tg_gated_delta_scan(const void* q, const void* k, const void* v, tg_dtype dtype,
                                     const float* log_alpha, const float* beta, int32_t batch,
                                     const int32_t* cu_kept_h, int32_t n_heads, int32_t head_dim,
                                     float eps, void* out, float* state_out, tg_stream_t stream);

/*
 * tg_gated_delta_scan_chunked: the function of tg_gated_delta_scan (same
 * arguments, results and errors, same tolerance to fp32 rounding) computed in
 * chunks of 64 rows.  With S_0 the state before a chunk, everything inside the
 * chunk that does not involve S_0 -- the unit lower-triangular solve of the
 * chunk's delta-rule corrections, the within-chunk decayed products of q, k and
 * v -- is computed for every (chunk, head) at once, in parallel; the state then
 * passes from chunk to chunk with three small products per chunk, split over
 * blocks of 16 state rows (rows of S are independent).  This is the chunked
 * linear-attention scan; the recurrence walks the rows one by one.
 *   workspace  device scratch of tg_delta_scan_workspace_bytes bytes, 256-byte
 *              aligned (TG_ERR_WORKSPACE when smaller or NULL with rows to scan,
 *              TG_ERR_ALIGNMENT when misaligned); every call overwrites it, so
 *              calls that share it must not overlap on the GPU.
 *   batch x n_heads above 65535: TG_ERR_UNSUPPORTED.
 */
TG_API tg_status tg_gated_delta_scan_chunked(const void* q, const void* k, const void* v,
                                             tg_dtype dtype, const float* log_alpha,
                                             const float* beta, int32_t batch,
                                             const int32_t* cu_kept_h, int32_t n_heads,
                                             int32_t head_dim, float eps, void* out,
                                             float* state_out, void* workspace,
                                             size_t workspace_bytes, tg_stream_t stream);

/*
 * Workspace bytes tg_gated_delta_scan_chunked needs (host-only): per chunk of 64
 * kept rows of a prompt and per head, five 64 x head_dim fp32 matrices and the
 * chunk's decay (about 160 KB at head_dim 128).
 */
TG_API tg_status tg_delta_scan_workspace_bytes(int32_t batch, const int32_t* cu_kept_h,
                                               int32_t n_heads, int32_t head_dim,
                                               size_t* bytes_out);

/* Workspace bytes tg_gated_attention_backward needs for this batch (host-only). */
TG_API tg_status tg_attention_backward_workspace_bytes(int32_t batch, const int32_t* cu_kept_h,
                                                       int32_t n_q_heads, size_t* bytes_out);

#ifdef __cplusplus
}
#endif

#endif /* TOKENGATE_H_ */
