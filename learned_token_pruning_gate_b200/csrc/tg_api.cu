// C ABI of libtokengate: argument validation, prompt-table construction and
// kernel dispatch.  No call allocates device memory or synchronises the stream
// (except tg_device_status, whose purpose is to read the status word).
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "tg_internal.cuh"

namespace tg {

static thread_local char g_msg[512] = "no error";

tg_status set_error(tg_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

tg_status cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return TG_OK;
  return set_error(TG_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Unique id of the calling thread's current CUDA context (0 when unavailable).
// Device addresses of the library's __device__ arrays belong to one context: a
// cudaDeviceReset destroys the primary context, and the next call runs in a new
// one with the module loaded again, possibly elsewhere.  Context ids are never
// reused within a process, so a cache keyed on them cannot hand out an address
// of a destroyed context.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

uint64_t current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return static_cast<uint64_t>(id) + 1;  // 0 stays "unknown"
}

void* SymbolAddressCache::get(const void* symbol) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu_);
  const uint64_t ctx = current_context_id();
  if (addr_[dev] && ctx != 0 && ctx == ctx_[dev]) return addr_[dev];
  // the lookup makes the device's primary context current when none is yet
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess) return nullptr;
  addr_[dev] = p;
  ctx_[dev] = current_context_id();  // 0 (unknown) makes every call look the address up
  return p;
}

// The status word lives in device global memory of each GPU that loaded the
// library; kernels only ever atomically OR bits into it.
static __device__ uint32_t g_status_word;

uint32_t* device_status_word() {
  static SymbolAddressCache cache;
  return static_cast<uint32_t*>(cache.get(reinterpret_cast<const void*>(&g_status_word)));
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n > 0 ? n : 148;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor map with 128-byte swizzle; out-of-range rows read as zero.
bool encode_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                         uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t elem_strides[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates a prompt batch and fills the table; returns the longest prompt.
static tg_status build_table(int32_t batch, const int32_t* cu, const int32_t* s, const int32_t* e,
                             const int32_t* k, PromptTable* t, int* max_len, int* max_kept) {
  if (batch < 0) return set_error(TG_ERR_INVALID_ARG, "batch=%d is negative", batch);
  if (batch > kMaxBatch)
    return set_error(TG_ERR_UNSUPPORTED, "batch=%d exceeds TG_MAX_BATCH=%d", batch, kMaxBatch);
  if (!cu || !s || !e || !k) return set_error(TG_ERR_INVALID_ARG, "null prompt array");
  memset(t, 0, sizeof(*t));
  t->batch = batch;
  if (cu[0] != 0) return set_error(TG_ERR_INVALID_ARG, "cu_seqlens[0]=%d must be 0", cu[0]);
  int ml = 0, mk = 0;
  int64_t kept = 0;
  for (int b = 0; b < batch; ++b) {
    int64_t n = static_cast<int64_t>(cu[b + 1]) - cu[b];
    if (n < 0) return set_error(TG_ERR_INVALID_ARG, "cu_seqlens decreases at prompt %d", b);
    if (s[b] < 0 || e[b] < s[b] || e[b] > n)
      return set_error(TG_ERR_INVALID_ARG, "prompt %d: document span [%d,%d) outside [0,%lld)", b,
                       s[b], e[b], static_cast<long long>(n));
    if (k[b] < 0) return set_error(TG_ERR_INVALID_ARG, "prompt %d: budget %d < 0", b, k[b]);
    int n_doc = e[b] - s[b];
    int keep = k[b] < n_doc ? k[b] : n_doc;
    int m = keep + static_cast<int>(n - n_doc);
    t->start[b] = cu[b];
    t->doc_begin[b] = s[b];
    t->doc_end[b] = e[b];
    t->k_keep[b] = keep;
    t->kept_start[b] = static_cast<int32_t>(kept);
    kept += m;
    if (n > ml) ml = static_cast<int>(n);
    if (m > mk) mk = m;
  }
  t->start[batch] = cu[batch];
  t->kept_start[batch] = static_cast<int32_t>(kept);
  if (max_len) *max_len = ml;
  if (max_kept) *max_kept = mk;
  return TG_OK;
}

// Table over the kept rows only (attention): kept_start from cu_kept, no spans.
static tg_status build_kept_table(int32_t batch, const int32_t* cu_kept, PromptTable* t,
                                  int* max_len) {
  if (batch < 0) return set_error(TG_ERR_INVALID_ARG, "batch=%d is negative", batch);
  if (batch > kMaxBatch)
    return set_error(TG_ERR_UNSUPPORTED, "batch=%d exceeds TG_MAX_BATCH=%d", batch, kMaxBatch);
  if (!cu_kept) return set_error(TG_ERR_INVALID_ARG, "cu_kept_h is null");
  if (cu_kept[0] != 0) return set_error(TG_ERR_INVALID_ARG, "cu_kept[0] must be 0");
  memset(t, 0, sizeof(*t));
  t->batch = batch;
  int ml = 0;
  for (int b = 0; b < batch; ++b) {
    int n = cu_kept[b + 1] - cu_kept[b];
    if (n < 0) return set_error(TG_ERR_INVALID_ARG, "cu_kept decreases at prompt %d", b);
    t->start[b] = cu_kept[b];
    t->kept_start[b] = cu_kept[b];
    if (n > ml) ml = n;
  }
  t->start[batch] = cu_kept[batch];
  t->kept_start[batch] = cu_kept[batch];
  *max_len = ml;
  return TG_OK;
}

}  // namespace tg

using namespace tg;

extern "C" {

const char* tg_status_string(tg_status s) {
  switch (s) {
    case TG_OK: return "TG_OK";
    case TG_ERR_INVALID_ARG: return "TG_ERR_INVALID_ARG";
    case TG_ERR_SHAPE: return "TG_ERR_SHAPE";
    case TG_ERR_DTYPE: return "TG_ERR_DTYPE";
    case TG_ERR_ALIGNMENT: return "TG_ERR_ALIGNMENT";
    case TG_ERR_UNSUPPORTED: return "TG_ERR_UNSUPPORTED";
    case TG_ERR_CUDA: return "TG_ERR_CUDA";
    case TG_ERR_DEVICE_CHECK: return "TG_ERR_DEVICE_CHECK";
    case TG_ERR_WORKSPACE: return "TG_ERR_WORKSPACE";
  }
  return "TG_ERR_UNKNOWN";
}

const char* tg_last_error_message(void) { return g_msg; }

const char* tg_version(void) { return "0.1.0 sm_100a"; }

tg_status tg_device_status(tg_stream_t stream, uint32_t* bits_out) {
  if (!bits_out) return set_error(TG_ERR_INVALID_ARG, "bits_out is null");
  uint32_t* w = device_status_word();
  if (!w) return set_error(TG_ERR_CUDA, "cannot resolve the device status word");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t bits = 0;
  tg_status r = cuda_check(cudaMemcpyAsync(&bits, w, sizeof(bits), cudaMemcpyDeviceToHost, st),
                           "read status word");
  if (r != TG_OK) return r;
  if ((r = cuda_check(cudaStreamSynchronize(st), "synchronize")) != TG_OK) return r;
  *bits_out = bits;
  if (bits) {
    const uint32_t zero = 0;
    if ((r = cuda_check(cudaMemcpy(w, &zero, sizeof(zero), cudaMemcpyHostToDevice),
                        "clear status word")) != TG_OK)
      return r;
    return set_error(TG_ERR_DEVICE_CHECK, "device status bits 0x%x", bits);
  }
  return TG_OK;
}

tg_status tg_last_device_error(tg_stream_t stream, int32_t* code_out) {
  if (!code_out) return set_error(TG_ERR_INVALID_ARG, "code_out is null");
  uint32_t bits = 0;
  const tg_status r = tg_device_status(stream, &bits);
  *code_out = static_cast<int32_t>(bits);
  return r;
}

tg_status tg_kept_offsets(int32_t batch, const int32_t* cu, const int32_t* s, const int32_t* e,
                          const int32_t* k, int32_t* cu_kept) {
  if (!cu_kept) return set_error(TG_ERR_INVALID_ARG, "cu_kept_h is null");
  PromptTable t;
  tg_status r = build_table(batch, cu, s, e, k, &t, nullptr, nullptr);
  if (r != TG_OK) return r;
  for (int b = 0; b <= batch; ++b) cu_kept[b] = t.kept_start[b];
  return TG_OK;
}

// The gate call with or without the top-K workspace's histograms.
static tg_status gate_score_impl(const void* h, tg_dtype dtype, int64_t n_tokens, int32_t d_model,
                                 const void* W1, const float* b1, int32_t d_hidden,
                                 const float* w2, float b2, float* z_out, int32_t algo,
                                 const GateHist& gh, tg_stream_t stream) {
  if (dtype != TG_BF16 && dtype != TG_FP32) return set_error(TG_ERR_DTYPE, "dtype %d", dtype);
  if (n_tokens < 0 || d_model <= 0 || d_hidden <= 0)
    return set_error(TG_ERR_INVALID_ARG, "n_tokens=%lld d_model=%d d_hidden=%d",
                     static_cast<long long>(n_tokens), d_model, d_hidden);
  if (n_tokens > 0x7FFFFFFFll) return set_error(TG_ERR_UNSUPPORTED, "n_tokens beyond int32");
  if (algo < TG_ALGO_AUTO || algo > TG_ALGO_TCGEN05)
    return set_error(TG_ERR_INVALID_ARG, "algo %d", algo);
  if (n_tokens == 0) return TG_OK;
  if (!h || !W1 || !b1 || !w2 || !z_out) return set_error(TG_ERR_INVALID_ARG, "null pointer");
  const int esz = dtype == TG_BF16 ? 2 : 4;
  if (!aligned16(h) || !aligned16(W1) || (static_cast<int64_t>(d_model) * esz) % 16 != 0)
    return set_error(TG_ERR_ALIGNMENT, "h/W1 rows must be 16-byte aligned");
  const bool tc_ok = dtype == TG_BF16 && d_model % 64 == 0 && d_hidden % 32 == 0 &&
                     d_hidden >= 32 && d_hidden <= 256;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (algo == TG_ALGO_TCGEN05 && !tc_ok)
    return set_error(TG_ERR_UNSUPPORTED,
                     "tcgen05 gate needs bf16, d_model%%64==0, d_hidden in 32..256 step 32");
  if (algo == TG_ALGO_SIMT || !tc_ok)
    return launch_gate_simt(h, dtype, n_tokens, d_model, W1, b1, d_hidden, w2, b2, z_out, gh, st);
  return launch_gate_tc(h, n_tokens, d_model, W1, b1, d_hidden, w2, b2, z_out, gh, st);
}

tg_status tg_gate_score(const void* h, tg_dtype dtype, int64_t n_tokens, int32_t d_model,
                        const void* W1, const float* b1, int32_t d_hidden, const float* w2,
                        float b2, float* z_out, int32_t algo, tg_stream_t stream) {
  static thread_local GateHist none;  // hist = nullptr: no histogram
  none.hist = nullptr;
  return gate_score_impl(h, dtype, n_tokens, d_model, W1, b1, d_hidden, w2, b2, z_out, algo, none,
                         stream);
}

size_t tg_topk_workspace_bytes(int32_t batch, int64_t total_tokens) {
  (void)total_tokens;  // the histograms are per prompt, whatever its length
  if (batch <= 0 || batch > kMaxBatch) return 0;
  return static_cast<size_t>(batch) * kHistStride * sizeof(uint32_t);
}

static tg_status check_topk_workspace(int32_t batch, const void* ws, size_t bytes) {
  if (!ws) return set_error(TG_ERR_INVALID_ARG, "top-K workspace is null");
  if (!aligned16(ws)) return set_error(TG_ERR_ALIGNMENT, "top-K workspace must be 16-byte aligned");
  const size_t need = tg_topk_workspace_bytes(batch, 0);
  if (bytes < need)
    return set_error(TG_ERR_WORKSPACE, "top-K workspace: %zu bytes given, %zu needed", bytes, need);
  return TG_OK;
}

tg_status tg_gate_score_hist(const void* h, tg_dtype dtype, int64_t n_tokens, int32_t d_model,
                             const void* W1, const float* b1, int32_t d_hidden, const float* w2,
                             float b2, float* z_out, int32_t batch, const int32_t* cu_seqlens_h,
                             const int32_t* doc_begin_h, const int32_t* doc_end_h,
                             void* topk_workspace, size_t topk_workspace_bytes, int32_t algo,
                             tg_stream_t stream) {
  static const int32_t kNoBudget[kMaxBatch] = {};  // the spans only: budgets play no part here
  PromptTable t;
  tg_status r = build_table(batch, cu_seqlens_h, doc_begin_h, doc_end_h, kNoBudget, &t, nullptr,
                            nullptr);
  if (r != TG_OK) return r;
  if (batch == 0) return set_error(TG_ERR_INVALID_ARG, "the histograms need at least one prompt");
  if (t.start[batch] != n_tokens)
    return set_error(TG_ERR_SHAPE, "cu_seqlens ends at %d, n_tokens=%lld", t.start[batch],
                     static_cast<long long>(n_tokens));
  if ((r = check_topk_workspace(batch, topk_workspace, topk_workspace_bytes)) != TG_OK) return r;
  static thread_local GateHist gh;
  gh.hist = static_cast<uint32_t*>(topk_workspace);
  gh.z = z_out;
  gh.n = static_cast<int32_t>(n_tokens);
  gh.batch = batch;
  for (int b = 0; b <= batch; ++b) gh.start[b] = t.start[b];
  for (int b = 0; b < batch; ++b) {
    gh.doc_lo[b] = t.start[b] + t.doc_begin[b];
    gh.doc_hi[b] = t.start[b] + t.doc_end[b];
  }
  return gate_score_impl(h, dtype, n_tokens, d_model, W1, b1, d_hidden, w2, b2, z_out, algo, gh,
                         stream);
}

// The selection with or without the gate's histograms.
static tg_status topk_select_impl(const float* z, int32_t batch, const int32_t* cu_seqlens_h,
                                  const int32_t* doc_begin_h, const int32_t* doc_end_h,
                                  const int32_t* budget_h, int32_t* kept_idx_out,
                                  int32_t* cu_kept_out, uint32_t* hist, tg_stream_t stream) {
  PromptTable t;
  int max_len = 0;
  tg_status r = build_table(batch, cu_seqlens_h, doc_begin_h, doc_end_h, budget_h, &t, &max_len,
                            nullptr);
  if (r != TG_OK) return r;
  if (batch == 0) return TG_OK;
  if (t.kept_start[batch] > 0 && !kept_idx_out)
    return set_error(TG_ERR_INVALID_ARG, "kept_idx_out is null");
  if (t.start[batch] > 0 && !z) return set_error(TG_ERR_INVALID_ARG, "z is null");
  if (max_len > 360448)
    return set_error(TG_ERR_UNSUPPORTED, "prompt of %d tokens exceeds 360448", max_len);
  return launch_topk(z, nullptr, &t, 1, max_len, &kept_idx_out, &cu_kept_out, hist,
                     reinterpret_cast<cudaStream_t>(stream));
}

tg_status tg_topk_select(const float* z, int32_t batch, const int32_t* cu_seqlens_h,
                         const int32_t* doc_begin_h, const int32_t* doc_end_h,
                         const int32_t* budget_h, int32_t* kept_idx_out, int32_t* cu_kept_out,
                         tg_stream_t stream) {
  return topk_select_impl(z, batch, cu_seqlens_h, doc_begin_h, doc_end_h, budget_h, kept_idx_out,
                          cu_kept_out, nullptr, stream);
}

tg_status tg_topk_select_ws(const float* z, int32_t batch, const int32_t* cu_seqlens_h,
                            const int32_t* doc_begin_h, const int32_t* doc_end_h,
                            const int32_t* budget_h, int32_t* kept_idx_out, int32_t* cu_kept_out,
                            void* workspace, size_t workspace_bytes, tg_stream_t stream) {
  if (batch > 0 && batch <= kMaxBatch) {
    tg_status r = check_topk_workspace(batch, workspace, workspace_bytes);
    if (r != TG_OK) return r;
  }
  return topk_select_impl(z, batch, cu_seqlens_h, doc_begin_h, doc_end_h, budget_h, kept_idx_out,
                          cu_kept_out, static_cast<uint32_t*>(workspace), stream);
}

static tg_status topk_select_multi_impl(const float* z, int32_t batch,
                                        const int32_t* cu_seqlens_h, const int32_t* doc_begin_h,
                                        const int32_t* doc_end_h, int32_t n_budgets,
                                        const int32_t* budgets_h, int32_t* const* kept_idx_out,
                                        int32_t* const* cu_kept_out, uint32_t* hist,
                                        tg_stream_t stream);

tg_status tg_topk_select_multi(const float* z, int32_t batch, const int32_t* cu_seqlens_h,
                               const int32_t* doc_begin_h, const int32_t* doc_end_h,
                               int32_t n_budgets, const int32_t* budgets_h,
                               int32_t* const* kept_idx_out, int32_t* const* cu_kept_out,
                               tg_stream_t stream) {
  return topk_select_multi_impl(z, batch, cu_seqlens_h, doc_begin_h, doc_end_h, n_budgets,
                                budgets_h, kept_idx_out, cu_kept_out, nullptr, stream);
}

tg_status tg_topk_select_multi_ws(const float* z, int32_t batch, const int32_t* cu_seqlens_h,
                                  const int32_t* doc_begin_h, const int32_t* doc_end_h,
                                  int32_t n_budgets, const int32_t* budgets_h,
                                  int32_t* const* kept_idx_out, int32_t* const* cu_kept_out,
                                  void* workspace, size_t workspace_bytes, tg_stream_t stream) {
  if (batch > 0 && batch <= kMaxBatch) {
    tg_status r = check_topk_workspace(batch, workspace, workspace_bytes);
    if (r != TG_OK) return r;
  }
  return topk_select_multi_impl(z, batch, cu_seqlens_h, doc_begin_h, doc_end_h, n_budgets,
                                budgets_h, kept_idx_out, cu_kept_out,
                                static_cast<uint32_t*>(workspace), stream);
}

static tg_status topk_select_multi_impl(const float* z, int32_t batch,
                                        const int32_t* cu_seqlens_h, const int32_t* doc_begin_h,
                                        const int32_t* doc_end_h, int32_t n_budgets,
                                        const int32_t* budgets_h, int32_t* const* kept_idx_out,
                                        int32_t* const* cu_kept_out, uint32_t* hist,
                                        tg_stream_t stream) {
  if (n_budgets < 1 || n_budgets > TG_MAX_BUDGETS)
    return set_error(TG_ERR_INVALID_ARG, "n_budgets=%d (1..%d)", n_budgets, TG_MAX_BUDGETS);
  if (!budgets_h || !kept_idx_out) return set_error(TG_ERR_INVALID_ARG, "null budget array");
  static thread_local PromptTable t[TG_MAX_BUDGETS];
  int max_len = 0;
  for (int q = 0; q < n_budgets; ++q) {
    tg_status r = build_table(batch, cu_seqlens_h, doc_begin_h, doc_end_h,
                              budgets_h + static_cast<int64_t>(q) * (batch > 0 ? batch : 0), &t[q],
                              &max_len, nullptr);
    if (r != TG_OK) return r;
    if (batch > 0 && t[q].kept_start[batch] > 0 && !kept_idx_out[q])
      return set_error(TG_ERR_INVALID_ARG, "kept_idx_out[%d] is null", q);
  }
  if (batch == 0) return TG_OK;
  if (t[0].start[batch] > 0 && !z) return set_error(TG_ERR_INVALID_ARG, "z is null");
  if (max_len > 360448)
    return set_error(TG_ERR_UNSUPPORTED, "prompt of %d tokens exceeds 360448", max_len);
  return launch_topk(z, nullptr, t, n_budgets, max_len, kept_idx_out, cu_kept_out, hist,
                     reinterpret_cast<cudaStream_t>(stream));
}

tg_status tg_random_select(const uint32_t* keys, int32_t batch, const int32_t* cu_seqlens_h,
                           const int32_t* doc_begin_h, const int32_t* doc_end_h,
                           const int32_t* budget_h, int32_t* kept_idx_out, int32_t* cu_kept_out,
                           tg_stream_t stream) {
  PromptTable t;
  int max_len = 0;
  tg_status r = build_table(batch, cu_seqlens_h, doc_begin_h, doc_end_h, budget_h, &t, &max_len,
                            nullptr);
  if (r != TG_OK) return r;
  if (batch == 0) return TG_OK;
  if (t.kept_start[batch] > 0 && !kept_idx_out)
    return set_error(TG_ERR_INVALID_ARG, "kept_idx_out is null");
  if (t.start[batch] > 0 && !keys) return set_error(TG_ERR_INVALID_ARG, "keys is null");
  if (max_len > 360448)
    return set_error(TG_ERR_UNSUPPORTED, "prompt of %d tokens exceeds 360448", max_len);
  return launch_topk(nullptr, keys, &t, 1, max_len, &kept_idx_out, &cu_kept_out, nullptr,
                     reinterpret_cast<cudaStream_t>(stream));
}

tg_status tg_compact_gather(const int32_t* kept_idx, int64_t m_total, int32_t batch,
                            const int32_t* cu_seqlens_h, const int32_t* doc_begin_h,
                            const int32_t* doc_end_h, const int32_t* budget_h, tg_dtype dtype,
                            const tg_gather_tensor* tensors, int32_t n_tensors, int32_t head_dim,
                            double rope_theta, const float* z, float* logsig_out,
                            tg_stream_t stream) {
  if (dtype != TG_BF16 && dtype != TG_FP32) return set_error(TG_ERR_DTYPE, "dtype %d", dtype);
  PromptTable t;
  tg_status r =
      build_table(batch, cu_seqlens_h, doc_begin_h, doc_end_h, budget_h, &t, nullptr, nullptr);
  if (r != TG_OK) return r;
  if (m_total != t.kept_start[batch])
    return set_error(TG_ERR_SHAPE, "m_total=%lld but the prompts keep %d rows",
                     static_cast<long long>(m_total), t.kept_start[batch]);
  if (n_tensors < 0 || n_tensors > TG_MAX_GATHER_TENSORS)
    return set_error(TG_ERR_INVALID_ARG, "n_tensors=%d", n_tensors);
  if (n_tensors > 0 && !tensors) return set_error(TG_ERR_INVALID_ARG, "tensors is null");
  const int esz = dtype == TG_BF16 ? 2 : 4;
  bool any_rope = false;
  for (int i = 0; i < n_tensors; ++i) {
    const tg_gather_tensor& g = tensors[i];
    if (g.row_elems <= 0 || g.rope_heads < 0)
      return set_error(TG_ERR_INVALID_ARG, "tensor %d: row_elems=%d rope_heads=%d", i,
                       g.row_elems, g.rope_heads);
    if (m_total > 0 && (!g.src || !g.dst))
      return set_error(TG_ERR_INVALID_ARG, "tensor %d: null pointer", i);
    if (!aligned16(g.src) || !aligned16(g.dst) || (g.row_elems * esz) % 16 != 0)
      return set_error(TG_ERR_ALIGNMENT, "tensor %d: rows must be 16-byte aligned", i);
    if (g.rope_heads > 0) {
      any_rope = true;
      if (static_cast<int64_t>(g.rope_heads) * head_dim > g.row_elems)
        return set_error(TG_ERR_SHAPE, "tensor %d: rope_heads*head_dim exceeds the row", i);
    }
  }
  if (any_rope) {
    if (head_dim <= 0 || head_dim % 16 != 0 || head_dim > 256)
      return set_error(TG_ERR_UNSUPPORTED, "RoPE head_dim=%d (needs a multiple of 16, <=256)",
                       head_dim);
    if (!(rope_theta > 1.0)) return set_error(TG_ERR_INVALID_ARG, "rope_theta must exceed 1");
  }
  if (logsig_out && m_total > 0 && !z) return set_error(TG_ERR_INVALID_ARG, "z is null");
  if (m_total == 0) return TG_OK;
  if (!kept_idx) return set_error(TG_ERR_INVALID_ARG, "kept_idx is null");
  return launch_gather(kept_idx, m_total, t, dtype, tensors, n_tensors, head_dim, rope_theta, z,
                       logsig_out, reinterpret_cast<cudaStream_t>(stream));
}

tg_status tg_attention_workspace_bytes(tg_dtype dtype, int32_t batch, const int32_t* cu_kept_h,
                                       int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                       int32_t algo, size_t* bytes_out) {
  if (!bytes_out) return set_error(TG_ERR_INVALID_ARG, "bytes_out is null");
  *bytes_out = 0;
  if (dtype != TG_BF16 && dtype != TG_FP32) return set_error(TG_ERR_DTYPE, "dtype %d", dtype);
  PromptTable t;
  int max_len = 0;
  tg_status r = build_kept_table(batch, cu_kept_h, &t, &max_len);
  if (r != TG_OK) return r;
  if (n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads % n_kv_heads != 0)
    return set_error(TG_ERR_SHAPE, "n_q_heads=%d n_kv_heads=%d", n_q_heads, n_kv_heads);
  if (head_dim != 64 && head_dim != 128)
    return set_error(TG_ERR_UNSUPPORTED, "head_dim=%d (supported: 64, 128)", head_dim);
  if (algo < TG_ALGO_AUTO || algo > TG_ALGO_TCGEN05)
    return set_error(TG_ERR_INVALID_ARG, "algo %d", algo);
  if (dtype != TG_BF16 || algo == TG_ALGO_SIMT) return TG_OK;
  *bytes_out = attn_tc_workspace_bytes(t, n_q_heads, n_kv_heads, head_dim);
  return TG_OK;
}

tg_status tg_attention_kernel(tg_dtype dtype, int32_t batch, const int32_t* cu_kept_h,
                              int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                              int32_t algo, int32_t with_workspace, int32_t* kernel_out) {
  if (!kernel_out) return set_error(TG_ERR_INVALID_ARG, "kernel_out is null");
  size_t bytes = 0;
  tg_status r = tg_attention_workspace_bytes(dtype, batch, cu_kept_h, n_q_heads, n_kv_heads,
                                             head_dim, algo, &bytes);  // validates the arguments
  if (r != TG_OK) return r;
  if (dtype != TG_BF16 || algo == TG_ALGO_SIMT) {
    *kernel_out = TG_ATTN_SIMT;
    return TG_OK;
  }
  PromptTable t;
  int max_len = 0;
  r = build_kept_table(batch, cu_kept_h, &t, &max_len);
  if (r != TG_OK) return r;
  *kernel_out = attn_tc_kernel_choice(t, n_q_heads, n_kv_heads, head_dim, with_workspace != 0);
  return TG_OK;
}

tg_status tg_gated_attention(const void* q, const void* k, const void* v, tg_dtype dtype,
                             int32_t batch, const int32_t* cu_kept_h, int32_t n_q_heads,
                             int32_t n_kv_heads, int32_t head_dim, const float* logsig,
                             const float* gain, const float* temp, void* out, float* lse,
                             void* workspace, size_t workspace_bytes, int32_t algo,
                             tg_stream_t stream) {
  if (dtype != TG_BF16 && dtype != TG_FP32) return set_error(TG_ERR_DTYPE, "dtype %d", dtype);
  PromptTable t;
  int max_len = 0;
  tg_status r = build_kept_table(batch, cu_kept_h, &t, &max_len);
  if (r != TG_OK) return r;
  if (n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads % n_kv_heads != 0)
    return set_error(TG_ERR_SHAPE, "n_q_heads=%d n_kv_heads=%d", n_q_heads, n_kv_heads);
  if (head_dim != 64 && head_dim != 128)
    return set_error(TG_ERR_UNSUPPORTED, "head_dim=%d (supported: 64, 128)", head_dim);
  if (algo < TG_ALGO_AUTO || algo > TG_ALGO_TCGEN05)
    return set_error(TG_ERR_INVALID_ARG, "algo %d", algo);
  const int64_t M = t.kept_start[batch];
  if (M == 0) return TG_OK;
  if (!q || !k || !v || !gain || !temp || !out) return set_error(TG_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return set_error(TG_ERR_ALIGNMENT, "q/k/v/out must be 16-byte aligned");
  const bool tc_ok = dtype == TG_BF16;
  if (algo == TG_ALGO_TCGEN05 && !tc_ok)
    return set_error(TG_ERR_UNSUPPORTED, "tcgen05 attention needs bf16");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (algo == TG_ALGO_SIMT || !tc_ok)
    return launch_attn_simt(q, k, v, dtype, t, max_len, n_q_heads, n_kv_heads, head_dim, logsig,
                            gain, temp, out, lse, st);
  if (workspace && !aligned16(workspace))
    return set_error(TG_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  return launch_attn_tc(q, k, v, t, max_len, n_q_heads, n_kv_heads, head_dim, logsig, gain, temp,
                        out, lse, workspace, workspace_bytes, st);
}

tg_status tg_rmsnorm(const void* x, const void* weight, void* out, tg_dtype dtype, int64_t rows,
                     int32_t dim, float eps, tg_stream_t stream) {
  if (dtype != TG_BF16 && dtype != TG_FP32) return set_error(TG_ERR_DTYPE, "dtype %d", dtype);
  if (rows < 0 || dim <= 0) return set_error(TG_ERR_SHAPE, "rows=%lld dim=%d", static_cast<long long>(rows), dim);
  if (!(eps >= 0.0f)) return set_error(TG_ERR_INVALID_ARG, "eps must be >= 0");
  if (rows == 0) return TG_OK;
  if (!x || !weight || !out) return set_error(TG_ERR_INVALID_ARG, "null pointer");
  return launch_rmsnorm(x, weight, out, dtype, rows, dim, eps, reinterpret_cast<cudaStream_t>(stream));
}

tg_status tg_qkv_rope_emit(const void* qkv, tg_dtype dtype, int32_t batch, const int32_t* cu_seqlens_h,
                           const int32_t* cu_kept_h, const int32_t* kept_idx, int32_t n_q_heads,
                           int32_t n_kv_heads, int32_t head_dim, const void* q_norm_w,
                           const void* k_norm_w, float eps, double rope_theta, void* q_out,
                           void* k_out, void* v_out, tg_stream_t stream) {
  if (dtype != TG_BF16 && dtype != TG_FP32) return set_error(TG_ERR_DTYPE, "dtype %d", dtype);
  PromptTable t;
  int max_len = 0;
  tg_status r = build_kept_table(batch, cu_kept_h, &t, &max_len);
  if (r != TG_OK) return r;
  if (!cu_seqlens_h) return set_error(TG_ERR_INVALID_ARG, "cu_seqlens_h is null");
  if (cu_seqlens_h[0] != 0) return set_error(TG_ERR_INVALID_ARG, "cu_seqlens[0] must be 0");
  for (int b = 0; b < batch; ++b) {
    const int64_t n = static_cast<int64_t>(cu_seqlens_h[b + 1]) - cu_seqlens_h[b];
    if (n < 0) return set_error(TG_ERR_INVALID_ARG, "cu_seqlens decreases at prompt %d", b);
    if (t.kept_start[b + 1] - t.kept_start[b] > n)
      return set_error(TG_ERR_INVALID_ARG, "prompt %d keeps more rows than it has", b);
    t.start[b] = cu_seqlens_h[b];
  }
  t.start[batch] = cu_seqlens_h[batch];
  if (n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads % n_kv_heads != 0)
    return set_error(TG_ERR_SHAPE, "n_q_heads=%d n_kv_heads=%d", n_q_heads, n_kv_heads);
  if (head_dim != 64 && head_dim != 128)
    return set_error(TG_ERR_UNSUPPORTED, "head_dim=%d (supported: 64, 128)", head_dim);
  if (!(rope_theta > 1.0) || !(eps >= 0.0f)) return set_error(TG_ERR_INVALID_ARG, "rope_theta / eps");
  if (t.kept_start[batch] == 0) return TG_OK;
  if (!qkv || !kept_idx || !q_norm_w || !k_norm_w || !q_out || !k_out || !v_out)
    return set_error(TG_ERR_INVALID_ARG, "null pointer");
  return launch_qkv_emit(qkv, dtype, t, kept_idx, n_q_heads, n_kv_heads, head_dim, q_norm_w,
                         k_norm_w, eps, rope_theta, q_out, k_out, v_out,
                         reinterpret_cast<cudaStream_t>(stream));
}

tg_status tg_swiglu(const void* gate_up, void* out, tg_dtype dtype, int64_t rows, int32_t inter,
                    tg_stream_t stream) {
  if (dtype != TG_BF16 && dtype != TG_FP32) return set_error(TG_ERR_DTYPE, "dtype %d", dtype);
  if (rows < 0 || inter <= 0)
    return set_error(TG_ERR_SHAPE, "rows=%lld inter=%d", static_cast<long long>(rows), inter);
  if (rows == 0) return TG_OK;
  if (!gate_up || !out) return set_error(TG_ERR_INVALID_ARG, "null pointer");
  return launch_swiglu(gate_up, out, dtype, rows, inter, reinterpret_cast<cudaStream_t>(stream));
}

tg_status tg_gated_delta_scan(const void* q, const void* k, const void* v, tg_dtype dtype,
                              const float* log_alpha, const float* beta, int32_t batch,
                              const int32_t* cu_kept_h, int32_t n_heads, int32_t head_dim, float eps,
                              void* out, float* state_out, tg_stream_t stream) {
  if (dtype != TG_BF16 && dtype != TG_FP32) return set_error(TG_ERR_DTYPE, "dtype %d", dtype);
  PromptTable t;
  int max_len = 0;
  tg_status r = build_kept_table(batch, cu_kept_h, &t, &max_len);
  if (r != TG_OK) return r;
  if (n_heads <= 0) return set_error(TG_ERR_SHAPE, "n_heads=%d", n_heads);
  if (head_dim != 64 && head_dim != 128)
    return set_error(TG_ERR_UNSUPPORTED, "head_dim=%d (supported: 64, 128)", head_dim);
  if (!(eps >= 0.0f)) return set_error(TG_ERR_INVALID_ARG, "eps must be >= 0");
  if (static_cast<int64_t>(batch) * n_heads * (head_dim / 32) > INT32_MAX)
    return set_error(TG_ERR_UNSUPPORTED, "batch x n_heads = %lld state slices exceed one launch",
                     static_cast<long long>(batch) * n_heads);
  if (batch == 0 || (t.kept_start[batch] == 0 && !state_out)) return TG_OK;
  if (t.kept_start[batch] > 0 && (!q || !k || !v || !log_alpha || !beta || !out))
    return set_error(TG_ERR_INVALID_ARG, "null pointer");
  for (const void* ptr : {q, k, v, static_cast<const void*>(state_out)})
    if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0)
      return set_error(TG_ERR_ALIGNMENT, "q, k, v and state_out must be 16-byte aligned");
  return launch_delta_scan(q, k, v, dtype, log_alpha, beta, t, n_heads, head_dim, eps, out, state_out,
                           reinterpret_cast<cudaStream_t>(stream));
}

// Shared argument checks of the two forms of the delta-rule scan.
static tg_status check_delta_args(const void* q, const void* k, const void* v, tg_dtype dtype,
                                  const float* log_alpha, const float* beta, int32_t batch,
                                  const int32_t* cu_kept_h, int32_t n_heads, int32_t head_dim,
                                  float eps, void* out, float* state_out, PromptTable* t) {
  if (dtype != TG_BF16 && dtype != TG_FP32) return set_error(TG_ERR_DTYPE, "dtype %d", dtype);
  int max_len = 0;
  tg_status r = build_kept_table(batch, cu_kept_h, t, &max_len);
  if (r != TG_OK) return r;
  if (n_heads <= 0) return set_error(TG_ERR_SHAPE, "n_heads=%d", n_heads);
  if (head_dim != 64 && head_dim != 128)
    return set_error(TG_ERR_UNSUPPORTED, "head_dim=%d (supported: 64, 128)", head_dim);
  if (!(eps >= 0.0f)) return set_error(TG_ERR_INVALID_ARG, "eps must be >= 0");
  if (t->kept_start[batch] > 0 && (!q || !k || !v || !log_alpha || !beta || !out))
    return set_error(TG_ERR_INVALID_ARG, "null pointer");
  for (const void* ptr : {q, k, v, static_cast<const void*>(state_out)})
    if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0)
      return set_error(TG_ERR_ALIGNMENT, "q, k, v and state_out must be 16-byte aligned");
  return TG_OK;
}

tg_status tg_delta_scan_workspace_bytes(int32_t batch, const int32_t* cu_kept_h, int32_t n_heads,
                                        int32_t head_dim, size_t* bytes_out) {
  if (!bytes_out) return set_error(TG_ERR_INVALID_ARG, "bytes_out is NULL");
  *bytes_out = 0;
  PromptTable t;
  int max_len = 0;
  tg_status r = build_kept_table(batch, cu_kept_h, &t, &max_len);
  if (r != TG_OK) return r;
  if (n_heads <= 0) return set_error(TG_ERR_SHAPE, "n_heads=%d", n_heads);
  if (head_dim != 64 && head_dim != 128)
    return set_error(TG_ERR_UNSUPPORTED, "head_dim=%d (supported: 64, 128)", head_dim);
  *bytes_out = delta_chunked_workspace_bytes(t, n_heads, head_dim);
  return TG_OK;
}

tg_status tg_gated_delta_scan_chunked(const void* q, const void* k, const void* v, tg_dtype dtype,
                                      const float* log_alpha, const float* beta, int32_t batch,
                                      const int32_t* cu_kept_h, int32_t n_heads, int32_t head_dim,
                                      float eps, void* out, float* state_out, void* workspace,
                                      size_t workspace_bytes, tg_stream_t stream) {
  PromptTable t;
  tg_status r = check_delta_args(q, k, v, dtype, log_alpha, beta, batch, cu_kept_h, n_heads,
                                 head_dim, eps, out, state_out, &t);
  if (r != TG_OK) return r;
  if (static_cast<int64_t>(batch) * n_heads > 65535)
    return set_error(TG_ERR_UNSUPPORTED, "n_heads=%d exceeds one launch", n_heads);
  if (batch == 0 || (t.kept_start[batch] == 0 && !state_out)) return TG_OK;
  const size_t need = delta_chunked_workspace_bytes(t, n_heads, head_dim);
  if (need > 0 && (!workspace || workspace_bytes < need))
    return set_error(TG_ERR_WORKSPACE, "delta-scan workspace: %zu bytes given, %zu needed",
                     workspace ? workspace_bytes : 0, need);
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
    return set_error(TG_ERR_ALIGNMENT, "the delta-scan workspace must be 256-byte aligned");
  return launch_delta_chunked(q, k, v, dtype, log_alpha, beta, t, n_heads, head_dim, eps, out,
                              state_out, workspace, reinterpret_cast<cudaStream_t>(stream));
}

tg_status tg_attention_backward_workspace_bytes(int32_t batch, const int32_t* cu_kept_h,
                                                int32_t n_q_heads, size_t* bytes_out) {
  if (!bytes_out) return set_error(TG_ERR_INVALID_ARG, "bytes_out is NULL");
  PromptTable t;
  int max_len = 0;
  tg_status r = build_kept_table(batch, cu_kept_h, &t, &max_len);
  if (r != TG_OK) return r;
  if (n_q_heads <= 0) return set_error(TG_ERR_SHAPE, "n_q_heads=%d", n_q_heads);
  *bytes_out = attn_bwd_workspace_bytes(t.kept_start[batch], n_q_heads);
  return TG_OK;
}

tg_status tg_gated_attention_backward(const void* q, const void* k, const void* v, tg_dtype dtype,
                                      int32_t batch, const int32_t* cu_kept_h, int32_t n_q_heads,
                                      int32_t n_kv_heads, int32_t head_dim, const float* logsig,
                                      const float* gain, const float* temp, const void* out,
                                      const float* lse, const void* dout, float* d_logsig,
                                      float* d_z_kept, float* d_gain, float* d_temp,
                                      void* workspace, size_t workspace_bytes, int32_t algo,
                                      tg_stream_t stream) {
  if (dtype != TG_BF16 && dtype != TG_FP32) return set_error(TG_ERR_DTYPE, "dtype %d", dtype);
  PromptTable t;
  int max_len = 0;
  tg_status r = build_kept_table(batch, cu_kept_h, &t, &max_len);
  if (r != TG_OK) return r;
  if (n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads % n_kv_heads != 0)
    return set_error(TG_ERR_SHAPE, "n_q_heads=%d n_kv_heads=%d", n_q_heads, n_kv_heads);
  if (head_dim != 64 && head_dim != 128)
    return set_error(TG_ERR_UNSUPPORTED, "head_dim=%d (supported: 64, 128)", head_dim);
  if (algo < TG_ALGO_AUTO || algo > TG_ALGO_TCGEN05)
    return set_error(TG_ERR_INVALID_ARG, "algo %d", algo);
  const int64_t M = t.kept_start[batch];
  if (M == 0) return TG_OK;
  if (!q || !k || !v || !logsig || !gain || !temp || !out || !lse || !dout || !d_logsig ||
      !d_z_kept || !d_gain || !d_temp || !workspace)
    return set_error(TG_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned16(workspace))
    return set_error(TG_ERR_ALIGNMENT, "q/k/v/out/dout/workspace must be 16-byte aligned");
  const size_t need = attn_bwd_workspace_bytes(M, n_q_heads);
  if (workspace_bytes < need)
    return set_error(TG_ERR_WORKSPACE, "attention backward workspace: %zu bytes given, %zu needed",
                     workspace_bytes, need);
  if (algo == TG_ALGO_TCGEN05 && dtype != TG_BF16)
    return set_error(TG_ERR_UNSUPPORTED, "tcgen05 attention backward needs bf16");
  return launch_attn_bwd(q, k, v, out, dout, dtype, t, n_q_heads, n_kv_heads, head_dim, logsig,
                         gain, temp, lse, d_logsig, d_z_kept, d_gain, d_temp, workspace, algo,
                         reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
