// Gated attention without any device allocation by the caller.
//
// tg_gated_attention can split the key range of long query tiles when the batch
// is too small to fill the GPU, and then needs scratch memory for the partial
// results; normally the caller passes it as a workspace.  Some callers cannot
// allocate device memory at all: a serving process whose allocator reserved the
// whole device up front (so a new cudaMalloc would fail or fragment its pool),
// or a host that must not allocate between the setup of a CUDA graph and its
// capture.  For them tg_gated_attention_noalloc takes its scratch from one
// fixed array compiled into the library.
//
// The array lives in device memory of every GPU whose context loads the
// library, until the process exits (kScratchBytes per GPU).  Its device address
// is looked up with cudaGetSymbolAddress (a runtime call that allocates
// nothing) on a device's first call, and again when that device's current
// context has changed -- after a cudaDeviceReset the module is loaded anew in a
// new context, so an address kept from before would point at freed memory.
// Make the first call on a device before any stream capture.  A batch whose
// split plan needs more than the array holds runs the unsplit plan instead,
// which needs no scratch.  All calls share the array, so two calls that run on
// the GPU at the same time -- on different streams, or from different threads
// -- race on it; order them on one stream.  Each call clears the array's
// arrival counters on its stream before the kernel runs (the attention launch
// does this for any workspace); nothing else must start at zero.
#include "tg_internal.cuh"

namespace tg {
namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;  // 32 MiB

static __device__ __align__(256) uint8_t g_attn_scratch[kScratchBytes];

// Device address of the array in the current context (nullptr on failure).
void* scratch_address() {
  static SymbolAddressCache cache;
  return cache.get(reinterpret_cast<const void*>(&g_attn_scratch));
}

}  // namespace
}  // namespace tg

using namespace tg;

extern "C" {

tg_status tg_gated_attention_noalloc(const void* q, const void* k, const void* v, tg_dtype dtype,
                                     int32_t batch, const int32_t* cu_kept_h, int32_t n_q_heads,
                                     int32_t n_kv_heads, int32_t head_dim, const float* logsig,
                                     const float* gain, const float* temp, void* out, float* lse,
                                     int32_t algo, tg_stream_t stream) {
  size_t need = 0;
  tg_status r = tg_attention_workspace_bytes(dtype, batch, cu_kept_h, n_q_heads, n_kv_heads,
                                             head_dim, algo, &need);
  if (r != TG_OK) return r;
  if (need == 0 || need > kScratchBytes)  // no split, or a split the array cannot hold
    return tg_gated_attention(q, k, v, dtype, batch, cu_kept_h, n_q_heads, n_kv_heads, head_dim,
                              logsig, gain, temp, out, lse, nullptr, 0, algo, stream);
  void* scratch = scratch_address();
  if (!scratch) return set_error(TG_ERR_CUDA, "cannot resolve the attention scratch array");
  return tg_gated_attention(q, k, v, dtype, batch, cu_kept_h, n_q_heads, n_kv_heads, head_dim,
                            logsig, gain, temp, out, lse, scratch, kScratchBytes, algo, stream);
}

}  // extern "C"
