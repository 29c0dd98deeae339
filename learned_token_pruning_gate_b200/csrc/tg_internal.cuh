// Internal definitions shared by the libtokengate kernels: the prompt table
// passed by value to kernels, the device status word, and thin wrappers over
// the sm_100a PTX used by the tensor-core kernels (mbarrier, TMA, tcgen05).
#pragma once

#include <cuda.h>  // CUtensorMap (type only; the driver entry point is fetched at run time)
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "../../include/tokengate.h"

namespace tg {

constexpr int kMaxBatch = TG_MAX_BATCH;

// Per-prompt description, validated on the host and passed by value.
struct PromptTable {
  int32_t batch;
  int32_t start[kMaxBatch + 1];       // cu_seqlens
  int32_t doc_begin[kMaxBatch];       // relative to the prompt start
  int32_t doc_end[kMaxBatch];
  int32_t k_keep[kMaxBatch];          // min(budget, n_doc)
  int32_t kept_start[kMaxBatch + 1];  // cu_kept
};

// First-pass radix histograms handed from the gate to the top-K select (the
// top-K workspace).  Per prompt: kHistBins counts of the top 11 bits of the
// order key (below) of its document tokens' scores, then a tag {magic, total
// tokens, score pointer lo, hi} naming the scores they were counted from, and a
// counter of the selections that have read them (word 4).
constexpr int kHistBins = 2048;
constexpr int kHistStride = 2112;  // words per prompt: 8448 bytes, a multiple of 256
constexpr uint32_t kHistMagic = 0x7A6E5B1Fu;

// What a gate launch needs to add its scores to the top-K workspace.
struct GateHist {
  uint32_t* hist;              // [batch][kHistStride] or null (no histogram)
  const float* z;              // the scores the gate writes (for the tag)
  int32_t n;                   // total tokens (for the tag)
  int32_t batch;
  int32_t start[kMaxBatch + 1];  // cu_seqlens
  int32_t doc_lo[kMaxBatch];     // absolute document span [doc_lo, doc_hi) of each prompt
  int32_t doc_hi[kMaxBatch];
};

// Bits of the device status word.
enum : uint32_t {
  kDevTimeoutGate = 1u << 0,
  kDevTimeoutAttn = 1u << 1,
  kDevTopkOverflow = 1u << 2,   // selection produced more rows than M_b (skipped)
  kDevGatherIndex = 1u << 3,    // a kept index outside the prompt batch (row skipped)
  kDevTimeoutGather = 1u << 4,
  kDevTimeoutDelta = 1u << 5,   // a chunk load of the chunked delta-rule scan did not land
};

// Host side: error reporting and the device status word.
tg_status set_error(tg_status s, const char* fmt, ...);
tg_status cuda_check(cudaError_t e, const char* what);
uint32_t* device_status_word();  // device address for the current device (nullptr on failure)
uint64_t current_context_id();    // unique id of the current CUDA context, 0 if unknown

// Per-device cache of a __device__ symbol's address, looked up with
// cudaGetSymbolAddress (a runtime call that allocates nothing) the first time
// a device asks and again whenever that device's current context has changed
// (after a cudaDeviceReset the module lives in a new context).
class SymbolAddressCache {
 public:
  void* get(const void* symbol);

 private:
  static constexpr int kDevices = 64;
  std::mutex mu_;
  void* addr_[kDevices] = {};
  uint64_t ctx_[kDevices] = {};
};
int num_sms();

// Kernel launchers (each validates nothing: the C ABI layer has done it).
// The gate launchers add the first-pass histograms when gh.hist is non-null.
tg_status launch_gate_simt(const void* h, tg_dtype dt, int64_t n, int d, const void* W1,
                           const float* b1, int dg, const float* w2, float b2, float* z,
                           const GateHist& gh, cudaStream_t st);
tg_status launch_gate_tc(const void* h, int64_t n, int d, const void* W1, const float* b1, int dg,
                         const float* w2, float b2, float* z, const GateHist& gh,
                         cudaStream_t st);
// hist: the top-K workspace of a single-budget score selection, or null.
tg_status launch_topk(const float* z, const uint32_t* keys, const PromptTable* tables,
                      int n_budgets, int max_len, int32_t* const* kept_idx,
                      int32_t* const* cu_kept, uint32_t* hist, cudaStream_t st);
tg_status launch_gather(const int32_t* kept_idx, int64_t m_total, const PromptTable& pt,
                        tg_dtype dt, const tg_gather_tensor* tensors, int n_tensors, int head_dim,
                        double theta, const float* z, float* logsig, cudaStream_t st);
tg_status launch_attn_simt(const void* q, const void* k, const void* v, tg_dtype dt,
                           const PromptTable& pt, int max_len, int hq, int hkv, int dh,
                           const float* logsig, const float* gain, const float* temp, void* out,
                           float* lse, cudaStream_t st);
tg_status launch_attn_tc(const void* q, const void* k, const void* v, const PromptTable& pt,
                         int max_len, int hq, int hkv, int dh, const float* logsig,
                         const float* gain, const float* temp, void* out, float* lse,
                         void* workspace, size_t workspace_bytes, cudaStream_t st);
// Backward of the gated attention (log-gates, gains, temperatures); workspace of
// attn_bwd_workspace_bytes (D per row and head, per-head accumulators).
tg_status launch_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                          const void* dout, tg_dtype dt, const PromptTable& pt, int hq, int hkv,
                          int dh, const float* logsig, const float* gain, const float* temp,
                          const float* lse, float* d_logsig, float* d_z_kept, float* d_gain,
                          float* d_temp, void* workspace, int algo, cudaStream_t st);
size_t attn_bwd_workspace_bytes(int64_t m_total, int hq);
// Element-wise steps of the gated upper-layer stack.
tg_status launch_rmsnorm(const void* x, const void* w, void* y, tg_dtype dt, int64_t rows, int dim,
                         float eps, cudaStream_t st);
tg_status launch_qkv_emit(const void* qkv, tg_dtype dt, const PromptTable& pt, const int32_t* kept_idx,
                          int hq, int hkv, int dh, const void* w_qn, const void* w_kn, float eps,
                          double theta, void* q_out, void* k_out, void* v_out, cudaStream_t st);
tg_status launch_delta_scan(const void* q, const void* k, const void* v, tg_dtype dt,
                            const float* log_alpha, const float* beta, const PromptTable& pt, int heads,
                            int head_dim, float eps, void* out, float* state, cudaStream_t st);
tg_status launch_swiglu(const void* gu, void* h, tg_dtype dt, int64_t rows, int inter,
                        cudaStream_t st);
// Chunked form of the gated delta rule (workspace of delta_chunked_workspace_bytes).
size_t delta_chunked_workspace_bytes(const PromptTable& pt, int heads, int head_dim);
tg_status launch_delta_chunked(const void* q, const void* k, const void* v, tg_dtype dt,
                               const float* log_alpha, const float* beta, const PromptTable& pt,
                               int heads, int head_dim, float eps, void* out, float* state,
                               void* workspace, cudaStream_t st);
// Workspace the tensor-core attention uses to split long items on this device (0 = none).
size_t attn_tc_workspace_bytes(const PromptTable& pt, int hq, int hkv, int dh);
// The tg_attn_kernel the tensor-core attention launches for this batch.
int attn_tc_kernel_choice(const PromptTable& pt, int hq, int hkv, int dh, bool with_workspace);

// Tensor map encoding through the driver entry point (no libcuda link).
bool encode_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                         uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_outer);

#if defined(__CUDACC__)

// Order-preserving key of an fp32 score: larger score -> larger key; -0.0 maps
// to +0.0; NaN maps to 0, below every number (-inf maps to 0x007FFFFF).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0u;
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Adds one score to its prompt's first-pass histogram when the row is a
// document token.  The warp's converged lanes call it together (active: the
// lane holds a row); lanes that hit the same bin add once, together.
__device__ __forceinline__ void gate_hist_add(const GateHist& gh, int row, float z, bool active) {
  uint32_t idx = 0xFFFFFFFFu;
  if (active) {
    int lo = 0, hi = gh.batch - 1;  // the prompt: last b with start[b] <= row
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (gh.start[mid] <= row) lo = mid;
      else hi = mid - 1;
    }
    if (row >= gh.doc_lo[lo] && row < gh.doc_hi[lo])
      idx = static_cast<uint32_t>(lo) * kHistStride + (order_key(z) >> 21);
  }
  const unsigned mask = __ballot_sync(__activemask(), idx != 0xFFFFFFFFu);
  if (idx != 0xFFFFFFFFu) {
    const unsigned peers = __match_any_sync(mask, idx);
    if (static_cast<int>(threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(gh.hist + idx, __popc(peers));
  }
}

// The tag of every prompt's histogram (written once per gate launch, by the
// threads [first, first + stride) of block 0).
__device__ __forceinline__ void gate_hist_tags(const GateHist& gh, int first, int stride) {
  if (!gh.hist || blockIdx.x != 0) return;
  const uint64_t zp = reinterpret_cast<uint64_t>(gh.z);
  for (int b = static_cast<int>(threadIdx.x) - first; b >= 0 && b < gh.batch; b += stride) {
    uint32_t* tag = gh.hist + static_cast<size_t>(b) * kHistStride + kHistBins;
    tag[0] = kHistMagic;
    tag[1] = static_cast<uint32_t>(gh.n);
    tag[2] = static_cast<uint32_t>(zp);
    tag[3] = static_cast<uint32_t>(zp >> 32);
  }
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---- mbarrier -------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
// Raise the barrier's expected transaction bytes without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// Bounded wait for the phase with the given parity.  On expiry (or when another
// role already gave up) it records `code` in the status word, raises the CTA's
// abort flag and returns false; the caller then leaves its loop.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status, uint32_t code) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        atomicOr(status, code);
        return false;
      }
    }
  }
}

// ---- TMA ------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x,
                                            int32_t y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap* map, int32_t x,
                                                 int32_t y, uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- tcgen05 ----------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D(tmem) (+)= A(smem desc) * B(smem desc)
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D(tmem) (+)= A(tmem) * B(smem desc)
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every tcgen05 operation issued so far by this thread completes.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns; thread t of the warp gets lane (base lane + t).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
// Wait for this thread's outstanding tcgen05.ld; the empty asm statements then
// tie the loaded registers to a point after the wait so no use is hoisted above it.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(r[i]));
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand tile whose
// 8-row x 128-byte swizzle atoms are stacked every `sbo` bytes; `lbo` is the
// byte distance between 64-element column blocks (MN-major operands only).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;  // descriptor version for sm_100
  d |= 2ull << 61;  // 128-byte swizzle
  return d;
}

// Shared-memory matrix descriptor for a K-major operand tile without swizzle:
// element (row r, k) sits at saddr + (k / 8) * lbo + (r / 8) * sbo + (r % 8) * 16 +
// (k % 8) * 2, i.e. 8-row x 16-byte core matrices, `lbo` bytes apart along K and
// `sbo` bytes apart along the rows.
__device__ __forceinline__ uint64_t nosw_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;  // descriptor version for sm_100; layout type 0 = no swizzle
  return d;
}

// Instruction descriptor: kind::f16 with bf16 A/B, fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major,
                                                      bool b_mn_major) {
  return (1u << 4)                                   // D format f32
         | (1u << 7)                                 // A format bf16
         | (1u << 10)                                // B format bf16
         | (static_cast<uint32_t>(a_mn_major) << 15)  // A major
         | (static_cast<uint32_t>(b_mn_major) << 16)  // B major
         | (static_cast<uint32_t>(N >> 3) << 17)      // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);     // M / 16
}

// ---- bulk (non-tensor) copies ---------------------------------------------------
// global -> shared, completion counted on an mbarrier of this CTA (16-byte aligned,
// size a multiple of 16)
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}
// shared -> global, tracked by the issuing thread's bulk async-groups
__device__ __forceinline__ void bulk_s2g(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                   reinterpret_cast<uint64_t>(dst)),
               "r"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// wait until at most N committed groups still read their shared-memory source
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// make generic-proxy shared-memory writes visible to the async proxy (bulk copies)
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- CTA pairs (tcgen05 cta_group::2) ----------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory offset in CTA `rank`
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(saddr), "r"(rank));
  return d;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// Arrival on a barrier that may live in the peer CTA of the pair.  Every use
// hands the tensor core of the pair something this thread produced on its own
// SM -- TMEM columns (ordered by tcgen05.wait and the tcgen05 fences) or
// shared-memory operands (ordered by fence.proxy.async) -- so the arrival keeps
// the default CTA-scope release.  A cluster-scope release also waits for the
// thread's outstanding global memory operations (prefetch loads, output
// stores), which put about half a microsecond on the softmax critical path.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA load whose completion is counted on a barrier that may live in the peer CTA
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int32_t x,
                                                 int32_t y, uint32_t bar_cluster,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// D(tmem, both CTAs) (+)= A(smem, both CTAs) * B(smem, half in each CTA)
__device__ __forceinline__ void umma_ss_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D(tmem, both CTAs) (+)= A(tmem, both CTAs) * B(smem, half in each CTA)
__device__ __forceinline__ void umma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// One commit that arrives on the barrier at this shared-memory offset in both
// CTAs of the pair (CTA mask 0b11) once the pair's prior tcgen05 ops complete:
// half the commits of one per CTA, each of which costs the tensor pipe ~64 cycles.
__device__ __forceinline__ void umma_commit_pair_both(uint32_t bar_local) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar_local),
      "h"(static_cast<uint16_t>(0x3))
      : "memory");
}
// Arrive on a (possibly peer) barrier once the pair's prior tcgen05 ops complete.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar_cluster) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          bar_cluster)
      : "memory");
}

__device__ __forceinline__ void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// Named barrier that also ORs a predicate over the participating threads, so a
// group leaves a loop together when any of its threads gave up waiting.
__device__ __forceinline__ bool named_barrier_or(int id, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}
// Bounded wait that ignores the abort flag: used only on the way out after an
// abort, so copies or MMAs already issued land before the CTA exits.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity) && global_timer_ns() - t0 < kWaitLimitNs) {
  }
}

// Programmatic dependent launch.  A kernel launched with launch_pdl() may start
// while the previous kernel in its stream is still running.  grid_dep_wait()
// returns once that kernel has completed and its writes are visible (at once
// when the kernel was launched without the attribute); a kernel reads nothing
// that earlier work in the stream writes, and writes nothing, before it.
// grid_dep_launch() lets the next kernel of the stream start; every kernel
// calls it only after its own grid_dep_wait(), so when a kernel starts, all
// work before its predecessor is complete.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Host: launch with programmatic dependent launch allowed (see grid_dep_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

#endif  // __CUDACC__

}  // namespace tg
