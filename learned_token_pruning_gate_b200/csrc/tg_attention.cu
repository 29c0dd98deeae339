// Token-gated causal GQA attention over the kept rows (TokenGate: each kept
// token's gate score is added to the attention logits above the gate as a
// bias scaled by a per-head learned gain -- the Mixture-of-Experts router
// trick -- and a per-head learned temperature corrects for each query seeing
// fewer keys):
//     logit_ij = q_i.k_j / (sqrt(d) tau_h) + g_h l_j,   j <= i in the prompt
// The kernel works in the log2 domain: t = s * log2(e)/(sqrt(d) tau_h) +
// g_h log2(e) l_j, so the per-key bias and the per-head temperature fold into
// one FMA per logit.
//
// attn_simt_kernel is the CUDA-core path (fp32, and any bf16 shape): a block of
// 8 warps owns 8 consecutive query rows of one head, stages 32-key K/V tiles in
// shared memory, and each warp runs an exact online softmax over its row.  The
// tensor-core path lives in tg_attention_tc.cu.
#include "tg_internal.cuh"

namespace tg {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct AttnParams {
  int32_t kept_start[kMaxBatch + 1];
  int32_t order[kMaxBatch];  // prompts by kept length, longest first
  const float* logsig;
  const float* gain;
  const float* temp;
  void* out;
  float* lse;
  uint32_t* status;
  int32_t batch;
  int32_t m_total;
  int32_t hq;
  int32_t hkv;
};

template <typename T>
__device__ __forceinline__ float ld_f(const T* p);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ int prompt_of_row(const int32_t* ks, int batch, int64_t i) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (ks[mid] <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ---- CUDA-core path ---------------------------------------------------------
constexpr int kSimtWarps = 8;
constexpr int kSimtKeys = 32;

template <typename T, int DH>
__global__ void __launch_bounds__(kSimtWarps * 32)
    attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     const __grid_constant__ AttnParams p) {
  constexpr int PL = DH / 32;  // elements per lane
  __shared__ float s_k[kSimtKeys][DH];
  __shared__ float s_v[kSimtKeys][DH];
  __shared__ float s_b[kSimtKeys];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = blockIdx.y;
  const int hk = h / (p.hq / p.hkv);
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kSimtWarps;
  const int64_t i = row0 + warp;
  const bool active = i < p.m_total;
  const int64_t last = min(row0 + kSimtWarps, static_cast<int64_t>(p.m_total)) - 1;
  const int b0 = prompt_of_row(p.kept_start, p.batch, row0);
  const int64_t kmin = p.kept_start[b0];
  const int64_t my_start = active ? p.kept_start[prompt_of_row(p.kept_start, p.batch, i)] : 0;

  const float scale = kLog2e / (sqrtf(static_cast<float>(DH)) * __ldg(p.temp + h));
  const float gl = __ldg(p.gain + h) * kLog2e;
  float qr[PL], o[PL];
#pragma unroll
  for (int e = 0; e < PL; ++e) {
    qr[e] = active ? ld_f(q + (i * p.hq + h) * DH + lane + 32 * e) : 0.0f;
    o[e] = 0.0f;
  }
  float m = -INFINITY, l = 0.0f;

  for (int64_t kb = kmin; kb <= last; kb += kSimtKeys) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < kSimtKeys * DH; idx += blockDim.x) {
      const int kr = idx / DH, c = idx - kr * DH;
      const int64_t j = kb + kr;
      const bool ok = j <= last;
      s_k[kr][c] = ok ? ld_f(k + (j * p.hkv + hk) * DH + c) : 0.0f;
      s_v[kr][c] = ok ? ld_f(v + (j * p.hkv + hk) * DH + c) : 0.0f;
    }
    for (int kr = threadIdx.x; kr < kSimtKeys; kr += blockDim.x) {
      const int64_t j = kb + kr;
      s_b[kr] = (p.logsig && j <= last) ? gl * __ldg(p.logsig + j) : 0.0f;
    }
    __syncthreads();
    if (!active) continue;
    const int64_t j_lo = max(kb, my_start);
    const int64_t j_hi = min(kb + kSimtKeys - 1, i);
    for (int64_t j = j_lo; j <= j_hi; ++j) {
      const int kr = static_cast<int>(j - kb);
      float dot = 0.0f;
#pragma unroll
      for (int e = 0; e < PL; ++e) dot = fmaf(qr[e], s_k[kr][lane + 32 * e], dot);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      const float t = fmaf(dot, scale, s_b[kr]);
      const float m_new = fmaxf(m, t);
      const float corr = exp2f(m - m_new);
      const float pj = exp2f(t - m_new);
      l = fmaf(l, corr, pj);
#pragma unroll
      for (int e = 0; e < PL; ++e) o[e] = fmaf(o[e], corr, pj * s_v[kr][lane + 32 * e]);
      m = m_new;
    }
  }
  if (!active) return;
  const float inv = 1.0f / l;
  T* out = static_cast<T*>(p.out);
#pragma unroll
  for (int e = 0; e < PL; ++e) out[(i * p.hq + h) * DH + lane + 32 * e] = from_f<T>(o[e] * inv);
  if (p.lse && lane == 0) p.lse[static_cast<int64_t>(h) * p.m_total + i] = (m + log2f(l)) * kLn2;
}

void fill_params(AttnParams* a, const PromptTable& pt) {
  memset(a, 0, sizeof(*a));
  a->batch = pt.batch;
  for (int b = 0; b <= pt.batch; ++b) a->kept_start[b] = pt.kept_start[b];
  // longest prompt first (stable)
  for (int b = 0; b < pt.batch; ++b) a->order[b] = b;
  for (int i = 1; i < pt.batch; ++i) {
    int x = a->order[i], j = i - 1;
    const int lx = pt.kept_start[x + 1] - pt.kept_start[x];
    while (j >= 0 && pt.kept_start[a->order[j] + 1] - pt.kept_start[a->order[j]] < lx) {
      a->order[j + 1] = a->order[j];
      --j;
    }
    a->order[j + 1] = x;
  }
  a->m_total = pt.kept_start[pt.batch];
}

}  // namespace

tg_status launch_attn_simt(const void* q, const void* k, const void* v, tg_dtype dt,
                           const PromptTable& pt, int max_len, int hq, int hkv, int dh,
                           const float* logsig, const float* gain, const float* temp, void* out,
                           float* lse, cudaStream_t st) {
  (void)max_len;
  AttnParams a;
  fill_params(&a, pt);
  a.logsig = logsig;
  a.gain = gain;
  a.temp = temp;
  a.out = out;
  a.lse = lse;
  a.hq = hq;
  a.hkv = hkv;
  dim3 grid(static_cast<unsigned>((a.m_total + kSimtWarps - 1) / kSimtWarps), hq);
  const int th = kSimtWarps * 32;
  if (dt == TG_BF16) {
    auto* qq = static_cast<const __nv_bfloat16*>(q);
    auto* kk = static_cast<const __nv_bfloat16*>(k);
    auto* vv = static_cast<const __nv_bfloat16*>(v);
    if (dh == 64) attn_simt_kernel<__nv_bfloat16, 64><<<grid, th, 0, st>>>(qq, kk, vv, a);
    else attn_simt_kernel<__nv_bfloat16, 128><<<grid, th, 0, st>>>(qq, kk, vv, a);
  } else {
    auto* qq = static_cast<const float*>(q);
    auto* kk = static_cast<const float*>(k);
    auto* vv = static_cast<const float*>(v);
    if (dh == 64) attn_simt_kernel<float, 64><<<grid, th, 0, st>>>(qq, kk, vv, a);
    else attn_simt_kernel<float, 128><<<grid, th, 0, st>>>(qq, kk, vv, a);
  }
  return cuda_check(cudaGetLastError(), "attn_simt launch");
}


}  // namespace tg
