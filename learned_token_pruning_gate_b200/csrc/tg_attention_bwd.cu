// Backward of the token-gated attention with respect to the gate's log-gates,
// the per-head gains and temperatures: the path that trains the gate (TokenGate:
// the gate's score enters the attention logits above the gate as a bias scaled
// by a per-head gain, the "MoE router trick", so the attention's loss reaches the
// scorer through it).
//
// For a loss L with dout = dL/dout, per prompt, head h and query row i (keys
// j <= i of the prompt):
//   P_ij = exp(logit_ij - LSE_i),  logit_ij = q_i.k_j / (sqrt(d) tau_h) + g_h l_j
//   dP_ij = dout_i . v_j,  D_i = dout_i . out_i,  dlogit_ij = P_ij (dP_ij - D_i)
//   dL/dl_j += g_h dlogit_ij,  dL/dg_h += l_j dlogit_ij,
//   dL/dtau_h += dlogit_ij * (-(q_i.k_j) / (sqrt(d) tau_h^2))
// and, for a kept row whose log-gate is l = log sigmoid(z), dL/dz = dL/dl (1 - e^l)
// (question rows have l fixed at 0, so 1 - e^l = 0 gives them none).
//
// Launches: bwd_prep_kernel (D_i for every row and head into the workspace, the
// outputs cleared), the main kernel, bwd_finish_kernel (dL/dz, and dL/dtau from
// its accumulated parts on the tensor-core path).
#include <cmath>

#include "tg_internal.cuh"

namespace tg {
namespace {

constexpr float kLn2f = 0.6931471805599453f;

struct BwdParams {
  int32_t kept_start[kMaxBatch + 1];
  int32_t batch;
  int32_t m_total;
  int32_t hq;
  int32_t group;  // query heads per KV head
  const float* logsig;
  const float* gain;
  const float* temp;
  const float* lse;  // [hq, m_total], natural log
  float* D;          // [hq, m_total] (workspace)
  float* acc;        // [2 * hq] (workspace): tensor-core path, sum of dlogit * log2 P per head
  float* d_logsig;
  float* d_z_kept;
  float* d_gain;
  float* d_temp;
};

template <typename T>
__device__ __forceinline__ float ld_f(const T* p);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ int prompt_of_row(const BwdParams& p, int64_t i) {
  int lo = 0, hi = p.batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.kept_start[mid] <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// D_i = dout_i . out_i for every (row, head); outputs and accumulators cleared.
template <typename T, int DH>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const T* __restrict__ out,
                                                       const T* __restrict__ dout,
                                                       const __grid_constant__ BwdParams p) {
  grid_dep_wait();
  grid_dep_launch();
  constexpr int E = DH / 32;
  const int lane = threadIdx.x & 31;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t w0 = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t total = static_cast<int64_t>(p.m_total) * p.hq;
  for (int64_t w = w0; w < total; w += nw) {
    const int64_t i = w / p.hq;
    const int h = static_cast<int>(w - i * p.hq);
    const T* o = out + (i * p.hq + h) * DH + lane * E;
    const T* d = dout + (i * p.hq + h) * DH + lane * E;
    float s = 0.0f;
#pragma unroll
    for (int e = 0; e < E; ++e) s = fmaf(ld_f(o + e), ld_f(d + e), s);
    s = warp_sum(s);
    if (lane == 0) p.D[static_cast<int64_t>(h) * p.m_total + i] = s;
  }
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nt = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t j = t0; j < p.m_total; j += nt) p.d_logsig[j] = 0.0f;
  for (int64_t h = t0; h < p.hq; h += nt) {
    p.d_gain[h] = 0.0f;
    p.d_temp[h] = 0.0f;
    p.acc[h] = 0.0f;
    p.acc[p.hq + h] = 0.0f;
  }
}

// CUDA-core path: one warp per (query row, head) walks the row's keys.
template <typename T, int DH>
__global__ void __launch_bounds__(256) bwd_simt_kernel(const T* __restrict__ q,
                                                       const T* __restrict__ k,
                                                       const T* __restrict__ v,
                                                       const T* __restrict__ dout,
                                                       const __grid_constant__ BwdParams p) {
  grid_dep_wait();
  grid_dep_launch();
  constexpr int E = DH / 32;
  const int lane = threadIdx.x & 31;
  const int hkv = p.hq / p.group;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t w0 = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t total = static_cast<int64_t>(p.m_total) * p.hq;
  for (int64_t w = w0; w < total; w += nw) {
    const int64_t i = w / p.hq;
    const int h = static_cast<int>(w - i * p.hq);
    const int hk = h / p.group;
    const int64_t j0 = p.kept_start[prompt_of_row(p, i)];
    const float tau = __ldg(p.temp + h), g = __ldg(p.gain + h);
    const float c = 1.0f / (sqrtf(static_cast<float>(DH)) * tau);
    const float lse = __ldg(p.lse + static_cast<int64_t>(h) * p.m_total + i);
    const float Di = p.D[static_cast<int64_t>(h) * p.m_total + i];
    float qi[E], di[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      qi[e] = ld_f(q + (i * p.hq + h) * DH + lane * E + e);
      di[e] = ld_f(dout + (i * p.hq + h) * DH + lane * E + e);
    }
    float dg = 0.0f, dt = 0.0f;
    for (int64_t j = j0; j <= i; ++j) {
      const T* kj = k + (j * hkv + hk) * DH + lane * E;
      const T* vj = v + (j * hkv + hk) * DH + lane * E;
      float s = 0.0f, dp = 0.0f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        s = fmaf(qi[e], ld_f(kj + e), s);
        dp = fmaf(di[e], ld_f(vj + e), dp);
      }
      s = warp_sum(s);
      dp = warp_sum(dp);
      const float lj = __ldg(p.logsig + j);
      const float P = __expf(fmaf(s, c, g * lj) - lse);
      const float dl = P * (dp - Di);
      if (lane == 0) atomicAdd(p.d_logsig + j, g * dl);
      dg = fmaf(lj, dl, dg);
      dt = fmaf(dl, -s * c / tau, dt);
    }
    if (lane == 0) {
      atomicAdd(p.d_gain + h, dg);
      atomicAdd(p.d_temp + h, dt);
    }
  }
}

// dL/dz of the kept rows; on the tensor-core path dL/dtau from its parts:
// sum dlogit * (q.k) / (sqrt(d) tau) = ln2 * sum dlogit * log2 P + sum_j l_j * ...
//   (the LSE term drops out because each row's dlogit sum to zero), so
// dL/dtau_h = -(ln2 * A_h - g_h * dL/dg_h) / tau_h with A_h = sum dlogit * log2 P.
__global__ void __launch_bounds__(256) bwd_finish_kernel(const __grid_constant__ BwdParams p,
                                                         int tau_from_parts) {
  grid_dep_wait();
  grid_dep_launch();
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nt = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t j = t0; j < p.m_total; j += nt) {
    const float l = __ldg(p.logsig + j);
    p.d_z_kept[j] = p.d_logsig[j] * (1.0f - __expf(l));
  }
  if (tau_from_parts)
    for (int64_t h = t0; h < p.hq; h += nt)
      p.d_temp[h] = -(kLn2f * p.acc[h] - __ldg(p.gain + h) * p.d_gain[h]) / __ldg(p.temp + h);
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

size_t attn_bwd_workspace_bytes(int64_t m_total, int hq) {
  return align256(static_cast<size_t>(m_total) * hq * sizeof(float)) + align256(2 * hq * sizeof(float));
}

tg_status launch_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                          const void* dout, tg_dtype dt, const PromptTable& pt, int hq, int hkv,
                          int dh, const float* logsig, const float* gain, const float* temp,
                          const float* lse, float* d_logsig, float* d_z_kept, float* d_gain,
                          float* d_temp, void* workspace, cudaStream_t st) {
  static thread_local BwdParams p;
  for (int b = 0; b <= pt.batch; ++b) p.kept_start[b] = pt.kept_start[b];
  p.batch = pt.batch;
  p.m_total = pt.kept_start[pt.batch];
  p.hq = hq;
  p.group = hq / hkv;
  p.logsig = logsig;
  p.gain = gain;
  p.temp = temp;
  p.lse = lse;
  p.D = static_cast<float*>(workspace);
  p.acc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                   align256(static_cast<size_t>(p.m_total) * hq * sizeof(float)));
  p.d_logsig = d_logsig;
  p.d_z_kept = d_z_kept;
  p.d_gain = d_gain;
  p.d_temp = d_temp;
  const int64_t warps = static_cast<int64_t>(p.m_total) * hq;
  int64_t blocks = (warps + 7) / 8;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (blocks > cap) blocks = cap;
  const dim3 grid(static_cast<unsigned>(blocks)), blk(256);
  tg_status r;
#define TG_BWD_LAUNCH(T, DH)                                                                    \
  do {                                                                                          \
    r = cuda_check(launch_pdl(bwd_prep_kernel<T, DH>, grid, blk, 0, st,                         \
                              static_cast<const T*>(out), static_cast<const T*>(dout), p),      \
                   "attention backward prep launch");                                           \
    if (r != TG_OK) return r;                                                                   \
    r = cuda_check(launch_pdl(bwd_simt_kernel<T, DH>, grid, blk, 0, st,                         \
                              static_cast<const T*>(q), static_cast<const T*>(k),               \
                              static_cast<const T*>(v), static_cast<const T*>(dout), p),        \
                   "attention backward launch");                                                \
    if (r != TG_OK) return r;                                                                   \
  } while (0)
  if (dt == TG_BF16) {
    if (dh == 64) TG_BWD_LAUNCH(__nv_bfloat16, 64);
    else TG_BWD_LAUNCH(__nv_bfloat16, 128);
  } else {
    if (dh == 64) TG_BWD_LAUNCH(float, 64);
    else TG_BWD_LAUNCH(float, 128);
  }
#undef TG_BWD_LAUNCH
  unsigned fb = static_cast<unsigned>((p.m_total + 255) / 256);
  if (fb == 0) fb = 1;
  return cuda_check(launch_pdl(bwd_finish_kernel, dim3(fb), blk, 0, st, p, 0),
                    "attention backward finish launch");
}

}  // namespace tg
