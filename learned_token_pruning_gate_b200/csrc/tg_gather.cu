// Compaction of the kept rows (TokenGate: "layers above L process only the kept
// tokens and create no KV cache for the removed ones").
//
// One warp moves one (kept row, tensor) pair with 16-byte vector loads and
// stores.  Rows that carry attention heads are rotated by RoPE at their
// original position inside the prompt: the warp evaluates that row's angles
// pos * theta^(-2i/d) in fp64 once (two sincos per lane for d = 128), keeps
// cos/sin in fp32 in shared memory, and rotates every head in fp32.  The warp
// handling tensor 0 of a row also writes the row's bias term
// l = log sigmoid(z) (0 for question tokens).
#include "tg_internal.cuh"

namespace tg {
namespace {

constexpr int kWarps = 8;
constexpr int kMaxHalf = 128;  // head_dim / 2

struct GatherTensorDev {
  const uint8_t* src;
  uint8_t* dst;
  int32_t row_vecs;    // 16-byte vectors per row
  int32_t rope_heads;  // heads rotated at the front of the row
};

struct GatherParams {
  PromptTable pt;
  GatherTensorDev t[TG_MAX_GATHER_TENSORS];
  const int32_t* kept_idx;
  const float* z;
  float* logsig;
  uint32_t* status;
  double theta;
  int64_t m_total;
  int32_t n_tensors;
  int32_t head_dim;
};

template <typename T>
struct Elem;
template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kPerVec = 8;
  static __device__ __forceinline__ float get(const uint4& v, int e) {
    const __nv_bfloat16* p = reinterpret_cast<const __nv_bfloat16*>(&v);
    return __bfloat162float(p[e]);
  }
  static __device__ __forceinline__ void set(uint4& v, int e, float x) {
    __nv_bfloat16* p = reinterpret_cast<__nv_bfloat16*>(&v);
    p[e] = __float2bfloat16_rn(x);
  }
};
template <>
struct Elem<float> {
  static constexpr int kPerVec = 4;
  static __device__ __forceinline__ float get(const uint4& v, int e) {
    return reinterpret_cast<const float*>(&v)[e];
  }
  static __device__ __forceinline__ void set(uint4& v, int e, float x) {
    reinterpret_cast<float*>(&v)[e] = x;
  }
};

__device__ __forceinline__ float log_sigmoid(float x) {
  return fminf(x, 0.0f) - log1pf(expf(-fabsf(x)));
}

// Prompt that owns kept row i (kept_start is ascending; empty prompts skipped).
__device__ __forceinline__ int prompt_of_kept(const int32_t* kept_start, int batch, int64_t i) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (kept_start[mid] <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32) gather_kernel(const __grid_constant__ GatherParams p) {
  using E = Elem<T>;
  constexpr int VE = E::kPerVec;
  __shared__ int32_t s_kept_start[kMaxBatch + 1];
  __shared__ int32_t s_start[kMaxBatch + 1];
  __shared__ int32_t s_doc_begin[kMaxBatch];
  __shared__ int32_t s_doc_end[kMaxBatch];
  __shared__ double s_inv_freq[kMaxHalf];
  __shared__ float s_cos[kWarps][kMaxHalf];
  __shared__ float s_sin[kWarps][kMaxHalf];

  const int B = p.pt.batch;
  for (int i = threadIdx.x; i <= B; i += blockDim.x) {
    s_kept_start[i] = p.pt.kept_start[i];
    s_start[i] = p.pt.start[i];
    if (i < B) {
      s_doc_begin[i] = p.pt.doc_begin[i];
      s_doc_end[i] = p.pt.doc_end[i];
    }
  }
  const int half = p.head_dim / 2;
  for (int i = threadIdx.x; i < half; i += blockDim.x)
    s_inv_freq[i] = pow(p.theta, -2.0 * static_cast<double>(i) / static_cast<double>(p.head_dim));
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t n_items = p.m_total * p.n_tensors;
  const int64_t warp_stride = static_cast<int64_t>(gridDim.x) * kWarps;
  int64_t last_pos_row = -1;  // kept row whose angles are cached in s_cos/s_sin

  for (int64_t item = static_cast<int64_t>(blockIdx.x) * kWarps + warp; item < n_items;
       item += warp_stride) {
    const int64_t i = item / p.n_tensors;
    const int ti = static_cast<int>(item - i * p.n_tensors);
    const int32_t src_row = __ldg(p.kept_idx + i);
    const int b = prompt_of_kept(s_kept_start, B, i);
    const int32_t pos = src_row - s_start[b];
    if (src_row < s_start[b] || src_row >= s_start[b + 1]) {  // not a row of its prompt
      if (lane == 0) atomicOr(p.status, kDevGatherIndex);
      continue;
    }

    if (ti == 0 && p.logsig && lane == 0) {
      const bool is_doc = pos >= s_doc_begin[b] && pos < s_doc_end[b];
      p.logsig[i] = is_doc ? log_sigmoid(__ldg(p.z + src_row)) : 0.0f;
    }

    const GatherTensorDev g = p.t[ti];
    const uint4* src = reinterpret_cast<const uint4*>(g.src) + static_cast<int64_t>(src_row) * g.row_vecs;
    uint4* dst = reinterpret_cast<uint4*>(g.dst) + i * g.row_vecs;
    int first_plain = 0;

    if (g.rope_heads > 0) {
      if (last_pos_row != i) {
        __syncwarp();  // every lane is done reading the previous row's angles
        for (int a = lane; a < half; a += 32) {
          double sn, cs;
          sincos(static_cast<double>(pos) * s_inv_freq[a], &sn, &cs);
          s_cos[warp][a] = static_cast<float>(cs);
          s_sin[warp][a] = static_cast<float>(sn);
        }
        __syncwarp();
        last_pos_row = i;
      }
      const int hv = p.head_dim / VE;  // vectors per head
      const int hh = hv / 2;           // vectors per half head
      const int n_tasks = g.rope_heads * hh;
      // four pair-tasks per lane per round: all eight loads are issued before any
      // rotation or store, so a warp keeps 4 KB of the row in flight
      constexpr int kU = 4;
      for (int base = 0; base < n_tasks; base += 32 * kU) {
        uint4 va[kU], vb[kU];
        int off[kU], cc[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int task = base + lane + 32 * u;
          const int head = task / hh;
          cc[u] = task - head * hh;
          off[u] = head * hv + cc[u];
          if (task < n_tasks) {
            va[u] = __ldg(src + off[u]);
            vb[u] = __ldg(src + off[u] + hh);
          }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          if (base + lane + 32 * u >= n_tasks) continue;
#pragma unroll
          for (int e = 0; e < VE; ++e) {
            const int a = cc[u] * VE + e;
            const float cs = s_cos[warp][a], sn = s_sin[warp][a];
            const float x0 = E::get(va[u], e), x1 = E::get(vb[u], e);
            E::set(va[u], e, x0 * cs - x1 * sn);
            E::set(vb[u], e, x1 * cs + x0 * sn);
          }
          dst[off[u]] = va[u];
          dst[off[u] + hh] = vb[u];
        }
      }
      first_plain = g.rope_heads * hv;
    }

    // Plain copy: eight independent 16-byte loads in flight per lane per round.
    constexpr int kC = 8;
    for (int base = first_plain; base < g.row_vecs; base += 32 * kC) {
      uint4 a[kC];
#pragma unroll
      for (int u = 0; u < kC; ++u) {
        const int vv = base + lane + 32 * u;
        if (vv < g.row_vecs) a[u] = __ldg(src + vv);
      }
#pragma unroll
      for (int u = 0; u < kC; ++u) {
        const int vv = base + lane + 32 * u;
        if (vv < g.row_vecs) dst[vv] = a[u];
      }
    }
  }
}

}  // namespace

tg_status launch_gather(const int32_t* kept_idx, int64_t m_total, const PromptTable& pt,
                        tg_dtype dt, const tg_gather_tensor* tensors, int n_tensors, int head_dim,
                        double theta, const float* z, float* logsig, cudaStream_t st) {
  GatherParams p;
  memset(&p, 0, sizeof(p));
  p.pt = pt;
  const int esz = dt == TG_BF16 ? 2 : 4;
  for (int i = 0; i < n_tensors; ++i) {
    p.t[i].src = static_cast<const uint8_t*>(tensors[i].src);
    p.t[i].dst = static_cast<uint8_t*>(tensors[i].dst);
    p.t[i].row_vecs = tensors[i].row_elems * esz / 16;
    p.t[i].rope_heads = tensors[i].rope_heads;
  }
  int nt = n_tensors;
  if (nt == 0 && logsig) {
    // bias term only: use a zero-length tensor slot so every row is visited once
    p.t[0].row_vecs = 0;
    p.t[0].rope_heads = 0;
    nt = 1;
  }
  if (nt == 0) return TG_OK;
  p.n_tensors = nt;
  p.kept_idx = kept_idx;
  p.z = z;
  p.logsig = logsig;
  p.status = device_status_word();
  if (!p.status) return set_error(TG_ERR_CUDA, "device status word unavailable");
  p.theta = theta;
  p.m_total = m_total;
  p.head_dim = head_dim > 0 ? head_dim : 2;
  const int64_t items = m_total * nt;
  int64_t blocks = (items + kWarps - 1) / kWarps;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (blocks > cap) blocks = cap;
  if (dt == TG_BF16)
    gather_kernel<__nv_bfloat16><<<static_cast<unsigned>(blocks), kWarps * 32, 0, st>>>(p);
  else
    gather_kernel<float><<<static_cast<unsigned>(blocks), kWarps * 32, 0, st>>>(p);
  return cuda_check(cudaGetLastError(), "gather launch");
}

}  // namespace tg
