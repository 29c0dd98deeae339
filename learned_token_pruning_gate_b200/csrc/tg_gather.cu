// Compaction of the kept rows (TokenGate: "layers above L process only the kept
// tokens and create no KV cache for the removed ones").
//
// Main path (bulk): a persistent CTA per SM streams batches of kept rows
// through a ring of shared-memory stages with the bulk copy engine
// (cp.async.bulk, whole rows, completion counted on an mbarrier): warp 0 reads
// the kept indices and loads every tensor's row of the batch, warps 2-7 rotate
// the q/k heads in place (RoPE) and write the bias term (two groups of three
// warps taking alternate batches, so two batches rotate at once), warp 1 stores the rows
// back with bulk shared->global copies.  A stage holds each tensor's rows of the
// batch back to back; the compacted rows of a batch are consecutive in every
// output, so each tensor leaves in one store (the copy engine is bound by its
// number of operations more than by bytes for rows of a few KB).  Bytes in flight
// are bounded by shared memory (4 x 48 KB per SM), not by registers, so a handful
// of threads keep the HBM busy.
//
// Fallback (rows wider than a stage): one warp moves one (kept row, tensor)
// pair with 16-byte vector loads and stores.  Rows that carry attention heads are rotated by RoPE at their
// original position inside the prompt: the warp evaluates that row's angles
// pos * theta^(-2i/d) in fp64 once (two sincos per lane for d = 128), keeps
// cos/sin in fp32 in shared memory, and rotates every head in fp32.  The warp
// handling tensor 0 of a row also writes the row's bias term
// l = log sigmoid(z) (0 for question tokens).
#include <cmath>

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
  grid_dep_wait();  // the kept indices and scores are complete
  grid_dep_launch();
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


// ---------------------------------------------------------------------------
// Bulk path
// ---------------------------------------------------------------------------
constexpr int kBulkThreads = 256;
constexpr int kBulkStages = 4;
constexpr uint32_t kStageBytes = 48 * 1024;
constexpr int kMaxBatchRows = 32;
constexpr int kMaxAngles = 1024;  // rows per batch x head_dim / 2
constexpr int kGroups = 2;        // rotating groups (alternate batches)
constexpr int kIdxCap = 2048;     // kept indices of a CTA's batches preloaded at start
constexpr int kGroupThreads = (kBulkThreads - 64) / kGroups;

struct BulkParams {
  PromptTable pt;
  const uint8_t* src[TG_MAX_GATHER_TENSORS];
  uint8_t* dst[TG_MAX_GATHER_TENSORS];
  int32_t row_bytes[TG_MAX_GATHER_TENSORS];
  int32_t row_off[TG_MAX_GATHER_TENSORS];  // bytes of the tensors before this one in a kept row
  int32_t rope_heads[TG_MAX_GATHER_TENSORS];
  // RoPE angle of position pos, dim i: pos * theta^(-2i/d) radians, kept as a
  // fraction of a turn in 0.64 fixed point (evaluated on the host in fp64): the
  // product with an integer position, mod 2^64, is the angle's fractional turn
  uint64_t turns[kMaxHalf];
  const int32_t* kept_idx;
  const float* z;
  float* logsig;
  uint32_t* status;
  int32_t m_total;
  int32_t n_tensors;
  int32_t head_dim;
  int32_t row_total;   // bytes of one kept row over all tensors
  int32_t rows;        // kept rows per batch
  int32_t n_batches;
};

struct BulkSmem {
  uint8_t stage[kBulkStages][kStageBytes];
  float2 cs[kGroups][kMaxAngles];  // (cos, sin) of each group's batch
  int32_t idx[kIdxCap];            // this CTA's kept indices, batch after batch
  int32_t src_row[kBulkStages][kMaxBatchRows];  // -1: invalid index, row skipped
  int32_t prompt[kBulkStages][kMaxBatchRows];
  int32_t kept_start[kMaxBatch + 1];
  int32_t start[kMaxBatch + 1];
  uint64_t full[kBulkStages], done[kBulkStages], empty[kBulkStages];
  int32_t loads_issued[kBulkStages];  // batches loaded into each stage so far
  int abort_flag;
};

template <typename T>
__global__ void __launch_bounds__(kBulkThreads, 1) gather_bulk_kernel(const __grid_constant__ BulkParams p) {
  using E = Elem<T>;
  constexpr int VE = E::kPerVec;
  extern __shared__ uint8_t smem_raw[];
  BulkSmem& sm = *reinterpret_cast<BulkSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                              ~static_cast<uintptr_t>(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int B = p.pt.batch;
  const int half = p.head_dim / 2;
  for (int i = threadIdx.x; i <= B; i += blockDim.x) {
    sm.kept_start[i] = p.pt.kept_start[i];
    sm.start[i] = p.pt.start[i];
  }
  grid_dep_wait();  // the kept indices and scores are complete
  grid_dep_launch();
  // this CTA's kept indices (batches blockIdx.x, blockIdx.x + G, ...), so the
  // load thread never waits on an index; batches past the buffer read theirs
  // one batch ahead instead
  for (int j = threadIdx.x; j < kIdxCap; j += blockDim.x) {
    const int kb = j / p.rows, r = j - kb * p.rows;
    const int64_t i = static_cast<int64_t>(blockIdx.x + kb * static_cast<int>(gridDim.x)) * p.rows + r;
    if ((blockIdx.x + kb * static_cast<int>(gridDim.x)) < p.n_batches && i < p.m_total)
      sm.idx[j] = __ldg(p.kept_idx + i);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kBulkStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);
      mbar_init(smem_u32(&sm.done[s]), kGroupThreads);
      mbar_init(smem_u32(&sm.empty[s]), 1);
      sm.loads_issued[s] = 0;
    }
    sm.abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  volatile int* abort_flag = &sm.abort_flag;
  const int G = gridDim.x;

  if (warp == 0) {
    // ---------------- loads ----------------
    if (lane == 0) {
      // kept indices are read one batch ahead, so their latency overlaps the
      // previous batch's copies
      int32_t srcs[kMaxBatchRows], nxt[kMaxBatchRows];
      auto fetch = [&](int batch, int32_t* dst) {
        if (batch >= p.n_batches) return;
        const int i0 = batch * p.rows;
        const int n = min(p.rows, p.m_total - i0);
        for (int r = 0; r < n; ++r) dst[r] = __ldg(p.kept_idx + i0 + r);
      };
      const int k_pre = kIdxCap / p.rows;  // batches whose indices are preloaded
      if (k_pre == 0) fetch(blockIdx.x, nxt);
      for (int k = 0;; ++k) {
        const int batch = blockIdx.x + k * G;
        if (batch >= p.n_batches) break;
        const int i0 = batch * p.rows;
        const int n = min(p.rows, p.m_total - i0);
        if (k < k_pre) {
          for (int r = 0; r < n; ++r) srcs[r] = sm.idx[k * p.rows + r];
          if (k + 1 == k_pre) fetch(batch + G, nxt);
        } else {
          for (int r = 0; r < n; ++r) srcs[r] = nxt[r];
          fetch(batch + G, nxt);
        }
        const int s = k % kBulkStages;
        const uint32_t ph = (k / kBulkStages) & 1;
        if (!mbar_wait(smem_u32(&sm.empty[s]), ph ^ 1, abort_flag, p.status, kDevTimeoutGather))
          break;
        uint32_t bytes = 0;
        for (int r = 0; r < n; ++r) {
          const int b = prompt_of_kept(sm.kept_start, B, i0 + r);
          const bool valid = srcs[r] >= sm.start[b] && srcs[r] < sm.start[b + 1];
          if (!valid) atomicOr(p.status, kDevGatherIndex);
          sm.src_row[s][r] = valid ? srcs[r] : -1;
          sm.prompt[s][r] = b;
          bytes += valid ? p.row_total : 0;
        }
        const uint32_t fb = smem_u32(&sm.full[s]);
        mbar_arrive_expect_tx(fb, bytes);
        ++sm.loads_issued[s];
        const uint32_t base = smem_u32(sm.stage[s]);
        for (int r = 0; r < n; ++r) {
          if (sm.src_row[s][r] < 0) continue;
          const int64_t row = sm.src_row[s][r];
          for (int t = 0; t < p.n_tensors; ++t)
            bulk_g2s(base + p.rows * p.row_off[t] + r * p.row_bytes[t], p.src[t] + row * p.row_bytes[t],
                     p.row_bytes[t], fb);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- stores ----------------
    if (lane == 0) {
      for (int k = 0;; ++k) {
        const int batch = blockIdx.x + k * G;
        if (batch >= p.n_batches) break;
        const int s = k % kBulkStages;
        const uint32_t ph = (k / kBulkStages) & 1;
        if (!mbar_wait(smem_u32(&sm.done[s]), ph, abort_flag, p.status, kDevTimeoutGather)) break;
        const int i0 = batch * p.rows;
        const int n = min(p.rows, p.m_total - i0);
        const uint32_t base = smem_u32(sm.stage[s]);
        // a stage holds each tensor's rows of the batch back to back, and the
        // compacted rows are consecutive: one store per tensor (per row only when
        // an invalid index left a row unloaded)
        bool all_valid = true;
        for (int r = 0; r < n; ++r) all_valid &= sm.src_row[s][r] >= 0;
        if (all_valid) {
          for (int t = 0; t < p.n_tensors; ++t)
            bulk_s2g(p.dst[t] + static_cast<int64_t>(i0) * p.row_bytes[t],
                     base + p.rows * p.row_off[t], n * p.row_bytes[t]);
        } else {
          for (int r = 0; r < n; ++r) {
            if (sm.src_row[s][r] < 0) continue;
            const int64_t i = i0 + r;
            for (int t = 0; t < p.n_tensors; ++t)
              bulk_s2g(p.dst[t] + i * p.row_bytes[t], base + p.rows * p.row_off[t] + r * p.row_bytes[t],
                       p.row_bytes[t]);
          }
        }
        bulk_commit();
        // hand the stage back as soon as these stores have read it
        bulk_wait_read<0>();
        mbar_arrive(smem_u32(&sm.empty[s]));
      }
      bulk_wait_all<0>();  // every store has landed before the CTA exits
    }
    __syncwarp();
  } else {
    // ---------------- RoPE and bias term (warps 2-7) ----------------
    const int gid = (threadIdx.x - 64) / kGroupThreads;  // group: batches k with k % kGroups == gid
    const int ct = (threadIdx.x - 64) - gid * kGroupThreads;
    bool any_rope = false;
    for (int t = 0; t < p.n_tensors; ++t) any_rope |= p.rope_heads[t] > 0;
    const int hv = half / VE;  // vectors per half head
    for (int k = gid;; k += kGroups) {
      const int batch = blockIdx.x + k * G;
      if (batch >= p.n_batches) break;
      const int s = k % kBulkStages;
      const uint32_t ph = (k / kBulkStages) & 1;
      const bool ok = mbar_wait(smem_u32(&sm.full[s]), ph, abort_flag, p.status, kDevTimeoutGather);
      if (named_barrier_or(2 + gid, kGroupThreads, !ok)) break;  // the group leaves together
      const int i0 = batch * p.rows;
      const int n = min(p.rows, p.m_total - i0);
      // bias term: the score load is issued first, its value used last
      const bool bias_row = p.logsig && ct < n && sm.src_row[s][ct] >= 0;
      const float zr = bias_row ? __ldg(p.z + sm.src_row[s][ct]) : 0.0f;
      if (any_rope) {
        float2* cs_buf = sm.cs[gid];
        for (int a = ct; a < n * half; a += kGroupThreads) {
          const int r = a / half, i = a - r * half;
          const int32_t src = sm.src_row[s][r];
          float sn = 0.0f, c = 1.0f;
          if (src >= 0) {
            const uint32_t pos = static_cast<uint32_t>(src - sm.start[sm.prompt[s][r]]);
            const uint64_t f = p.turns[i];
            // top 32 bits of pos * f mod 2^64: the angle's fractional turn
            const uint32_t top = pos * static_cast<uint32_t>(f >> 32) + __umulhi(pos, static_cast<uint32_t>(f));
            // as a signed fraction of a half turn in [-1, 1): angle = pi * x
            sincospif(static_cast<float>(static_cast<int32_t>(top)) * 4.656612873077393e-10f, &sn, &c);
          }
          cs_buf[a] = make_float2(c, sn);
        }
        named_barrier(4 + gid, kGroupThreads);
        // rotate-half pairs (i, i + d/2): a thread owns one vector column (VE
        // dims) of one kept row, holds that row's cos/sin for those dims in
        // registers and rotates a share of the row's heads, two at a time
        const int cvec = ct % hv;
        const int slot = ct / hv, lanes = kGroupThreads / hv;
        const int nhg = lanes >= n ? lanes / n : 1;  // head groups per row
        for (int unit = slot; slot < lanes && unit < n * nhg; unit += lanes) {
          const int r = unit / nhg, hg = unit - r * nhg;
          if (sm.src_row[s][r] < 0) continue;
          float2 w[VE];
#pragma unroll
          for (int e = 0; e < VE; ++e) w[e] = cs_buf[r * half + cvec * VE + e];
          for (int t = 0; t < p.n_tensors; ++t) {
            const int nh = p.rope_heads[t];
            uint4* base = reinterpret_cast<uint4*>(sm.stage[s] + p.rows * p.row_off[t] + r * p.row_bytes[t]) + cvec;
            const int hstep = p.head_dim / VE;  // vectors per head
            for (int h = hg; h < nh; h += 2 * nhg) {
              const bool two = h + nhg < nh;
              uint4* pa0 = base + h * hstep;
              uint4* pa1 = base + (two ? h + nhg : h) * hstep;
              uint4 a0 = pa0[0], b0 = pa0[hv], a1 = pa1[0], b1 = pa1[hv];
#pragma unroll
              for (int e = 0; e < VE; ++e) {
                const float x0 = E::get(a0, e), x1 = E::get(b0, e);
                const float y0 = E::get(a1, e), y1 = E::get(b1, e);
                E::set(a0, e, x0 * w[e].x - x1 * w[e].y);
                E::set(b0, e, x1 * w[e].x + x0 * w[e].y);
                E::set(a1, e, y0 * w[e].x - y1 * w[e].y);
                E::set(b1, e, y1 * w[e].x + y0 * w[e].y);
              }
              pa0[0] = a0;
              pa0[hv] = b0;
              if (two) {
                pa1[0] = a1;
                pa1[hv] = b1;
              }
            }
          }
        }
        named_barrier(4 + gid, kGroupThreads);  // cs is rewritten for the group's next batch
      }
      if (bias_row) {
        const int b = sm.prompt[s][ct];
        const int32_t pos = sm.src_row[s][ct] - sm.start[b];
        const bool is_doc = pos >= p.pt.doc_begin[b] && pos < p.pt.doc_end[b];
        p.logsig[i0 + ct] = is_doc ? log_sigmoid(zr) : 0.0f;
      }
      fence_proxy_async_smem();  // the rotated rows are read by the bulk stores
      mbar_arrive(smem_u32(&sm.done[s]));
    }
  }
  // After a timed-out wait, loads may still be in flight into this CTA's shared
  // memory: let each stage's latest load complete (bounded) before exiting.
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    for (int s = 0; s < kBulkStages; ++s) {
      const int n = sm.loads_issued[s];
      if (n > 0) mbar_drain(smem_u32(&sm.full[s]), (n - 1) & 1);
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
  // bulk path: every tensor's row of a kept row fits in one stage together
  {
    int32_t row_total = 0;
    BulkParams b;
    memset(&b, 0, sizeof(b));
    for (int i = 0; i < n_tensors; ++i) {
      b.src[i] = p.t[i].src;
      b.dst[i] = p.t[i].dst;
      b.row_bytes[i] = p.t[i].row_vecs * 16;
      b.row_off[i] = row_total;
      b.rope_heads[i] = p.t[i].rope_heads;
      row_total += b.row_bytes[i];
    }
    const int half = p.head_dim / 2;
    int rows = row_total > 0 ? static_cast<int>(kStageBytes / row_total) : kMaxBatchRows;
    if (rows > kMaxBatchRows) rows = kMaxBatchRows;
    if (half > 0 && rows > kMaxAngles / half) rows = kMaxAngles / half;
    if (rows > kGroupThreads) rows = kGroupThreads;  // one thread per row writes the bias term
    if (n_tensors > 0 && rows >= 1 && m_total < (int64_t(1) << 31)) {
      b.pt = pt;
      for (int i = 0; i < half && i < kMaxHalf; ++i) {
        const double f = std::pow(theta, -2.0 * i / static_cast<double>(p.head_dim)) /
                         (2.0 * 3.14159265358979323846);
        b.turns[i] = static_cast<uint64_t>(std::ldexp(f, 64));  // f < 1: fits
      }
      b.kept_idx = kept_idx;
      b.z = z;
      b.logsig = logsig;
      b.status = p.status;
      b.m_total = static_cast<int32_t>(m_total);
      b.n_tensors = n_tensors;
      b.head_dim = p.head_dim;
      b.row_total = row_total;
      b.rows = rows;
      b.n_batches = static_cast<int32_t>((m_total + rows - 1) / rows);
      int grid = num_sms();
      if (grid > b.n_batches) grid = b.n_batches;
      const size_t smem = sizeof(BulkSmem) + 128;
      tg_status r;
      if (dt == TG_BF16) {
        r = cuda_check(cudaFuncSetAttribute(gather_bulk_kernel<__nv_bfloat16>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            static_cast<int>(smem)),
                       "gather smem attribute");
        if (r != TG_OK) return r;
        r = cuda_check(launch_pdl(gather_bulk_kernel<__nv_bfloat16>, dim3(grid), dim3(kBulkThreads),
                                  smem, st, b),
                       "gather launch");
      } else {
        r = cuda_check(cudaFuncSetAttribute(gather_bulk_kernel<float>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            static_cast<int>(smem)),
                       "gather smem attribute");
        if (r != TG_OK) return r;
        r = cuda_check(launch_pdl(gather_bulk_kernel<float>, dim3(grid), dim3(kBulkThreads), smem,
                                  st, b),
                       "gather launch");
      }
      return r;
    }
  }
  const int64_t items = m_total * nt;
  int64_t blocks = (items + kWarps - 1) / kWarps;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (blocks > cap) blocks = cap;
  const dim3 g(static_cast<unsigned>(blocks)), blk(kWarps * 32);
  if (dt == TG_BF16)
    return cuda_check(launch_pdl(gather_kernel<__nv_bfloat16>, g, blk, 0, st, p), "gather launch");
  return cuda_check(launch_pdl(gather_kernel<float>, g, blk, 0, st, p), "gather launch");
}

}  // namespace tg
