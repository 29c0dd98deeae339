// Token-gated causal GQA attention over the kept rows (TokenGate: each kept
// token's gate score is added to the attention logits above the gate as a
// bias scaled by a per-head learned gain -- the Mixture-of-Experts router
// trick -- and a per-head learned temperature corrects for each query seeing
// fewer keys):
//     logit_ij = q_i.k_j / (sqrt(d) tau_h) + g_h l_j,   j <= i in the prompt
// Both kernels work in the log2 domain: t = s * log2(e)/(sqrt(d) tau_h) +
// g_h log2(e) l_j, so the per-key bias and the per-head temperature fold into
// one FMA per logit.
//
// attn_tc_kernel (bf16, head_dim 64/128) -- one CTA per (head, 128-query tile):
//   warp 0     TMA: the Q tile once, then K and V tiles (128 keys) into a
//              2-stage ring, 128-byte swizzle
//   warp 1     tcgen05.mma: S = Q K^T into one of two TMEM buffers (fp32,
//              128 x 128), then O += P V with P read from TMEM (bf16) and V
//              from shared memory (MN-major), O accumulating in TMEM
//   warps 2-5  softmax, one query row per thread: tcgen05.ld of S, scale+bias,
//              causal mask on the diagonal tile, online max/sum, rescale of O
//              in TMEM when the row max grows, P written back over S as bf16;
//              finally O / l -> bf16 -> global, and the row's LSE.
// Query tiles are issued longest-first (last tile of the longest prompt first).
// attn_simt_kernel is the CUDA-core path (fp32 and the reference for bf16).
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

// ---- tensor-core path -------------------------------------------------------
constexpr int kThreads = 192;
constexpr int kBM = 128;  // queries per tile
constexpr int kBN = 128;  // keys per tile
constexpr uint32_t kTmemCols = 512;

template <int DH>
struct TcLayout {
  static constexpr uint32_t kChunks = DH / 64;
  static constexpr uint32_t kBox = 128 * 128;       // one 128-row x 64-col bf16 box (16 KB)
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kChunks * kBox;            // 2 stages
  static constexpr uint32_t kV = kK + 2 * kChunks * kBox;   // 2 stages
  static constexpr uint32_t kBias = kV + 2 * kChunks * kBox;  // [2][128] fp32
  static constexpr uint32_t kBars = kBias + 2 * 128 * 4;
  static constexpr uint32_t kMisc = kBars + 16 * 8;
  static constexpr uint32_t kTotal = kMisc + 16;
  static constexpr uint32_t kTileBytes = kChunks * kBox;  // one K or V tile
  // keep one CTA per SM so the 512-column TMEM allocation never waits
  static constexpr uint32_t kDynSmem = (kTotal + 1024 > 120 * 1024) ? kTotal + 1024 : 120 * 1024;
};

// barrier slots
enum { kBarQ = 0, kBarK = 1, kBarV = 3, kBarKvEmpty = 5, kBarS = 7, kBarP = 9, kBarPv = 11 };

template <int DH>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ AttnParams p) {
  using Lay = TcLayout<DH>;
  const int h = blockIdx.x;
  const int b = p.order[blockIdx.z];
  const int32_t kstart = p.kept_start[b];
  const int32_t len = p.kept_start[b + 1] - kstart;
  const int n_tiles = (len + kBM - 1) / kBM;
  const int qt = n_tiles - 1 - static_cast<int>(blockIdx.y);
  if (qt < 0) return;  // this prompt has fewer query tiles
  const int q0 = qt * kBM;
  const int n_kv = qt + 1;  // causal: key tiles 0..qt
  const int hk = h / (p.hq / p.hkv);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMisc + 4);
  float* s_bias = reinterpret_cast<float*>(smem + Lay::kBias);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    mbar_init(bar(kBarQ), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarK + s), 1);
      mbar_init(bar(kBarV + s), 1);
      mbar_init(bar(kBarKvEmpty + s), 1);
      mbar_init(bar(kBarS + s), 1);
      mbar_init(bar(kBarP + s), 128);
    }
    mbar_init(bar(kBarPv), 1);
    *abort_flag = 0;
    mbar_fence_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_o = tmem + 256;  // O accumulator columns [256, 256 + DH)

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(kBarQ), Lay::kTileBytes);
      for (uint32_t c = 0; c < Lay::kChunks; ++c)
        tma_load_2d(sbase + Lay::kQ + c * Lay::kBox, &tm_q, h * DH + c * 64, kstart + q0, bar(kBarQ));
      for (int j = 0; j < n_kv; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(bar(kBarKvEmpty + s), ph ^ 1, abort_flag, p.status, kDevTimeoutAttn)) break;
        const int krow = kstart + j * kBN;
        mbar_arrive_expect_tx(bar(kBarK + s), Lay::kTileBytes);
        for (uint32_t c = 0; c < Lay::kChunks; ++c)
          tma_load_2d(sbase + Lay::kK + (s * Lay::kChunks + c) * Lay::kBox, &tm_k, hk * DH + c * 64,
                      krow, bar(kBarK + s));
        mbar_arrive_expect_tx(bar(kBarV + s), Lay::kTileBytes);
        for (uint32_t c = 0; c < Lay::kChunks; ++c)
          tma_load_2d(sbase + Lay::kV + (s * Lay::kChunks + c) * Lay::kBox, &tm_v, hk * DH + c * 64,
                      krow, bar(kBarV + s));
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, DH, false, true);
      auto issue_pv = [&](int jj) -> bool {
        const int sp = jj & 1;
        const uint32_t php = (jj >> 1) & 1;
        if (!mbar_wait(bar(kBarP + sp), php, abort_flag, p.status, kDevTimeoutAttn)) return false;
        if (!mbar_wait(bar(kBarV + sp), php, abort_flag, p.status, kDevTimeoutAttn)) return false;
        tc_fence_after();
        const uint32_t vb = sbase + Lay::kV + sp * Lay::kChunks * Lay::kBox;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          umma_ts(t_o, tmem + sp * 128 + kk * 8, sw128_desc(vb + kk * 2048, Lay::kBox, 1024),
                  idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(kBarPv));
        umma_commit(bar(kBarKvEmpty + sp));
        return true;
      };
      bool ok = mbar_wait(bar(kBarQ), 0, abort_flag, p.status, kDevTimeoutAttn);
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!(ok = mbar_wait(bar(kBarK + s), ph, abort_flag, p.status, kDevTimeoutAttn))) break;
        if (j >= 2 &&
            !(ok = mbar_wait(bar(kBarPv), (j - 2) & 1, abort_flag, p.status, kDevTimeoutAttn)))
          break;
        tc_fence_after();
        const uint32_t kb = sbase + Lay::kK + s * Lay::kChunks * Lay::kBox;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t off = (kk >> 2) * Lay::kBox + (kk & 3) * 32;
          umma_ss(tmem + s * 128, sw128_desc(sbase + Lay::kQ + off, 16, 1024),
                  sw128_desc(kb + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(kBarS + s));
        if (j >= 1 && !(ok = issue_pv(j - 1))) break;
      }
      if (ok) issue_pv(n_kv - 1);
    }
    __syncwarp();
  } else {
    // softmax: thread owns query row r of the tile
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float scale = kLog2e / (sqrtf(static_cast<float>(DH)) * __ldg(p.temp + h));
    const float gl = __ldg(p.gain + h) * kLog2e;
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int s = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      // this tile's per-key bias into shared memory (buffer s)
      {
        const int key = j * kBN + r;
        float bv = 0.0f;
        if (p.logsig && key < len) bv = gl * __ldg(p.logsig + kstart + key);
        s_bias[s * 128 + r] = bv;
      }
      named_barrier(1, 128);
      if (!(ok = mbar_wait(bar(kBarS + s), ph, abort_flag, p.status, kDevTimeoutAttn))) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + s * 128 + c * 32, sr[c]);
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_wait(sr[c]);
      const float* bias = s_bias + s * 128;
      const bool diag = (j == n_kv - 1);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = c * 32 + e;
          float t = fmaf(__uint_as_float(sr[c][e]), scale, bias[col]);
          if (diag && col > r) t = -INFINITY;
          sr[c][e] = __float_as_uint(t);
          mx = fmaxf(mx, t);
        }
      }
      const float m_new = fmaxf(m, mx);
      const float alpha = exp2_approx(m - m_new);
      float rowsum = 0.0f;
      uint32_t pk[2][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float p0 = exp2_approx(__uint_as_float(sr[c][e]) - m_new);
          const float p1 = exp2_approx(__uint_as_float(sr[c][e + 1]) - m_new);
          rowsum += p0 + p1;
          __nv_bfloat162 pp = __floats2bfloat162_rn(p0, p1);
          pk[c >> 1][(c & 1) * 16 + (e >> 1)] = *reinterpret_cast<uint32_t*>(&pp);
        }
      }
      l = fmaf(l, alpha, rowsum);
      if (j >= 1) {
        // O may only be touched once the previous P V has finished
        if (!(ok = mbar_wait(bar(kBarPv), (j - 1) & 1, abort_flag, p.status, kDevTimeoutAttn)))
          break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, m_new > m)) {
#pragma unroll
          for (int c = 0; c < DH / 32; ++c) {
            uint32_t orow[32];
            tmem_ld32(t_o + lane_off + c * 32, orow);
            tmem_ld_wait(orow);
#pragma unroll
            for (int e = 0; e < 32; ++e) orow[e] = __float_as_uint(__uint_as_float(orow[e]) * alpha);
            tmem_st32(t_o + lane_off + c * 32, orow);
          }
        }
      }
      // P (bf16 pairs) over the first 64 columns of this S buffer
      tmem_st32(tmem + lane_off + s * 128, pk[0]);
      tmem_st32(tmem + lane_off + s * 128 + 32, pk[1]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(kBarP + s));
      m = m_new;
    }
    if (ok && mbar_wait(bar(kBarPv), (n_kv - 1) & 1, abort_flag, p.status, kDevTimeoutAttn)) {
      tc_fence_after();
      const int qi = q0 + r;
      const float inv = 1.0f / l;
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) +
                           (static_cast<int64_t>(kstart + qi) * p.hq + h) * DH;
#pragma unroll
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t orow[32];
        tmem_ld32(t_o + lane_off + c * 32, orow);
        tmem_ld_wait(orow);
        if (qi < len) {
          uint32_t pkd[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            __nv_bfloat162 pp = __floats2bfloat162_rn(__uint_as_float(orow[2 * e]) * inv,
                                                      __uint_as_float(orow[2 * e + 1]) * inv);
            pkd[e] = *reinterpret_cast<uint32_t*>(&pp);
          }
          uint4* dst = reinterpret_cast<uint4*>(out + c * 32);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dst[v4] = make_uint4(pkd[4 * v4], pkd[4 * v4 + 1], pkd[4 * v4 + 2], pkd[4 * v4 + 3]);
        }
      }
      if (p.lse && qi < len)
        p.lse[static_cast<int64_t>(h) * p.m_total + kstart + qi] = (m + log2f(l)) * kLn2;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
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

template <int DH>
static tg_status launch_tc_dh(const void* q, const void* k, const void* v, const AttnParams& a,
                              int max_len, cudaStream_t st) {
  using Lay = TcLayout<DH>;
  CUtensorMap tq, tk, tv;
  const uint64_t M = static_cast<uint64_t>(a.m_total);
  if (!encode_tmap_2d_bf16(&tq, q, static_cast<uint64_t>(a.hq) * DH, M,
                           static_cast<uint64_t>(a.hq) * DH * 2, 64, kBM) ||
      !encode_tmap_2d_bf16(&tk, k, static_cast<uint64_t>(a.hkv) * DH, M,
                           static_cast<uint64_t>(a.hkv) * DH * 2, 64, kBN) ||
      !encode_tmap_2d_bf16(&tv, v, static_cast<uint64_t>(a.hkv) * DH, M,
                           static_cast<uint64_t>(a.hkv) * DH * 2, 64, kBN))
    return set_error(TG_ERR_CUDA, "cuTensorMapEncodeTiled failed for q/k/v");
  tg_status r = cuda_check(cudaFuncSetAttribute(attn_tc_kernel<DH>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                static_cast<int>(Lay::kDynSmem)),
                           "attn smem attribute");
  if (r != TG_OK) return r;
  dim3 grid(a.hq, (max_len + kBM - 1) / kBM, a.batch);
  attn_tc_kernel<DH><<<grid, kThreads, Lay::kDynSmem, st>>>(tq, tk, tv, a);
  return cuda_check(cudaGetLastError(), "attn_tc launch");
}

tg_status launch_attn_tc(const void* q, const void* k, const void* v, const PromptTable& pt,
                         int max_len, int hq, int hkv, int dh, const float* logsig,
                         const float* gain, const float* temp, void* out, float* lse,
                         cudaStream_t st) {
  AttnParams a;
  fill_params(&a, pt);
  a.logsig = logsig;
  a.gain = gain;
  a.temp = temp;
  a.out = out;
  a.lse = lse;
  a.hq = hq;
  a.hkv = hkv;
  a.status = device_status_word();
  if (!a.status) return set_error(TG_ERR_CUDA, "device status word unavailable");
  if (max_len == 0) return TG_OK;
  if (dh == 64) return launch_tc_dh<64>(q, k, v, a, max_len, st);
  return launch_tc_dh<128>(q, k, v, a, max_len, st);
}

}  // namespace tg
