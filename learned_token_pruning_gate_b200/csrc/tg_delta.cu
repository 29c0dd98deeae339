// Gated delta rule over each prompt's kept rows: the linear-attention (Gated
// DeltaNet) layers of a hybrid backbone above the gate see only the kept tokens
// (TokenGate prunes those layers too; the rule itself is the published gated
// delta rule of Gated DeltaNet):
//   k^ = k / sqrt(|k|^2 + eps),  q^ = q / sqrt(|q|^2 + eps) / sqrt(d)
//   S_t = alpha_t S_{t-1} + beta_t (v_t - alpha_t S_{t-1} k^_t) k^_t^T,  o_t = S_t q^_t
// per (prompt, head), S (d x d, fp32) starting at zero; the final S is written
// out as the layer's state for decoding.
//
// The recurrence is sequential in t but independent across rows of S: row i
// needs only (S k)_i and v_i.  A CTA owns 32 rows of one head's state; in each
// warp, 8 rows x 4 column groups, a thread holding d/4 columns of one row in
// registers, so the three dot products of a step (S k, S q, and the norms) end
// in two shuffles.  The inputs stream through a shared-memory ring of chunks of
// rows (asynchronous copies, three chunks in flight), so a step waits on no
// global load.
#include <cmath>

#include "tg_internal.cuh"

namespace tg {
namespace {

constexpr int kDeltaRows = 32;  // state rows per CTA
constexpr int kDeltaThreads = 128;

struct DeltaParams {
  const float* log_alpha;
  const float* beta;
  float* state;  // [B, H, d, d] or null
  int32_t kept_start[kMaxBatch + 1];
  int32_t heads;
  float eps;
  float q_scale;  // 1 / sqrt(d)
};

__device__ __forceinline__ float to_out(float x, float*) { return x; }
__device__ __forceinline__ __nv_bfloat16 to_out(float x, __nv_bfloat16*) { return __float2bfloat16_rn(x); }

// sum over the four column groups of a row (lanes l, l^1, l^2, l^3)
__device__ __forceinline__ float rowgroup_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

template <int JN>
__device__ __forceinline__ float dot_pairs(const float2 (&a)[JN / 2], const float2 (&b)[JN / 2]) {
  float2 s0 = make_float2(0.0f, 0.0f), s1 = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int j = 0; j < JN / 2; j += 2) {
    s0 = __ffma2_rn(a[j], b[j], s0);
    s1 = __ffma2_rn(a[j + 1], b[j + 1], s1);
  }
  return (s0.x + s0.y) + (s1.x + s1.y);
}

// (a . b, a . c) with the two chains interleaved
template <int JN>
__device__ __forceinline__ float2 dot2_pairs(const float2 (&a)[JN / 2], const float2 (&b)[JN / 2],
                                             const float2 (&c)[JN / 2]) {
  float2 s0 = make_float2(0.0f, 0.0f), s1 = s0, t0 = s0, t1 = s0;
#pragma unroll
  for (int j = 0; j < JN / 2; j += 2) {
    s0 = __ffma2_rn(a[j], b[j], s0);
    t0 = __ffma2_rn(a[j], c[j], t0);
    s1 = __ffma2_rn(a[j + 1], b[j + 1], s1);
    t1 = __ffma2_rn(a[j + 1], c[j + 1], t1);
  }
  return make_float2((s0.x + s0.y) + (s1.x + s1.y), (t0.x + t0.y) + (t1.x + t1.y));
}

// asynchronous global -> shared copies (16 or 4 bytes), counted in groups
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// The inputs of kChunk consecutive rows of one (prompt, head): k and q rows,
// this CTA's 32 entries of v, alpha and beta.  kStages chunks are in flight.
constexpr int kChunk = 16;
constexpr int kStages = 3;
template <typename T, int D>
struct DeltaStage {
  static constexpr int kK = 0;
  static constexpr int kQ = kK + kChunk * D * static_cast<int>(sizeof(T));
  static constexpr int kV = kQ + kChunk * D * static_cast<int>(sizeof(T));
  static constexpr int kLA = kV + kChunk * kDeltaRows * static_cast<int>(sizeof(T));
  static constexpr int kBeta = kLA + kChunk * 4;
  static constexpr int kBytes = kBeta + kChunk * 4;
  static_assert(kQ % 16 == 0 && kV % 16 == 0 && kLA % 16 == 0 && kBytes % 16 == 0, "alignment");
  // the chunk's normalised k^ and q^ rows in fp32 (shared by all rows of the state):
  // each row as 4 column groups of D/4, padded by 4 floats so that the 4 groups'
  // 16-byte reads of a warp fall in different banks; then alpha per row
  static constexpr int kPad = D / 4 + 4;
  static constexpr int kPrepRow = 4 * kPad;
  static constexpr int kPrepBytes = (2 * kChunk * kPrepRow + kChunk) * 4;
};

template <typename T, int D>
__global__ void __launch_bounds__(kDeltaThreads) delta_scan_kernel(const T* __restrict__ q,
                                                                   const T* __restrict__ k,
                                                                   const T* __restrict__ v,
                                                                   T* __restrict__ out,
                                                                   const __grid_constant__ DeltaParams p) {
  using St = DeltaStage<T, D>;
  constexpr int JN = D / 4;  // state columns per thread
  constexpr int kSlices = D / kDeltaRows;
  constexpr int kRow16 = D * static_cast<int>(sizeof(T)) / 16;          // 16-byte pieces of a k/q row
  constexpr int kV16 = kDeltaRows * static_cast<int>(sizeof(T)) / 16;   // of this CTA's v entries
  extern __shared__ __align__(16) uint8_t smem[];
  grid_dep_wait();
  grid_dep_launch();
  const int slice = blockIdx.x % kSlices;
  const int bh = blockIdx.x / kSlices;
  const int h = bh % p.heads, b = bh / p.heads;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row_local = warp * 8 + (lane >> 2);
  const int row = slice * kDeltaRows + row_local;
  const int j0 = (lane & 3) * JN;
  const int t0 = p.kept_start[b], t1 = p.kept_start[b + 1];
  const int n_chunks = (t1 - t0 + kChunk - 1) / kChunk;
  const int64_t H = p.heads;
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  float* const prep_k = reinterpret_cast<float*>(smem + kStages * St::kBytes);
  float* const prep_q = prep_k + kChunk * St::kPrepRow;
  float* const prep_alpha = prep_q + kChunk * St::kPrepRow;

  // copies of chunk c into its stage, spread over the CTA's threads
  auto issue = [&](int c) {
    if (c < n_chunks) {
      const uint32_t st = sbase + (c % kStages) * St::kBytes;
      const int tc0 = t0 + c * kChunk;
      const int rows = min(kChunk, t1 - tc0);
      for (int i = threadIdx.x; i < kChunk * (2 * kRow16 + kV16 + 2); i += kDeltaThreads) {
        const int r = i % kChunk, part = i / kChunk;
        if (r >= rows) continue;
        const int64_t idx = static_cast<int64_t>(tc0 + r) * H + h;
        if (part < kRow16) {
          cp_async16(st + St::kK + (r * kRow16 + part) * 16, reinterpret_cast<const uint8_t*>(k + idx * D) + part * 16);
        } else if (part < 2 * kRow16) {
          const int pq = part - kRow16;
          cp_async16(st + St::kQ + (r * kRow16 + pq) * 16, reinterpret_cast<const uint8_t*>(q + idx * D) + pq * 16);
        } else if (part < 2 * kRow16 + kV16) {
          const int pv = part - 2 * kRow16;
          cp_async16(st + St::kV + (r * kV16 + pv) * 16,
                     reinterpret_cast<const uint8_t*>(v + idx * D + slice * kDeltaRows) + pv * 16);
        } else if (part == 2 * kRow16 + kV16) {
          cp_async4(st + St::kLA + r * 4, p.log_alpha + idx);
        } else {
          cp_async4(st + St::kBeta + r * 4, p.beta + idx);
        }
      }
    }
    cp_async_commit();  // one group per chunk (empty past the end) keeps the count uniform
  };

  float2 S[JN / 2];
#pragma unroll
  for (int j = 0; j < JN / 2; ++j) S[j] = make_float2(0.0f, 0.0f);

#pragma unroll
  for (int c = 0; c < kStages - 1; ++c) issue(c);
  for (int c = 0; c < n_chunks; ++c) {
    cp_async_wait<kStages - 2>();  // this thread's copies of chunk c have landed
    __syncthreads();               // everyone's have, and chunk c - 1 is consumed
    issue(c + kStages - 1);        // into the stage chunk c - 1 used
    const uint8_t* st = smem + (c % kStages) * St::kBytes;
    const T* sk_ = reinterpret_cast<const T*>(st + St::kK);
    const T* sq_ = reinterpret_cast<const T*>(st + St::kQ);
    const T* sv_ = reinterpret_cast<const T*>(st + St::kV);
    const float* sla = reinterpret_cast<const float*>(st + St::kLA);
    const float* sbe = reinterpret_cast<const float*>(st + St::kBeta);
    const int tc0 = t0 + c * kChunk;
    const int rows = min(kChunk, t1 - tc0);
    // k^ = k / |k|, q^ = q / |q| / sqrt(D) and alpha of the chunk's rows, once per
    // CTA: eight lanes per row, each warp four rows at a time
    {
      constexpr int kPer = D / 8;  // elements of a row per lane
      const int r = warp * 4 + (lane >> 3), sub = lane & 7;
      float kv[kPer], qv[kPer];
      float ssk = 0.0f, ssq = 0.0f;
#pragma unroll
      for (int e = 0; e < kPer; ++e) {
        kv[e] = r < rows ? static_cast<float>(sk_[r * D + sub * kPer + e]) : 0.0f;
        qv[e] = r < rows ? static_cast<float>(sq_[r * D + sub * kPer + e]) : 0.0f;
        ssk = fmaf(kv[e], kv[e], ssk);
        ssq = fmaf(qv[e], qv[e], ssq);
      }
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        ssk += __shfl_xor_sync(0xffffffffu, ssk, o);
        ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
      }
      if (r < rows) {
        const float ik = rsqrtf(ssk + p.eps), iq = rsqrtf(ssq + p.eps) * p.q_scale;
        // a lane's kPer columns lie inside one column group (kPer divides JN)
        const int at = r * St::kPrepRow + ((sub * kPer) / JN) * St::kPad + (sub * kPer) % JN;
#pragma unroll
        for (int e = 0; e < kPer; e += 4) {
          *reinterpret_cast<float4*>(prep_k + at + e) =
              make_float4(kv[e] * ik, kv[e + 1] * ik, kv[e + 2] * ik, kv[e + 3] * ik);
          *reinterpret_cast<float4*>(prep_q + at + e) =
              make_float4(qv[e] * iq, qv[e + 1] * iq, qv[e + 2] * iq, qv[e + 3] * iq);
        }
        if (sub == 0) prep_alpha[r] = expf(sla[r]);
      }
    }
    __syncthreads();
    // row r: c_r from (S_{r-1} k^_r), the update, then S_r q^_r together with the
    // next row's S_r k^_{r+1}, so the output's dot product is off the chain
    auto load_row = [&](const float* src, float2 (&x)[JN / 2]) {
      const float4* s4 = reinterpret_cast<const float4*>(src + (lane & 3) * St::kPad);
#pragma unroll
      for (int j = 0; j < JN / 4; ++j) {
        const float4 a = s4[j];
        x[2 * j] = make_float2(a.x, a.y);
        x[2 * j + 1] = make_float2(a.z, a.w);
      }
    };
    float2 kx[JN / 2];
    load_row(prep_k, kx);
    float sk = rowgroup_sum(dot_pairs<JN>(S, kx));  // (S k^)_row for the chunk's first row
    for (int r = 0; r < rows; ++r) {
      float2 qx[JN / 2], kn[JN / 2];
      load_row(prep_q + r * St::kPrepRow, qx);
      const bool more = r + 1 < rows;
      if (more) load_row(prep_k + (r + 1) * St::kPrepRow, kn);
      const float vx = static_cast<float>(sv_[r * kDeltaRows + row_local]);
      const float alpha = prep_alpha[r];
      const float cf = sbe[r] * (vx - alpha * sk);
      const float2 a2 = make_float2(alpha, alpha), c2 = make_float2(cf, cf);
#pragma unroll
      for (int j = 0; j < JN / 2; ++j) S[j] = __ffma2_rn(c2, kx[j], __fmul2_rn(a2, S[j]));
      float o;
      if (more) {
        const float2 d2 = dot2_pairs<JN>(S, qx, kn);
        o = d2.x;
        sk = d2.y;
#pragma unroll
        for (int j = 0; j < JN / 2; ++j) kx[j] = kn[j];
      } else {
        o = dot_pairs<JN>(S, qx);
      }
      o = rowgroup_sum(o);
      if (more) sk = rowgroup_sum(sk);
      if ((lane & 3) == 0) out[(static_cast<int64_t>(tc0 + r) * H + h) * D + row] = to_out(o, out);
    }
  }
  cp_async_wait<0>();  // no copy is still in flight when the CTA exits
  if (p.state) {
    float4* dst = reinterpret_cast<float4*>(p.state + ((static_cast<int64_t>(b) * H + h) * D + row) * D + j0);
#pragma unroll
    for (int j = 0; j < JN / 4; ++j)
      dst[j] = make_float4(S[2 * j].x, S[2 * j].y, S[2 * j + 1].x, S[2 * j + 1].y);
  }
}

template <typename T, int D>
tg_status launch_delta_t(const void* q, const void* k, const void* v, void* out, const DeltaParams& p,
                         int batch, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(kStages) * DeltaStage<T, D>::kBytes + DeltaStage<T, D>::kPrepBytes;
  tg_status r = cuda_check(cudaFuncSetAttribute(delta_scan_kernel<T, D>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                static_cast<int>(smem)),
                           "delta scan smem attribute");
  if (r != TG_OK) return r;
  const dim3 grid(static_cast<unsigned>(batch * p.heads * (D / kDeltaRows))), block(kDeltaThreads);
  return cuda_check(launch_pdl(delta_scan_kernel<T, D>, grid, block, smem, st, static_cast<const T*>(q),
                               static_cast<const T*>(k), static_cast<const T*>(v), static_cast<T*>(out), p),
                    "delta scan launch");
}

}  // namespace

tg_status launch_delta_scan(const void* q, const void* k, const void* v, tg_dtype dt,
                            const float* log_alpha, const float* beta, const PromptTable& pt, int heads,
                            int head_dim, float eps, void* out, float* state, cudaStream_t st) {
  DeltaParams p;
  p.log_alpha = log_alpha;
  p.beta = beta;
  p.state = state;
  for (int i = 0; i <= pt.batch; ++i) p.kept_start[i] = pt.kept_start[i];
  p.heads = heads;
  p.eps = eps;
  p.q_scale = 1.0f / std::sqrt(static_cast<float>(head_dim));
  if (dt == TG_BF16)
    return head_dim == 128 ? launch_delta_t<__nv_bfloat16, 128>(q, k, v, out, p, pt.batch, st)
                           : launch_delta_t<__nv_bfloat16, 64>(q, k, v, out, p, pt.batch, st);
  return head_dim == 128 ? launch_delta_t<float, 128>(q, k, v, out, p, pt.batch, st)
                         : launch_delta_t<float, 64>(q, k, v, out, p, pt.batch, st);
}

}  // namespace tg
