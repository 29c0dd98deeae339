// Gated delta rule in chunked form: the same function as tg_delta.cu's
// recurrence (a Gated DeltaNet layer of a hybrid backbone above the gate, run
// over each prompt's kept rows), computed chunk by chunk so that the work inside
// a chunk is parallel.
//
// With S_0 the state before a chunk of C rows, g_t the product of alpha from the
// chunk's first row through row t, and ratio(t, s) = g_t / g_s (s <= t), the
// recurrence unrolls to
//   u_t = beta_t (v_t - g_t S_0 k^_t - sum_{s<t} ratio(t,s) (k^_s . k^_t) u_s)
//   o_t = g_t S_0 q^_t + sum_{s<=t} ratio(t,s) (k^_s . q^_t) u_s
//   S_C = g_C S_0 + sum_s ratio(C,s) u_s k^_s^T
// The u_t solve a unit lower-triangular system (I + A) U = diag(beta) (V - diag(g)
// K^ S_0^T) with A_ts = beta_t ratio(t,s) k^_t . k^_s (s < t).  Writing T = (I + A)^-1
// and splitting what depends on S_0 from what does not:
//   U   = U_v - W_k S_0^T,         U_v = T diag(beta) V,  W_k = T diag(beta g) K^
//   O   = O_v + Q_e S_0^T,         O_v = M U_v,  Q_e = diag(g) Q^ - M W_k,
//                                  M_ts = ratio(t,s) q^_t . k^_s (s <= t)
//   S_C = g_C S_0 + (U_v - W_k S_0^T)^T K~,   K~ = diag(ratio(C, s)) K^
// delta_chunk_prep_kernel computes U_v, W_k, Q_e, O_v, K~ and g_C for every
// (chunk, head) at once -- none of them depends on the state -- into the
// caller's workspace.  delta_chunk_scan_kernel then runs the short sequential
// part: per (prompt, head, block of 16 state rows), chunk after chunk,
// X = W_k S_0^T and Y = Q_e S_0^T for its rows, o = O_v + Y, and the state
// update.  Rows of S are independent, so the state blocks of a head run on
// different SMs.  All arithmetic is fp32 on the CUDA cores (the state and the
// decays need fp32: the recurrence's results agree to fp32 rounding).
// Decays: ratio(t, s) = exp(P_t - P_s) with P the prefix sum (fp64) of the
// finite log alphas; a row with log alpha = -inf (alpha = 0) between s and t
// makes the ratio exactly 0.
#include <cmath>

#include "tg_internal.cuh"

namespace tg {
namespace {

constexpr int kC = 64;             // rows per chunk
constexpr int kPrepThreads = 256;
constexpr int kScanRows = 16;      // state rows per scan CTA
constexpr int kScanThreads = 256;

// One workspace record per (chunk, head): W_k, Q_e and K~ as [kC][DH] fp32
// (contiguous: the scan loads them with one bulk copy), U_v and O_v as
// [DH / kScanRows][kC][kScanRows] (each scan block's columns contiguous), g_C.
template <int DH>
struct ChunkRec {
  static constexpr int kMat = kC * DH;
  static constexpr int kWk = 0, kQe = kMat, kKt = 2 * kMat, kUv = 3 * kMat, kOv = 4 * kMat;
  static constexpr int kG = 5 * kMat;
  static constexpr int kFloats = 5 * kMat + 64;  // 256-byte multiple
  static constexpr int kSlice = kC * kScanRows;  // one scan block's U_v or O_v columns
  // index of (chunk row t, column c) in U_v / O_v
  static __device__ __forceinline__ int blocked(int t, int c) {
    return (c / kScanRows) * kSlice + t * kScanRows + (c % kScanRows);
  }
};

struct ChunkParams {
  const float* log_alpha;
  const float* beta;
  float* ws;     // [total chunks][heads] records
  float* state;  // [B, H, d, d] or null
  uint32_t* status;
  int32_t kept_start[kMaxBatch + 1];
  int32_t chunk_start[kMaxBatch + 1];  // prefix sums of ceil(M_b / kC)
  int32_t batch;
  int32_t heads;
  float eps;
  float q_scale;  // 1 / sqrt(d)
};

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ void store_out(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_out(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// a . b added to a pair of partial sums (packed fp32x2 FMAs: half the instructions)
__device__ __forceinline__ float2 dot4x2(float4 a, float4 b, float2 acc) {
  acc = __ffma2_rn(make_float2(a.x, a.y), make_float2(b.x, b.y), acc);
  return __ffma2_rn(make_float2(a.z, a.w), make_float2(b.z, b.w), acc);
}

template <int DH>
struct PrepLay {
  static constexpr int LD = DH + 4;  // padded row pitch (floats) of the row matrices
  static constexpr int LC = kC + 4;  // pitch of the chunk x chunk matrices (rows read as float4)
  static constexpr int kK = 0, kQ = kC * LD;
  static constexpr int kA = 2 * kC * LD, kM = kA + kC * LC;
  static constexpr int kBeta = kM + kC * LC, kGam = kBeta + kC, kRho = kGam + kC;
  static constexpr int kP = kRho + kC;  // double[kC] (8-byte aligned: all offsets even)
  static constexpr int kNinf = kP + 2 * kC;
  static constexpr int kFloats = kNinf + kC;
  static constexpr size_t kBytes = static_cast<size_t>(kFloats) * 4;
};

// Prompt of a global chunk index (chunk_start is non-decreasing).
__device__ __forceinline__ int prompt_of_chunk(const ChunkParams& p, int g) {
  int lo = 0, hi = p.batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.chunk_start[mid] <= g) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// 16 bytes of a row as fp32 (8 bf16 or 4 fp32 values)
template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int kN = 8;
  static __device__ __forceinline__ void to_f32(uint4 u, float* f) {
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = __bfloat1622float2(b[i]);
      f[2 * i] = x.x;
      f[2 * i + 1] = x.y;
    }
  }
};
template <>
struct Vec16<float> {
  static constexpr int kN = 4;
  static __device__ __forceinline__ void to_f32(uint4 u, float* f) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
};

// ratio(t, s) = g_t / g_s for s <= t from the prefix sums (0 above the diagonal,
// past the chunk's end, and across a row with alpha = 0)
__device__ __forceinline__ float decay_ratio(const double* sP, const int* sNinf, int n, int t, int s) {
  return (t < n && s <= t && sNinf[t] == sNinf[s]) ? expf(static_cast<float>(sP[t] - sP[s])) : 0.0f;
}

template <typename T, int DH>
__global__ void __launch_bounds__(kPrepThreads, 2) delta_chunk_prep_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const __grid_constant__ ChunkParams p) {
  using L = PrepLay<DH>;
  using R = ChunkRec<DH>;
  using V = Vec16<T>;
  constexpr int LD = L::LD, LC = L::LC;
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  float* sK = sm + L::kK;  // k^ rows
  float* sQ = sm + L::kQ;  // q^ rows
  float* sA = sm + L::kA;
  float* sM = sm + L::kM;
  float* sBeta = sm + L::kBeta;
  float* sGam = sm + L::kGam;
  float* sRho = sm + L::kRho;
  double* sP = reinterpret_cast<double*>(sm + L::kP);
  int* sNinf = reinterpret_cast<int*>(sm + L::kNinf);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.x, h = blockIdx.y, H = p.heads;
  const int b = prompt_of_chunk(p, g);
  const int r0 = p.kept_start[b] + (g - p.chunk_start[b]) * kC;
  const int n = min(kC, p.kept_start[b + 1] - r0);
  float* rec = p.ws + (static_cast<size_t>(g) * H + h) * R::kFloats;

  // rows of q and k as fp32 (16-byte loads), zero past the chunk's end
  constexpr int kVecRow = DH / V::kN;
  for (int idx = tid; idx < kC * kVecRow; idx += kPrepThreads) {
    const int t = idx / kVecRow, c = (idx - t * kVecRow) * V::kN;
    float fk[V::kN], fq[V::kN];
    if (t < n) {
      const size_t off = (static_cast<size_t>(r0 + t) * H + h) * DH + c;
      V::to_f32(__ldg(reinterpret_cast<const uint4*>(k + off)), fk);
      V::to_f32(__ldg(reinterpret_cast<const uint4*>(q + off)), fq);
    } else {
#pragma unroll
      for (int e = 0; e < V::kN; ++e) fk[e] = fq[e] = 0.0f;
    }
#pragma unroll
    for (int e = 0; e < V::kN; e += 4) {
      *reinterpret_cast<float4*>(sK + t * LD + c + e) = make_float4(fk[e], fk[e + 1], fk[e + 2], fk[e + 3]);
      *reinterpret_cast<float4*>(sQ + t * LD + c + e) = make_float4(fq[e], fq[e + 1], fq[e + 2], fq[e + 3]);
    }
  }
  if (tid < kC) {
    const int t = tid;
    sBeta[t] = t < n ? p.beta[static_cast<size_t>(r0 + t) * H + h] : 0.0f;
    sRho[t] = t < n ? p.log_alpha[static_cast<size_t>(r0 + t) * H + h] : 0.0f;  // log alpha, for now
  }
  __syncthreads();
  if (tid == 0) {
    // prefix sums of the finite log alphas (fp64) and counts of alpha = 0 rows
    double P = 0.0;
    int ninf = 0;
    for (int t = 0; t < kC; ++t) {
      const float la = sRho[t];
      if (la == -INFINITY) ++ninf;
      else P += static_cast<double>(la);
      sP[t] = P;
      sNinf[t] = ninf;
    }
  }
  __syncthreads();
  // row norms: k^ = k / sqrt(|k|^2 + eps), q^ = q / sqrt(|q|^2 + eps) / sqrt(d)
  for (int t = warp; t < n; t += kPrepThreads / 32) {
    float ssk = 0.0f, ssq = 0.0f;
    for (int c = lane; c < DH; c += 32) {
      ssk = fmaf(sK[t * LD + c], sK[t * LD + c], ssk);
      ssq = fmaf(sQ[t * LD + c], sQ[t * LD + c], ssq);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ssk += __shfl_xor_sync(0xffffffffu, ssk, o);
      ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
    }
    const float ik = rsqrtf(ssk + p.eps), iq = rsqrtf(ssq + p.eps) * p.q_scale;
    for (int c = lane; c < DH; c += 32) {
      sK[t * LD + c] *= ik;
      sQ[t * LD + c] *= iq;
    }
  }
  // g_t (decay from the chunk's start through t) and g_{n-1} / g_t
  if (tid < kC) {
    const int t = tid;
    sGam[t] = (t < n && sNinf[t] == 0) ? expf(static_cast<float>(sP[t])) : 0.0f;
    sRho[t] = decay_ratio(sP, sNinf, n, n - 1, t);
  }
  __syncthreads();
  // k^_t . k^_s and q^_t . k^_s, 4 x 4 per thread on rows t = bt + 16 i and
  // s = bs + 16 j: the 16 rows s a warp reads at once are consecutive, so they
  // fall in distinct 16-byte bank groups (a pitch of DH + 4 floats); t is one of
  // two rows per warp (a broadcast)
  {
    const int bt = tid >> 4, bs = tid & 15;
    // accumulators paired over the output columns s (j, j + 1): one packed FMA
    // serves two dot products
    float2 ak[4][2], aq[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int jp = 0; jp < 2; ++jp) ak[i][jp] = aq[i][jp] = make_float2(0.0f, 0.0f);
#pragma unroll 1
    for (int d = 0; d < DH; d += 4) {
      float4 kt[4], ks[4], qt[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        kt[i] = *reinterpret_cast<const float4*>(sK + (bt + 16 * i) * LD + d);
        qt[i] = *reinterpret_cast<const float4*>(sQ + (bt + 16 * i) * LD + d);
        ks[i] = *reinterpret_cast<const float4*>(sK + (bs + 16 * i) * LD + d);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jp = 0; jp < 2; ++jp) {
          const float4 s0 = ks[2 * jp], s1 = ks[2 * jp + 1];
          const float2 sx = make_float2(s0.x, s1.x), sy = make_float2(s0.y, s1.y);
          const float2 sz = make_float2(s0.z, s1.z), sw = make_float2(s0.w, s1.w);
          ak[i][jp] = __ffma2_rn(make_float2(kt[i].x, kt[i].x), sx, ak[i][jp]);
          ak[i][jp] = __ffma2_rn(make_float2(kt[i].y, kt[i].y), sy, ak[i][jp]);
          ak[i][jp] = __ffma2_rn(make_float2(kt[i].z, kt[i].z), sz, ak[i][jp]);
          ak[i][jp] = __ffma2_rn(make_float2(kt[i].w, kt[i].w), sw, ak[i][jp]);
          aq[i][jp] = __ffma2_rn(make_float2(qt[i].x, qt[i].x), sx, aq[i][jp]);
          aq[i][jp] = __ffma2_rn(make_float2(qt[i].y, qt[i].y), sy, aq[i][jp]);
          aq[i][jp] = __ffma2_rn(make_float2(qt[i].z, qt[i].z), sz, aq[i][jp]);
          aq[i][jp] = __ffma2_rn(make_float2(qt[i].w, qt[i].w), sw, aq[i][jp]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int t = bt + 16 * i, s = bs + 16 * j;
        const float gts = decay_ratio(sP, sNinf, n, t, s);
        const float kk = (j & 1) ? ak[i][j >> 1].y : ak[i][j >> 1].x;
        const float qk = (j & 1) ? aq[i][j >> 1].y : aq[i][j >> 1].x;
        sA[t * LC + s] = s < t ? sBeta[t] * gts * kk : 0.0f;
        sM[t * LC + s] = gts * qk;
      }
  }
  __syncthreads();
  // One column per thread, kept in registers from the solve to the products:
  // threads [0, DH) solve (I + A) U_v = diag(beta) V for column c and then form
  // O_v = M U_v; threads [DH, 2 DH) solve (I + A) W_k = diag(beta g) K^ and form
  // Q_e = diag(g) Q^ - M W_k (they also write K~ = diag(ratio(C, s)) K^ from their
  // column first).  Forward substitution: x_t = r_t - sum_{s<t} A_ts x_s.
  if (tid < 2 * DH) {
    const bool wk = tid >= DH;
    const int c = wk ? tid - DH : tid;
    float x[kC];
    if (wk) {
#pragma unroll
      for (int t = 0; t < kC; ++t) {
        const float e = sK[t * LD + c];
        x[t] = sBeta[t] * sGam[t] * e;
        rec[R::kKt + t * DH + c] = sRho[t] * e;
      }
    } else {
#pragma unroll
      for (int t = 0; t < kC; ++t)
        x[t] = t < n ? sBeta[t] * to_f32(v[(static_cast<size_t>(r0 + t) * H + h) * DH + c]) : 0.0f;
    }
    // rows of A and M are the same for every thread: float4 broadcast reads
#pragma unroll
    for (int t = 1; t < kC; ++t) {
      float a0 = x[t], a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
      const float* arow = sA + t * LC;
#pragma unroll
      for (int s = 0; s + 3 < t; s += 4) {
        const float4 a = *reinterpret_cast<const float4*>(arow + s);
        a0 = fmaf(-a.x, x[s], a0);
        a1 = fmaf(-a.y, x[s + 1], a1);
        a2 = fmaf(-a.z, x[s + 2], a2);
        a3 = fmaf(-a.w, x[s + 3], a3);
      }
#pragma unroll
      for (int s = t & ~3; s < t; ++s) a0 = fmaf(-arow[s], x[s], a0);
      x[t] = (a0 + a1) + (a2 + a3);
    }
#pragma unroll
    for (int t = 0; t < kC; ++t) {
      if (wk) rec[R::kWk + t * DH + c] = x[t];
      else rec[R::kUv + R::blocked(t, c)] = x[t];
      const float* mrow = sM + t * LC;
      float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll
      for (int s = 0; s + 3 <= t; s += 4) {
        const float4 mv = *reinterpret_cast<const float4*>(mrow + s);
        a0 = fmaf(mv.x, x[s], a0);
        a1 = fmaf(mv.y, x[s + 1], a1);
        a2 = fmaf(mv.z, x[s + 2], a2);
        a3 = fmaf(mv.w, x[s + 3], a3);
      }
#pragma unroll
      for (int s = (t + 1) & ~3; s <= t; ++s) a0 = fmaf(mrow[s], x[s], a0);
      const float acc = (a0 + a1) + (a2 + a3);
      if (wk) rec[R::kQe + t * DH + c] = fmaf(sGam[t], sQ[t * LD + c], -acc);
      else rec[R::kOv + R::blocked(t, c)] = acc;
    }
  }
  if (tid == 0) rec[R::kG] = n > 0 ? sGam[n - 1] : 1.0f;
}

template <int DH>
struct ScanLay {
  static constexpr int LS = DH + 4;               // state rows (padded: 16 rows read at once)
  static constexpr int kMat = kC * DH;            // W_k, Q_e, K~ unpadded
  static constexpr int kStage = 3 * kMat + 2 * kC * kScanRows;  // + U_v, O_v columns
  static constexpr int kS = 2 * kStage;
  static constexpr int kD = kS + kScanRows * LS;  // [kC][kScanRows + 1]
  static constexpr int kFloats = kD + kC * (kScanRows + 1);
  static constexpr size_t kBytes = static_cast<size_t>(kFloats) * 4;
};

template <typename T, int DH>
__global__ void __launch_bounds__(kScanThreads) delta_chunk_scan_kernel(
    T* __restrict__ out, const __grid_constant__ ChunkParams p) {
  using L = ScanLay<DH>;
  using R = ChunkRec<DH>;
  constexpr int LS = L::LS;
  constexpr int NC = DH / 16;  // state columns per thread in the update (4 or 8)
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  float* sS = sm + L::kS;
  float* sD = sm + L::kD;
  const int tid = threadIdx.x;
  const int i0 = blockIdx.x * kScanRows, h = blockIdx.y, b = blockIdx.z, H = p.heads;
  const int c_first = p.chunk_start[b], n_chunks = p.chunk_start[b + 1] - c_first;
  const int row0 = p.kept_start[b], len = p.kept_start[b + 1] - row0;
  __shared__ uint64_t s_full[2];  // stage s holds chunks s, s + 2, ...
  __shared__ int s_abort;
  if (tid == 0) {
    mbar_init(smem_u32(&s_full[0]), 1);
    mbar_init(smem_u32(&s_full[1]), 1);
    s_abort = 0;
    mbar_fence_init();
  }
  __syncthreads();

  // Thread 0: chunk c's W_k, Q_e and K~ (one bulk copy) and this block's U_v and
  // O_v columns (one each) into stage c & 1.  Every thread has finished reading
  // that stage (the barrier at the end of the previous chunk).
  constexpr uint32_t kMatsBytes = 3 * R::kMat * 4, kSliceBytes = R::kSlice * 4;
  auto load_chunk = [&](int c) {
    const float* rec = p.ws + (static_cast<size_t>(c_first + c) * H + h) * R::kFloats;
    const uint32_t sb = smem_u32(sm + (c & 1) * L::kStage), bar = smem_u32(&s_full[c & 1]);
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, kMatsBytes + 2 * kSliceBytes);
    bulk_g2s(sb, rec, kMatsBytes, bar);
    bulk_g2s(sb + kMatsBytes, rec + R::kUv + blockIdx.x * R::kSlice, kSliceBytes, bar);
    bulk_g2s(sb + kMatsBytes + kSliceBytes, rec + R::kOv + blockIdx.x * R::kSlice, kSliceBytes, bar);
  };

  // update mapping: thread owns state row ru and the float4 column groups
  // cu + 64 m (m < NC / 4): the 16 threads of a row read 16 consecutive float4
  // of a K~ row (two bank-conflict-free wavefronts per load)
  const int ru = tid >> 4, cu = (tid & 15) * 4;
  // product mapping: thread owns chunk rows tg + 16 i (i < 4) of state row rp: a
  // warp reads two consecutive rows of W_k / Q_e at once (a broadcast)
  const int tg = tid >> 4, rp = tid & 15;
  float sreg[NC];
#pragma unroll
  for (int j = 0; j < NC; ++j) sreg[j] = 0.0f;
#pragma unroll
  for (int m = 0; m < NC / 4; ++m)
    *reinterpret_cast<float4*>(sS + ru * LS + cu + 64 * m) = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  if (tid == 0 && n_chunks > 0) load_chunk(0);
  int loaded = n_chunks > 0 ? 1 : 0;  // chunks whose load was issued
  bool ok = true;
  for (int c = 0; c < n_chunks; ++c) {
    if (tid == 0 && c + 1 < n_chunks) load_chunk(c + 1);
    loaded = min(c + 2, n_chunks);
    const bool landed =
        mbar_wait(smem_u32(&s_full[c & 1]), (c >> 1) & 1, &s_abort, p.status, kDevTimeoutDelta);
    if (__syncthreads_or(!landed)) {  // one way out for the whole CTA
      ok = false;
      break;
    }
    const float* st = sm + (c & 1) * L::kStage;
    const float* sW = st;
    const float* sQe = st + R::kMat;
    const float* sKt = st + 2 * R::kMat;
    const float* sUv = st + 3 * R::kMat;
    const float* sOv = sUv + kC * kScanRows;
    const float gC = __ldg(p.ws + (static_cast<size_t>(c_first + c) * H + h) * R::kFloats + R::kG);
    // X = W_k S^T and Y = Q_e S^T for this thread's 4 chunk rows and state row rp
    float2 ax2[4], ay2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) ax2[i] = ay2[i] = make_float2(0.0f, 0.0f);
#pragma unroll 4
    for (int d = 0; d < DH; d += 4) {
      const float4 s4 = *reinterpret_cast<const float4*>(sS + rp * LS + d);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ax2[i] = dot4x2(*reinterpret_cast<const float4*>(sW + (tg + 16 * i) * DH + d), s4, ax2[i]);
        ay2[i] = dot4x2(*reinterpret_cast<const float4*>(sQe + (tg + 16 * i) * DH + d), s4, ay2[i]);
      }
    }
    float ax[4], ay[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      ax[i] = ax2[i].x + ax2[i].y;
      ay[i] = ay2[i].x + ay2[i].y;
    }
    const int t0 = c * kC;  // chunk rows within the prompt
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = tg + 16 * i;
      sD[t * (kScanRows + 1) + rp] = sUv[t * kScanRows + rp] - ax[i];
      if (t0 + t < len)
        store_out(out + (static_cast<size_t>(row0 + t0 + t) * H + h) * DH + i0 + rp,
                  sOv[t * kScanRows + rp] + ay[i]);
    }
    __syncthreads();
    // S <- g_C S + (U_v - X)^T K~ for this thread's row and columns
#pragma unroll
    for (int j = 0; j < NC; ++j) sreg[j] *= gC;
#pragma unroll 4
    for (int t = 0; t < kC; ++t) {
      const float dd = sD[t * (kScanRows + 1) + ru];
      const float2 d2 = make_float2(dd, dd);
#pragma unroll
      for (int m = 0; m < NC / 4; ++m) {
        const float4 kt = *reinterpret_cast<const float4*>(sKt + t * DH + cu + 64 * m);
        const float2 lo = __ffma2_rn(d2, make_float2(kt.x, kt.y), make_float2(sreg[4 * m], sreg[4 * m + 1]));
        const float2 hi = __ffma2_rn(d2, make_float2(kt.z, kt.w), make_float2(sreg[4 * m + 2], sreg[4 * m + 3]));
        sreg[4 * m] = lo.x;
        sreg[4 * m + 1] = lo.y;
        sreg[4 * m + 2] = hi.x;
        sreg[4 * m + 3] = hi.y;
      }
    }
#pragma unroll
    for (int m = 0; m < NC / 4; ++m)
      *reinterpret_cast<float4*>(sS + ru * LS + cu + 64 * m) =
          make_float4(sreg[4 * m], sreg[4 * m + 1], sreg[4 * m + 2], sreg[4 * m + 3]);
    __syncthreads();  // state and stage free for the next chunk
  }
  if (!ok) {
    // a load did not land in time: wait (bounded) for every load in flight before
    // the shared memory is released; the outputs are undefined
    if (tid == 0)
      for (int c = 0; c < loaded; ++c) mbar_drain(smem_u32(&s_full[c & 1]), (c >> 1) & 1);
    __syncthreads();
    return;
  }
  if (p.state) {
    float* dst = p.state + ((static_cast<size_t>(b) * H + h) * DH + i0 + ru) * DH + cu;
#pragma unroll
    for (int m = 0; m < NC / 4; ++m)
      *reinterpret_cast<float4*>(dst + 64 * m) =
          make_float4(sreg[4 * m], sreg[4 * m + 1], sreg[4 * m + 2], sreg[4 * m + 3]);
  }
}

template <typename T, int DH>
tg_status launch_chunked_t(const void* q, const void* k, const void* v, void* out,
                           const ChunkParams& p, int total_chunks, cudaStream_t st) {
  using PL = PrepLay<DH>;
  using SL = ScanLay<DH>;
  tg_status r = cuda_check(cudaFuncSetAttribute(delta_chunk_prep_kernel<T, DH>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                static_cast<int>(PL::kBytes)),
                           "delta prep smem attribute");
  if (r != TG_OK) return r;
  r = cuda_check(cudaFuncSetAttribute(delta_chunk_scan_kernel<T, DH>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(SL::kBytes)),
                 "delta scan smem attribute");
  if (r != TG_OK) return r;
  if (total_chunks > 0) {
    delta_chunk_prep_kernel<T, DH><<<dim3(total_chunks, p.heads), kPrepThreads, PL::kBytes, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), p);
    r = cuda_check(cudaGetLastError(), "delta prep launch");
    if (r != TG_OK) return r;
  }
  delta_chunk_scan_kernel<T, DH><<<dim3(DH / kScanRows, p.heads, p.batch), kScanThreads, SL::kBytes,
                                   st>>>(static_cast<T*>(out), p);
  return cuda_check(cudaGetLastError(), "delta scan launch");
}

int64_t total_chunks_of(const PromptTable& pt) {
  int64_t n = 0;
  for (int b = 0; b < pt.batch; ++b) n += (pt.kept_start[b + 1] - pt.kept_start[b] + kC - 1) / kC;
  return n;
}

}  // namespace

size_t delta_chunked_workspace_bytes(const PromptTable& pt, int heads, int head_dim) {
  const int64_t recs = total_chunks_of(pt) * heads;
  const int64_t floats = head_dim == 128 ? ChunkRec<128>::kFloats : ChunkRec<64>::kFloats;
  return static_cast<size_t>(recs) * static_cast<size_t>(floats) * sizeof(float);
}

tg_status launch_delta_chunked(const void* q, const void* k, const void* v, tg_dtype dt,
                               const float* log_alpha, const float* beta, const PromptTable& pt,
                               int heads, int head_dim, float eps, void* out, float* state,
                               void* workspace, cudaStream_t st) {
  ChunkParams p;
  memset(&p, 0, sizeof(p));
  p.log_alpha = log_alpha;
  p.beta = beta;
  p.ws = static_cast<float*>(workspace);
  p.state = state;
  p.status = device_status_word();
  if (!p.status) return set_error(TG_ERR_CUDA, "device status word unavailable");
  p.batch = pt.batch;
  p.heads = heads;
  p.eps = eps;
  p.q_scale = 1.0f / std::sqrt(static_cast<float>(head_dim));
  int64_t chunks = 0;
  for (int b = 0; b <= pt.batch; ++b) {
    p.kept_start[b] = pt.kept_start[b];
    p.chunk_start[b] = static_cast<int32_t>(chunks);
    if (b < pt.batch) chunks += (pt.kept_start[b + 1] - pt.kept_start[b] + kC - 1) / kC;
  }
  if (chunks > 0x7FFFFFFF) return set_error(TG_ERR_UNSUPPORTED, "too many chunks");
  const int tc = static_cast<int>(chunks);
  if (dt == TG_BF16)
    return head_dim == 128 ? launch_chunked_t<__nv_bfloat16, 128>(q, k, v, out, p, tc, st)
                           : launch_chunked_t<__nv_bfloat16, 64>(q, k, v, out, p, tc, st);
  return head_dim == 128 ? launch_chunked_t<float, 128>(q, k, v, out, p, tc, st)
                         : launch_chunked_t<float, 64>(q, k, v, out, p, tc, st);
}

}  // namespace tg
