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

// One workspace record per (chunk, head), fp32: W_k and Q_e transposed, [DH][kC]
// (the scan reads 4 consecutive chunk rows of one column at once), K~ as
// [kC][DH], U_v and O_v as [DH / kScanRows][kC][kScanRows] (each scan block's
// columns contiguous), g_C.
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

__device__ __forceinline__ void store_out(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_out(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

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

  // rows of q and k (16-byte loads, all in flight at once), normalised on the
  // way into shared memory: k^ = k / sqrt(|k|^2 + eps), q^ = q / sqrt(|q|^2 + eps)
  // / sqrt(d).  A row's vectors sit in kVecRow consecutive lanes, so its squared
  // norm is a shuffle reduction.  Rows past the chunk's end are zero.
  constexpr int kVecRow = DH / V::kN;
  constexpr int kIters = kC * kVecRow / kPrepThreads;
  static_assert(kC * kVecRow % kPrepThreads == 0 && 32 % kVecRow == 0, "row vectors per warp");
  uint4 ku[kIters], qu[kIters];
#pragma unroll
  for (int u = 0; u < kIters; ++u) {
    const int idx = tid + u * kPrepThreads;
    const int t = idx / kVecRow, c = (idx - t * kVecRow) * V::kN;
    ku[u] = qu[u] = make_uint4(0u, 0u, 0u, 0u);
    if (t < n) {
      const size_t off = (static_cast<size_t>(r0 + t) * H + h) * DH + c;
      ku[u] = __ldg(reinterpret_cast<const uint4*>(k + off));
      qu[u] = __ldg(reinterpret_cast<const uint4*>(q + off));
    }
  }
  if (tid < kC) {
    const int t = tid;
    sBeta[t] = t < n ? p.beta[static_cast<size_t>(r0 + t) * H + h] : 0.0f;
    sRho[t] = t < n ? p.log_alpha[static_cast<size_t>(r0 + t) * H + h] : 0.0f;  // log alpha, for now
  }
#pragma unroll
  for (int u = 0; u < kIters; ++u) {
    const int idx = tid + u * kPrepThreads;
    const int t = idx / kVecRow, c = (idx - t * kVecRow) * V::kN;
    float fk[V::kN], fq[V::kN];
    V::to_f32(ku[u], fk);
    V::to_f32(qu[u], fq);
    float ssk = 0.0f, ssq = 0.0f;
#pragma unroll
    for (int e = 0; e < V::kN; ++e) {
      ssk = fmaf(fk[e], fk[e], ssk);
      ssq = fmaf(fq[e], fq[e], ssq);
    }
#pragma unroll
    for (int o = kVecRow / 2; o > 0; o >>= 1) {
      ssk += __shfl_xor_sync(0xffffffffu, ssk, o);
      ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
    }
    // rows past the chunk's end stay zero (with eps = 0 their scale would be inf)
    const float ik = t < n ? rsqrtf(ssk + p.eps) : 0.0f;
    const float iq = t < n ? rsqrtf(ssq + p.eps) * p.q_scale : 0.0f;
#pragma unroll
    for (int e = 0; e < V::kN; e += 4) {
      *reinterpret_cast<float4*>(sK + t * LD + c + e) =
          make_float4(fk[e] * ik, fk[e + 1] * ik, fk[e + 2] * ik, fk[e + 3] * ik);
      *reinterpret_cast<float4*>(sQ + t * LD + c + e) =
          make_float4(fq[e] * iq, fq[e + 1] * iq, fq[e + 2] * iq, fq[e + 3] * iq);
    }
  }
  __syncthreads();
  if (warp == 0) {
    // prefix sums of the finite log alphas (fp64) and counts of alpha = 0 rows:
    // two rows per lane, then a scan over the warp
    static_assert(kC == 64, "two chunk rows per lane");
    const float l0 = sRho[2 * lane], l1 = sRho[2 * lane + 1];
    const double d0 = l0 == -INFINITY ? 0.0 : static_cast<double>(l0);
    const double d1 = l1 == -INFINITY ? 0.0 : static_cast<double>(l1);
    const int i0 = l0 == -INFINITY ? 1 : 0, i1 = l1 == -INFINITY ? 1 : 0;
    double P = d0 + d1;
    int ni = i0 + i1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double yP = __shfl_up_sync(0xffffffffu, P, o);
      const int yn = __shfl_up_sync(0xffffffffu, ni, o);
      if (lane >= o) {
        P += yP;
        ni += yn;
      }
    }
    sP[2 * lane] = P - d1;
    sP[2 * lane + 1] = P;
    sNinf[2 * lane] = ni - i1;
    sNinf[2 * lane + 1] = ni;
  }
  __syncthreads();
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
  // V reaches shared memory (over K^, once read) with coalesced 16-byte loads;
  // W_k (over V, once read) and Q_e (over Q^, element by element) leave it for
  // the record transposed, with coalesced stores.
  const bool col = tid < 2 * DH, wk = tid >= DH;
  const int c = wk ? tid - DH : tid;
  float x[kC];
  if (col && wk) {
#pragma unroll
    for (int t = 0; t < kC; ++t) {
      const float e = sK[t * LD + c];
      x[t] = sBeta[t] * sGam[t] * e;
      rec[R::kKt + t * DH + c] = sRho[t] * e;
    }
  }
  __syncthreads();  // K^ is read: its rows take V
  float* sV = sK;
  {
    uint4 vu[kIters];
#pragma unroll
    for (int u = 0; u < kIters; ++u) {
      const int idx = tid + u * kPrepThreads;
      const int t = idx / kVecRow, cc = (idx - t * kVecRow) * V::kN;
      vu[u] = make_uint4(0u, 0u, 0u, 0u);
      if (t < n)
        vu[u] = __ldg(reinterpret_cast<const uint4*>(v + (static_cast<size_t>(r0 + t) * H + h) * DH + cc));
    }
#pragma unroll
    for (int u = 0; u < kIters; ++u) {
      const int idx = tid + u * kPrepThreads;
      const int t = idx / kVecRow, cc = (idx - t * kVecRow) * V::kN;
      float fv[V::kN];
      V::to_f32(vu[u], fv);
#pragma unroll
      for (int e = 0; e < V::kN; e += 4)
        *reinterpret_cast<float4*>(sV + t * LD + cc + e) = make_float4(fv[e], fv[e + 1], fv[e + 2], fv[e + 3]);
    }
  }
  __syncthreads();
  if (col && !wk) {
#pragma unroll
    for (int t = 0; t < kC; ++t) x[t] = sBeta[t] * sV[t * LD + c];  // zero past the chunk's end
  }
  __syncthreads();  // V is read: its rows take W_k
  if (col) {
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
    if (wk) {
#pragma unroll
      for (int t = 0; t < kC; ++t) sV[t * LD + c] = x[t];
    }
#pragma unroll
    for (int t = 0; t < kC; ++t) {
      if (!wk) rec[R::kUv + R::blocked(t, c)] = x[t];
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
      if (wk) sQ[t * LD + c] = fmaf(sGam[t], sQ[t * LD + c], -acc);  // Q_e over Q^
      else rec[R::kOv + R::blocked(t, c)] = acc;
    }
  }
  __syncthreads();
  // W_k^T and Q_e^T: a thread takes four consecutive chunk rows of one column,
  // so 16 consecutive threads write one 256-byte row of the transposed matrix
  for (int i = tid; i < DH * (kC / 4); i += kPrepThreads) {
    const int cc = i / (kC / 4), t4 = (i - cc * (kC / 4)) * 4;
    *reinterpret_cast<float4*>(rec + R::kWk + cc * kC + t4) =
        make_float4(sV[t4 * LD + cc], sV[(t4 + 1) * LD + cc], sV[(t4 + 2) * LD + cc], sV[(t4 + 3) * LD + cc]);
    *reinterpret_cast<float4*>(rec + R::kQe + cc * kC + t4) =
        make_float4(sQ[t4 * LD + cc], sQ[(t4 + 1) * LD + cc], sQ[(t4 + 2) * LD + cc], sQ[(t4 + 3) * LD + cc]);
  }
  if (tid == 0) rec[R::kG] = n > 0 ? sGam[n - 1] : 1.0f;
}

// Scan CTA (prompt, head, block of kScanRows state rows), per chunk:
//   1. X = W_k S^T and Y = Q_e S^T for the block's rows: a thread owns 4 chunk
//      rows x 4 state rows of both over a quarter of d (W_k^T, Q_e^T and the
//      transposed state give it a float4 of each per d), then the quarters are
//      summed; D = U_v - X goes to shared memory, O_v + Y to the output.
//   2. S <- g_C S + D^T K~: a thread owns 4 state rows x 4 columns over a share
//      of the chunk rows, the shares are summed by the threads that keep S in
//      registers across chunks, which also write S^T for the next chunk.
// W_k^T and Q_e^T of the next chunk load (one bulk copy) while this chunk's
// update runs; K~ and the U_v / O_v columns are double-buffered.
template <int DH>
struct ScanLay {
  static constexpr int R = kScanRows;
  static constexpr int kWQ = 0;                       // W_k^T, Q_e^T: [2][DH][kC]
  static constexpr int kK = kWQ + 2 * DH * kC;        // K~: [2 buffers][kC][DH]
  static constexpr int kUO = kK + 2 * kC * DH;        // U_v, O_v columns: [2 buffers][2][kC][R]
  static constexpr int kSt = kUO + 2 * 2 * kC * R;    // S^T of the block: [DH][R]
  static constexpr int LDD = R + 4;                   // D pitch (float4 rows)
  static constexpr int kD = kSt + DH * R;             // D = U_v - X: [kC][LDD]
  static constexpr int kUpd = 4 * (DH / 4);           // update threads per chunk-row share
  static constexpr int kTs = kScanThreads / kUpd;     // shares (2 at d = 128, 4 at d = 64)
  static constexpr int kRedXY = 4 * 64 * 32;          // partial X, Y of the four quarters
  static constexpr int kRedS = (kTs - 1) * kUpd * 16; // partial updates of shares 1..
  static constexpr int kRed = kD + kC * LDD;
  static constexpr int kFloats = kRed + (kRedXY > kRedS ? kRedXY : kRedS);
  static constexpr size_t kBytes = static_cast<size_t>(kFloats) * 4;
  static_assert(kScanThreads == 256 && kC == 64 && R == 16, "thread mapping");
  static_assert(kBytes <= 227 * 1024, "shared memory");
};

template <typename T, int DH>
__global__ void __launch_bounds__(kScanThreads, 1) delta_chunk_scan_kernel(
    T* __restrict__ out, const __grid_constant__ ChunkParams p) {
  using L = ScanLay<DH>;
  using R = ChunkRec<DH>;
  constexpr int RS = kScanRows;
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  float* sWT = sm + L::kWQ;
  float* sQT = sWT + DH * kC;
  float* sSt = sm + L::kSt;
  float* sD = sm + L::kD;
  float* sRed = sm + L::kRed;
  const int tid = threadIdx.x;
  const int i0 = blockIdx.x * RS, h = blockIdx.y, b = blockIdx.z, H = p.heads;
  const int c_first = p.chunk_start[b], n_chunks = p.chunk_start[b + 1] - c_first;
  const int row0 = p.kept_start[b], len = p.kept_start[b + 1] - row0;
  __shared__ uint64_t s_wq, s_k[2];  // W_k^T, Q_e^T and the U_v / O_v columns; K~ per buffer
  __shared__ int s_abort;
  if (tid == 0) {
    mbar_init(smem_u32(&s_wq), 1);
    mbar_init(smem_u32(&s_k[0]), 1);
    mbar_init(smem_u32(&s_k[1]), 1);
    s_abort = 0;
    mbar_fence_init();
  }
  auto rec_of = [&](int c) { return p.ws + (static_cast<size_t>(c_first + c) * H + h) * R::kFloats; };
  // Thread 0 issues the loads; every thread has finished reading the target
  // buffer (a barrier precedes each call).
  int wq_loads = 0, k_loads[2] = {0, 0};  // thread 0: for the drain after an abort
  constexpr uint32_t kWQBytes = 2 * DH * kC * 4, kKBytes = kC * DH * 4, kSliceBytes = R::kSlice * 4;
  auto load_wq = [&](int c) {
    const float* rec = rec_of(c);
    const uint32_t bar = smem_u32(&s_wq);
    float* uo = sm + L::kUO + (c & 1) * 2 * kC * RS;
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, kWQBytes + 2 * kSliceBytes);
    bulk_g2s(smem_u32(sWT), rec + R::kWk, kWQBytes, bar);  // W_k^T and Q_e^T are adjacent
    bulk_g2s(smem_u32(uo), rec + R::kUv + blockIdx.x * R::kSlice, kSliceBytes, bar);
    bulk_g2s(smem_u32(uo + kC * RS), rec + R::kOv + blockIdx.x * R::kSlice, kSliceBytes, bar);
    ++wq_loads;
  };
  auto load_k = [&](int c) {
    const uint32_t bar = smem_u32(&s_k[c & 1]);
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, kKBytes);
    bulk_g2s(smem_u32(sm + L::kK + (c & 1) * kC * DH), rec_of(c) + R::kKt, kKBytes, bar);
    ++k_loads[c & 1];
  };

  // product mapping: quarter dq of d; within it, a warp covers 8 chunk-row groups
  // (4 rows each, consecutive) x 4 state-row groups (4 rows each)
  const int dq = tid >> 6, w64 = tid & 63;
  const int tq = ((w64 >> 5) << 3) | (w64 & 7), rq = (w64 >> 3) & 3;
  // update mapping: share ts of the chunk rows; a warp covers consecutive
  // column groups of one (d = 128) or two (d = 64) state-row groups
  constexpr int kCq = DH / 4;
  const int ts = tid / L::kUpd, u = tid % L::kUpd;
  const int cq = u % kCq, ru = u / kCq;
  float sreg[16];  // S rows 4 ru + i, columns 4 cq + j (threads of share 0)
#pragma unroll
  for (int e = 0; e < 16; ++e) sreg[e] = 0.0f;
  for (int e = tid; e < DH * RS; e += kScanThreads) sSt[e] = 0.0f;
  __syncthreads();
  if (tid == 0 && n_chunks > 0) {
    load_wq(0);
    load_k(0);
    if (n_chunks > 1) load_k(1);
  }
  bool ok = true;
  for (int c = 0; c < n_chunks; ++c) {
    const float* uo = sm + L::kUO + (c & 1) * 2 * kC * RS;
    const float* sUv = uo;
    const float* sOv = uo + kC * RS;
    const float* sKt = sm + L::kK + (c & 1) * kC * DH;
    const float gC = __ldg(rec_of(c) + R::kG);
    // ---- X and Y ------------------------------------------------------------
    bool landed = mbar_wait(smem_u32(&s_wq), c & 1, &s_abort, p.status, kDevTimeoutDelta);
    if (__syncthreads_or(!landed)) {
      ok = false;
      break;
    }
    float2 ax[4][2], ay[4][2];  // [chunk row i][state rows (2 jp, 2 jp + 1)]
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int jp = 0; jp < 2; ++jp) ax[i][jp] = ay[i][jp] = make_float2(0.0f, 0.0f);
    {
      constexpr int kDq = DH / 4;
      const float* wt = sWT + (dq * kDq) * kC + 4 * tq;
      const float* qt = sQT + (dq * kDq) * kC + 4 * tq;
      const float* st = sSt + (dq * kDq) * RS + 4 * rq;
#pragma unroll 4
      for (int d = 0; d < kDq; ++d) {
        const float4 w4 = *reinterpret_cast<const float4*>(wt + d * kC);
        const float4 q4 = *reinterpret_cast<const float4*>(qt + d * kC);
        const float4 s4 = *reinterpret_cast<const float4*>(st + d * RS);
        const float2 s01 = make_float2(s4.x, s4.y), s23 = make_float2(s4.z, s4.w);
        const float wv[4] = {w4.x, w4.y, w4.z, w4.w}, qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          ax[i][0] = __ffma2_rn(make_float2(wv[i], wv[i]), s01, ax[i][0]);
          ax[i][1] = __ffma2_rn(make_float2(wv[i], wv[i]), s23, ax[i][1]);
          ay[i][0] = __ffma2_rn(make_float2(qv[i], qv[i]), s01, ay[i][0]);
          ay[i][1] = __ffma2_rn(make_float2(qv[i], qv[i]), s23, ay[i][1]);
        }
      }
    }
    // every quarter hands its partial sums over (one column per value:
    // consecutive threads, consecutive words); quarter dq then finishes chunk
    // row 4 tq + dq of the block, summing the four quarters' partials
    {
      float* red = sRed + dq * 32 * 64 + w64;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jp = 0; jp < 2; ++jp) {
          red[((i * 2 + jp) * 2 + 0) * 64] = ax[i][jp].x;
          red[((i * 2 + jp) * 2 + 1) * 64] = ax[i][jp].y;
          red[(16 + (i * 2 + jp) * 2 + 0) * 64] = ay[i][jp].x;
          red[(16 + (i * 2 + jp) * 2 + 1) * 64] = ay[i][jp].y;
        }
    }
    __syncthreads();  // W_k^T and Q_e^T are read: the next chunk's may load
    if (tid == 0 && c + 1 < n_chunks) load_wq(c + 1);
    {
      float xs[4] = {0.0f, 0.0f, 0.0f, 0.0f}, ys[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const float* red = sRed + q4 * 32 * 64 + w64;
#pragma unroll
        for (int e = 0; e < 4; ++e) {  // state row 4 rq + e: accumulator (dq * 2 + e / 2) * 2 + e % 2
          xs[e] += red[(dq * 4 + e) * 64];
          ys[e] += red[(16 + dq * 4 + e) * 64];
        }
      }
      const int t = 4 * tq + dq, t0 = c * kC;
      const float4 uv = *reinterpret_cast<const float4*>(sUv + t * RS + 4 * rq);
      const float4 ov = *reinterpret_cast<const float4*>(sOv + t * RS + 4 * rq);
      *reinterpret_cast<float4*>(sD + t * L::LDD + 4 * rq) =
          make_float4(uv.x - xs[0], uv.y - xs[1], uv.z - xs[2], uv.w - xs[3]);
      if (t0 + t < len) {
        T* o = out + (static_cast<size_t>(row0 + t0 + t) * H + h) * DH + i0 + 4 * rq;
        store_out(o + 0, ov.x + ys[0]);
        store_out(o + 1, ov.y + ys[1]);
        store_out(o + 2, ov.z + ys[2]);
        store_out(o + 3, ov.w + ys[3]);
      }
    }
    // ---- S <- g_C S + D^T K~ ---------------------------------------------------
    landed = mbar_wait(smem_u32(&s_k[c & 1]), (c >> 1) & 1, &s_abort, p.status, kDevTimeoutDelta);
    if (__syncthreads_or(!landed)) {  // also: D is complete
      ok = false;
      break;
    }
    float2 acc[4][2];  // [state row i][columns (2 jp, 2 jp + 1)]
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = make_float2(0.0f, 0.0f);
    {
      constexpr int kTper = kC / L::kTs;
      const float* dr = sD + (ts * kTper) * L::LDD + 4 * ru;
      const float* kr = sKt + (ts * kTper) * DH + 4 * cq;
#pragma unroll 4
      for (int t = 0; t < kTper; ++t) {
        const float4 d4 = *reinterpret_cast<const float4*>(dr + t * L::LDD);
        const float4 k4 = *reinterpret_cast<const float4*>(kr + t * DH);
        const float2 k01 = make_float2(k4.x, k4.y), k23 = make_float2(k4.z, k4.w);
        const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[i][0] = __ffma2_rn(make_float2(dv[i], dv[i]), k01, acc[i][0]);
          acc[i][1] = __ffma2_rn(make_float2(dv[i], dv[i]), k23, acc[i][1]);
        }
      }
    }
    if (ts > 0) {
      float* red = sRed + (ts - 1) * 16 * L::kUpd + u;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        red[(i * 4 + 0) * L::kUpd] = acc[i][0].x;
        red[(i * 4 + 1) * L::kUpd] = acc[i][0].y;
        red[(i * 4 + 2) * L::kUpd] = acc[i][1].x;
        red[(i * 4 + 3) * L::kUpd] = acc[i][1].y;
      }
    }
    __syncthreads();  // K~ of this buffer is read: the chunk after next may load
    if (tid == 0 && c + 2 < n_chunks) load_k(c + 2);
    if (ts == 0) {
#pragma unroll
      for (int s2 = 1; s2 < L::kTs; ++s2) {
        const float* red = sRed + (s2 - 1) * 16 * L::kUpd + u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[i][0].x += red[(i * 4 + 0) * L::kUpd];
          acc[i][0].y += red[(i * 4 + 1) * L::kUpd];
          acc[i][1].x += red[(i * 4 + 2) * L::kUpd];
          acc[i][1].y += red[(i * 4 + 3) * L::kUpd];
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        sreg[i * 4 + 0] = fmaf(gC, sreg[i * 4 + 0], acc[i][0].x);
        sreg[i * 4 + 1] = fmaf(gC, sreg[i * 4 + 1], acc[i][0].y);
        sreg[i * 4 + 2] = fmaf(gC, sreg[i * 4 + 2], acc[i][1].x);
        sreg[i * 4 + 3] = fmaf(gC, sreg[i * 4 + 3], acc[i][1].y);
      }
      // S^T for the next chunk's products: column 4 cq + j, rows 4 ru .. 4 ru + 3
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<float4*>(sSt + (4 * cq + j) * RS + 4 * ru) =
            make_float4(sreg[j], sreg[4 + j], sreg[8 + j], sreg[12 + j]);
    }
    __syncthreads();  // S^T complete; the reduction buffer is free
  }
  if (!ok) {
    // a load did not land in time: wait (bounded) for every load in flight before
    // the shared memory is released; the outputs are undefined
    if (tid == 0) {
      if (wq_loads > 0) mbar_drain(smem_u32(&s_wq), (wq_loads - 1) & 1);
      for (int kb = 0; kb < 2; ++kb)
        if (k_loads[kb] > 0) mbar_drain(smem_u32(&s_k[kb]), (k_loads[kb] - 1) & 1);
    }
    __syncthreads();
    return;
  }
  if (p.state && ts == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float* dst = p.state + ((static_cast<size_t>(b) * H + h) * DH + i0 + 4 * ru + i) * DH + 4 * cq;
      *reinterpret_cast<float4*>(dst) =
          make_float4(sreg[i * 4 + 0], sreg[i * 4 + 1], sreg[i * 4 + 2], sreg[i * 4 + 3]);
    }
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
