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

// One workspace record per (chunk, head): five [kC][DH] fp32 matrices and g_C.
template <int DH>
struct ChunkRec {
  static constexpr int kMat = kC * DH;
  static constexpr int kWk = 0, kQe = kMat, kKt = 2 * kMat, kUv = 3 * kMat, kOv = 4 * kMat;
  static constexpr int kG = 5 * kMat;
  static constexpr int kFloats = 5 * kMat + 64;  // 256-byte multiple
};

struct ChunkParams {
  const float* log_alpha;
  const float* beta;
  float* ws;     // [total chunks][heads] records
  float* state;  // [B, H, d, d] or null
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

__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
  acc = fmaf(a.x, b.x, acc);
  acc = fmaf(a.y, b.y, acc);
  acc = fmaf(a.z, b.z, acc);
  return fmaf(a.w, b.w, acc);
}

template <int DH>
struct PrepLay {
  static constexpr int LD = DH + 4;  // padded row pitch (floats) of the row matrices
  static constexpr int LC = kC + 1;  // pitch of the chunk x chunk matrices
  static constexpr int kK = 0, kQ = kC * LD, kV = 2 * kC * LD;
  static constexpr int kA = 3 * kC * LD, kM = kA + kC * LC, kG = kM + kC * LC;
  static constexpr int kBeta = kG + kC * LC, kGam = kBeta + kC, kRho = kGam + kC;
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

template <typename T, int DH>
__global__ void __launch_bounds__(kPrepThreads) delta_chunk_prep_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const __grid_constant__ ChunkParams p) {
  using L = PrepLay<DH>;
  using R = ChunkRec<DH>;
  constexpr int LD = L::LD, LC = L::LC;
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  float* sK = sm + L::kK;  // k^ rows, later W_k
  float* sQ = sm + L::kQ;  // q^ rows
  float* sV = sm + L::kV;  // v rows, later U_v
  float* sA = sm + L::kA;
  float* sM = sm + L::kM;
  float* sG = sm + L::kG;
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

  // rows of q, k, v (fp32), zero past the chunk's end
  for (int idx = tid; idx < kC * DH; idx += kPrepThreads) {
    const int t = idx / DH, c = idx - t * DH;
    float kq = 0.0f, qq = 0.0f, vv = 0.0f;
    if (t < n) {
      const size_t off = (static_cast<size_t>(r0 + t) * H + h) * DH + c;
      kq = to_f32(k[off]);
      qq = to_f32(q[off]);
      vv = to_f32(v[off]);
    }
    sK[t * LD + c] = kq;
    sQ[t * LD + c] = qq;
    sV[t * LD + c] = vv;
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
  // decay ratios g_t / g_s (s <= t), g_t and g_{n-1} / g_s
  for (int idx = tid; idx < kC * kC; idx += kPrepThreads) {
    const int t = idx / kC, s = idx - t * kC;
    float r = 0.0f;
    if (t < n && s <= t && sNinf[t] == sNinf[s])
      r = expf(static_cast<float>(sP[t] - sP[s]));
    sG[t * LC + s] = r;
  }
  if (tid < kC) {
    const int t = tid;
    sGam[t] = (t < n && sNinf[t] == 0) ? expf(static_cast<float>(sP[t])) : 0.0f;
    sRho[t] = (t < n && sNinf[n - 1] == sNinf[t]) ? expf(static_cast<float>(sP[n - 1] - sP[t])) : 0.0f;
  }
  __syncthreads();
  // k^_t . k^_s and q^_t . k^_s in 4 x 4 blocks (blocks above the diagonal are zero)
  {
    const int bt = tid >> 4, bs = tid & 15;
    float ak[4][4], aq[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) ak[i][j] = aq[i][j] = 0.0f;
    if (bs <= bt) {
      for (int d = 0; d < DH; d += 4) {
        float4 kt[4], ks[4], qt[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          kt[i] = *reinterpret_cast<const float4*>(sK + (4 * bt + i) * LD + d);
          qt[i] = *reinterpret_cast<const float4*>(sQ + (4 * bt + i) * LD + d);
          ks[i] = *reinterpret_cast<const float4*>(sK + (4 * bs + i) * LD + d);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            ak[i][j] = dot4(kt[i], ks[j], ak[i][j]);
            aq[i][j] = dot4(qt[i], ks[j], aq[i][j]);
          }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int t = 4 * bt + i, s = 4 * bs + j;
        const float gts = sG[t * LC + s];  // 0 above the diagonal and past the end
        sA[t * LC + s] = s < t ? sBeta[t] * gts * ak[i][j] : 0.0f;
        sM[t * LC + s] = gts * aq[i][j];
      }
  }
  __syncthreads();
  // (I + A) X = R by forward substitution, one column per thread: threads
  // [0, DH) solve U_v (R = diag(beta) V), threads [DH, 2 DH) W_k (R = diag(beta g) K^);
  // the latter also write K~ = diag(ratio(C, s)) K^ from their column first.
  if (tid < 2 * DH) {
    const bool wk = tid >= DH;
    const int c = wk ? tid - DH : tid;
    float* col = (wk ? sK : sV) + c;
    float x[kC];
#pragma unroll
    for (int t = 0; t < kC; ++t) {
      const float e = col[t * LD];
      x[t] = wk ? sBeta[t] * sGam[t] * e : sBeta[t] * e;
      if (wk) rec[R::kKt + t * DH + c] = sRho[t] * e;
    }
#pragma unroll
    for (int t = 1; t < kC; ++t) {
      float a0 = x[t], a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
      const float* arow = sA + t * LC;
#pragma unroll
      for (int s = 0; s + 3 < t; s += 4) {
        a0 = fmaf(-arow[s], x[s], a0);
        a1 = fmaf(-arow[s + 1], x[s + 1], a1);
        a2 = fmaf(-arow[s + 2], x[s + 2], a2);
        a3 = fmaf(-arow[s + 3], x[s + 3], a3);
      }
#pragma unroll
      for (int s = t & ~3; s < t; ++s) a0 = fmaf(-arow[s], x[s], a0);
      x[t] = (a0 + a1) + (a2 + a3);
    }
    float* dst = rec + (wk ? R::kWk : R::kUv) + c;
#pragma unroll
    for (int t = 0; t < kC; ++t) {
      dst[t * DH] = x[t];
      col[t * LD] = x[t];
    }
  }
  __syncthreads();
  // O_v = M U_v and Q_e = diag(g) Q^ - M W_k, one column per thread
  if (tid < 2 * DH) {
    const bool qe = tid >= DH;
    const int c = qe ? tid - DH : tid;
    const float* col = (qe ? sK : sV) + c;
    float y[kC];
#pragma unroll
    for (int s = 0; s < kC; ++s) y[s] = col[s * LD];
    float* dst = rec + (qe ? R::kQe : R::kOv) + c;
#pragma unroll
    for (int t = 0; t < kC; ++t) {
      const float* mrow = sM + t * LC;
      float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
      for (int s = 0; s + 1 <= t; s += 2) {
        a0 = fmaf(mrow[s], y[s], a0);
        a1 = fmaf(mrow[s + 1], y[s + 1], a1);
      }
      if ((t & 1) == 0) a0 = fmaf(mrow[t], y[t], a0);
      const float acc = a0 + a1;
      dst[t * DH] = qe ? fmaf(sGam[t], sQ[t * LD + c], -acc) : acc;
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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <typename T, int DH>
__global__ void __launch_bounds__(kScanThreads) delta_chunk_scan_kernel(
    T* __restrict__ out, const __grid_constant__ ChunkParams p) {
  using L = ScanLay<DH>;
  using R = ChunkRec<DH>;
  constexpr int LS = L::LS;
  constexpr int NC = DH / 16;  // state columns per thread in the update
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  float* sS = sm + L::kS;
  float* sD = sm + L::kD;
  const int tid = threadIdx.x;
  const int i0 = blockIdx.x * kScanRows, h = blockIdx.y, b = blockIdx.z, H = p.heads;
  const int c_first = p.chunk_start[b], n_chunks = p.chunk_start[b + 1] - c_first;
  const int row0 = p.kept_start[b], len = p.kept_start[b + 1] - row0;

  // chunk c's matrices and this block's U_v / O_v columns into stage c & 1
  auto load_chunk = [&](int c) {
    float* st = sm + (c & 1) * L::kStage;
    const float* rec = p.ws + (static_cast<size_t>(c_first + c) * H + h) * R::kFloats;
    const uint32_t sb = smem_u32(st);
    for (int i = tid; i < 3 * R::kMat / 4; i += kScanThreads)  // W_k, Q_e, K~: contiguous
      cp_async16(sb + i * 16, rec + 4 * i);
    for (int i = tid; i < 2 * kC * kScanRows / 4; i += kScanThreads) {
      const int m = i / (kC * kScanRows / 4), j = i - m * (kC * kScanRows / 4);
      const int t = j / (kScanRows / 4), q4 = j - t * (kScanRows / 4);
      cp_async16(sb + (3 * R::kMat + m * kC * kScanRows + t * kScanRows + 4 * q4) * 4,
                 rec + (m ? R::kOv : R::kUv) + t * DH + i0 + 4 * q4);
    }
  };

  // update mapping: thread owns state row ru, columns [cu, cu + NC)
  const int ru = tid >> 4, cu = (tid & 15) * NC;
  // product mapping: thread owns chunk rows 4 tg .. 4 tg + 3 of state row rp
  const int tg = tid >> 4, rp = tid & 15;
  float sreg[NC];
#pragma unroll
  for (int j = 0; j < NC; ++j) sreg[j] = 0.0f;
#pragma unroll
  for (int j = 0; j < NC; ++j) sS[ru * LS + cu + j] = 0.0f;
  if (n_chunks > 0) load_chunk(0);
  cp_async_commit();
  for (int c = 0; c < n_chunks; ++c) {
    if (c + 1 < n_chunks) load_chunk(c + 1);
    cp_async_commit();
    cp_async_wait<1>();  // chunk c has landed
    __syncthreads();
    const float* st = sm + (c & 1) * L::kStage;
    const float* sW = st;
    const float* sQe = st + R::kMat;
    const float* sKt = st + 2 * R::kMat;
    const float* sUv = st + 3 * R::kMat;
    const float* sOv = sUv + kC * kScanRows;
    const float gC = __ldg(p.ws + (static_cast<size_t>(c_first + c) * H + h) * R::kFloats + R::kG);
    // X = W_k S^T and Y = Q_e S^T for this thread's 4 chunk rows and state row rp
    float ax[4] = {0.0f, 0.0f, 0.0f, 0.0f}, ay[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 4
    for (int d = 0; d < DH; d += 4) {
      const float4 s4 = *reinterpret_cast<const float4*>(sS + rp * LS + d);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ax[i] = dot4(*reinterpret_cast<const float4*>(sW + (4 * tg + i) * DH + d), s4, ax[i]);
        ay[i] = dot4(*reinterpret_cast<const float4*>(sQe + (4 * tg + i) * DH + d), s4, ay[i]);
      }
    }
    const int t0 = c * kC;  // chunk rows within the prompt
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = 4 * tg + i;
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
#pragma unroll
      for (int j = 0; j < NC; j += 4) {
        const float4 kt = *reinterpret_cast<const float4*>(sKt + t * DH + cu + j);
        sreg[j] = fmaf(dd, kt.x, sreg[j]);
        sreg[j + 1] = fmaf(dd, kt.y, sreg[j + 1]);
        sreg[j + 2] = fmaf(dd, kt.z, sreg[j + 2]);
        sreg[j + 3] = fmaf(dd, kt.w, sreg[j + 3]);
      }
    }
#pragma unroll
    for (int j = 0; j < NC; ++j) sS[ru * LS + cu + j] = sreg[j];
    __syncthreads();  // state and stage free for the next chunk
  }
  if (p.state) {
    float* dst = p.state + ((static_cast<size_t>(b) * H + h) * DH + i0 + ru) * DH + cu;
#pragma unroll
    for (int j = 0; j < NC; j += 4)
      *reinterpret_cast<float4*>(dst + j) = make_float4(sreg[j], sreg[j + 1], sreg[j + 2], sreg[j + 3]);
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
