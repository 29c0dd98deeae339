// Element-wise steps of the gated upper-layer stack.  Every attention layer above
// the gate keeps working on the same kept rows (TokenGate: the layers above L
// process only the kept tokens and create KV only for them) with its own gain
// and temperature; the layers are Qwen3-shaped (RMSNorm, fused QKV projection,
// per-head RMSNorm of q and k, RoPE at the rows' original positions, SwiGLU
// MLP).  The projections are plain GEMMs (cuBLAS); these kernels do the rest:
//   rmsnorm_kernel    y = x / sqrt(mean(x^2) + eps) * w, one warp per row
//   qkv_emit_kernel   split of the QKV projection: q and k get their per-head
//                     RMSNorm and RoPE, k and v go straight into the layer's
//                     slot of the compacted KV cache, one warp per (row, head)
//   swiglu_kernel     h = SiLU(gate) * up from the fused [gate | up] projection
#include <cmath>

#include "tg_internal.cuh"

namespace tg {
namespace {

constexpr int kStackMaxHalf = 128;

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_allsum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <typename T>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const T* __restrict__ x, const T* __restrict__ w,
                                                      T* __restrict__ y, int64_t rows, int dim,
                                                      float eps) {
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       r < rows; r += nw) {
    const T* xr = x + r * dim;
    float ss = 0.0f;
    for (int c = lane; c < dim; c += 32) {
      const float v = to_f(xr[c]);
      ss = fmaf(v, v, ss);
    }
    const float inv = rsqrtf(warp_allsum(ss) / static_cast<float>(dim) + eps);
    T* yr = y + r * dim;
    for (int c = lane; c < dim; c += 32) yr[c] = from_f<T>(to_f(xr[c]) * inv * to_f(w[c]));
  }
}

struct EmitParams {
  PromptTable pt;
  uint64_t turns[kStackMaxHalf];  // RoPE angle per position unit, fraction of a turn, 0.64
  int64_t rows;
  int32_t hq, hkv, dh;
  float eps;
};

template <typename T>
__global__ void __launch_bounds__(256) qkv_emit_kernel(const T* __restrict__ qkv,
                                                       const int32_t* __restrict__ kept_idx,
                                                       const T* __restrict__ w_qn,
                                                       const T* __restrict__ w_kn,
                                                       T* __restrict__ q_out, T* __restrict__ k_out,
                                                       T* __restrict__ v_out,
                                                       const __grid_constant__ EmitParams p) {
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const int dh = p.dh, half = dh / 2, per = dh / 32;  // elements per lane (2 or 4)
  const int heads = p.hq + 2 * p.hkv;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t total = p.rows * heads;
  for (int64_t w = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       w < total; w += nw) {
    const int64_t i = w / heads;
    const int hh = static_cast<int>(w - i * heads);
    const T* src = qkv + (i * heads + hh) * dh;
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = e < per ? to_f(src[lane * per + e]) : 0.0f;
    if (hh >= p.hq + p.hkv) {  // v: into the cache as it is
      T* dst = v_out + (i * p.hkv + (hh - p.hq - p.hkv)) * dh;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (e < per) dst[lane * per + e] = src[lane * per + e];
      continue;
    }
    const bool is_q = hh < p.hq;
    const T* wn = is_q ? w_qn : w_kn;
    float ss = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) ss = fmaf(x[e], x[e], ss);
    const float inv = rsqrtf(warp_allsum(ss) / static_cast<float>(dh) + p.eps);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (e < per) x[e] = x[e] * inv * to_f(wn[lane * per + e]);
    // original position of the kept row inside its prompt
    const int32_t src_row = __ldg(kept_idx + i);
    int lo = 0, hi = p.pt.batch - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.pt.kept_start[mid] <= i) lo = mid; else hi = mid - 1;
    }
    const uint32_t pos = static_cast<uint32_t>(src_row - p.pt.start[lo]);
    // rotate-half pairs (j, j + d/2): the partner element sits in lane ^ 16
    float y[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float partner = __shfl_xor_sync(0xffffffffu, x[e], 16);
      const int j = lane * per + e;  // dim index
      const int fi = j < half ? j : j - half;
      const uint64_t f = p.turns[fi];
      const uint32_t top = pos * static_cast<uint32_t>(f >> 32) + __umulhi(pos, static_cast<uint32_t>(f));
      float sn, c;
      sincospif(static_cast<float>(static_cast<int32_t>(top)) * 4.656612873077393e-10f, &sn, &c);
      y[e] = j < half ? x[e] * c - partner * sn : x[e] * c + partner * sn;
    }
    T* dst = is_q ? q_out + (i * p.hq + hh) * dh : k_out + (i * p.hkv + (hh - p.hq)) * dh;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (e < per) dst[lane * per + e] = from_f<T>(y[e]);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) swiglu_kernel(const T* __restrict__ gu, T* __restrict__ h,
                                                     int64_t rows, int inter) {
  grid_dep_wait();
  grid_dep_launch();
  const int64_t total = rows * inter;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = t / inter;
    const int c = static_cast<int>(t - r * inter);
    const float g = to_f(gu[r * 2 * inter + c]), u = to_f(gu[r * 2 * inter + inter + c]);
    h[t] = from_f<T>(g / (1.0f + __expf(-g)) * u);
  }
}

unsigned grid_for(int64_t items, int per_block) {
  int64_t blocks = (items + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (blocks > cap) blocks = cap;
  return static_cast<unsigned>(blocks < 1 ? 1 : blocks);
}

}  // namespace

tg_status launch_rmsnorm(const void* x, const void* w, void* y, tg_dtype dt, int64_t rows, int dim,
                         float eps, cudaStream_t st) {
  const dim3 g(grid_for(rows, 8)), b(256);
  if (dt == TG_BF16)
    return cuda_check(launch_pdl(rmsnorm_kernel<__nv_bfloat16>, g, b, 0, st,
                                 static_cast<const __nv_bfloat16*>(x),
                                 static_cast<const __nv_bfloat16*>(w),
                                 static_cast<__nv_bfloat16*>(y), rows, dim, eps),
                      "rmsnorm launch");
  return cuda_check(launch_pdl(rmsnorm_kernel<float>, g, b, 0, st, static_cast<const float*>(x),
                               static_cast<const float*>(w), static_cast<float*>(y), rows, dim, eps),
                    "rmsnorm launch");
}

tg_status launch_qkv_emit(const void* qkv, tg_dtype dt, const PromptTable& pt, const int32_t* kept_idx,
                          int hq, int hkv, int dh, const void* w_qn, const void* w_kn, float eps,
                          double theta, void* q_out, void* k_out, void* v_out, cudaStream_t st) {
  static thread_local EmitParams p;
  p.pt = pt;
  p.rows = pt.kept_start[pt.batch];
  p.hq = hq;
  p.hkv = hkv;
  p.dh = dh;
  p.eps = eps;
  for (int i = 0; i < dh / 2 && i < kStackMaxHalf; ++i) {
    const double f = std::pow(theta, -2.0 * i / static_cast<double>(dh)) / (2.0 * 3.14159265358979323846);
    p.turns[i] = static_cast<uint64_t>(std::ldexp(f, 64));  // f < 1: fits
  }
  const dim3 g(grid_for(p.rows * (hq + 2 * hkv), 8)), b(256);
  if (dt == TG_BF16)
    return cuda_check(
        launch_pdl(qkv_emit_kernel<__nv_bfloat16>, g, b, 0, st,
                   static_cast<const __nv_bfloat16*>(qkv), kept_idx,
                   static_cast<const __nv_bfloat16*>(w_qn), static_cast<const __nv_bfloat16*>(w_kn),
                   static_cast<__nv_bfloat16*>(q_out), static_cast<__nv_bfloat16*>(k_out),
                   static_cast<__nv_bfloat16*>(v_out), p),
        "qkv emit launch");
  return cuda_check(launch_pdl(qkv_emit_kernel<float>, g, b, 0, st, static_cast<const float*>(qkv),
                               kept_idx, static_cast<const float*>(w_qn),
                               static_cast<const float*>(w_kn), static_cast<float*>(q_out),
                               static_cast<float*>(k_out), static_cast<float*>(v_out), p),
                    "qkv emit launch");
}

tg_status launch_swiglu(const void* gu, void* h, tg_dtype dt, int64_t rows, int inter,
                        cudaStream_t st) {
  const dim3 g(grid_for(rows * inter, 256)), b(256);
  if (dt == TG_BF16)
    return cuda_check(launch_pdl(swiglu_kernel<__nv_bfloat16>, g, b, 0, st,
                                 static_cast<const __nv_bfloat16*>(gu),
                                 static_cast<__nv_bfloat16*>(h), rows, inter),
                      "swiglu launch");
  return cuda_check(launch_pdl(swiglu_kernel<float>, g, b, 0, st, static_cast<const float*>(gu),
                               static_cast<float*>(h), rows, inter),
                    "swiglu launch");
}

}  // namespace tg
