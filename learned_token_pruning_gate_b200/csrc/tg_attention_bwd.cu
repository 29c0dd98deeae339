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
#include <algorithm>
#include <cmath>

#include "tg_internal.cuh"

namespace tg {
namespace {

constexpr float kLn2f = 0.6931471805599453f;
constexpr float kLog2e_b = 1.4426950408889634f;

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
  uint32_t* status_word;
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

// ---- tensor-core path (bf16, head_dim 64/128) ---------------------------------
// Work unit = (prompt, 128-key tile, query head); the unit walks the query tiles
// at or after its key tile.  Everything is transposed with respect to the
// forward: TMEM lane = key, column = query, so one thread owns one key and the
// sums over queries that the log-gate gradient needs are thread-local.
//   S'  = K Q^T  + 1 x_i,  x_i = -LSE_i sqrt(d) tau_h   -> scale * S' = log2 P_ji - g log2e l_j
//   dP' = V dO^T + 1 y_i,  y_i = -D_i                     -> dP' = dP_ji - D_i
// Both bias rows enter as one extra K=16 step (A rows [1,1,1,0..], B rows the
// three bf16 parts of x_i or y_i, K-major without swizzle), as in the forward.
//   warp 0     TMA: the unit's K and V tiles, then Q and dO tiles of each query
//              tile into a 2-stage ring
//   warp 1     TMEM owner (512 columns) and MMA issuer: per query tile S' and dP'
//              into the 256 columns of the softmax warpgroup that takes the tile
//   warps 2-3  write the B rows of x_i and y_i for each query stage
//   warps 4-7, 8-11  two warpgroups take alternate query tiles: p = 2^(S' scale
//              + g log2e l_j), dlogit = p dP'; per key: sum dlogit and sum
//              dlogit log2 p, added to the outputs with atomics at the unit's end
constexpr int kBwdThreads = 384;
constexpr int kBwdMaxTiles = 1024;  // 128-row key tiles over all prompts
constexpr int kBwdStages = 2;

struct BwdTcParams {
  BwdParams b;
  int16_t tile_b[kBwdMaxTiles];  // key tiles by decreasing query-tile count
  int16_t tile_j[kBwdMaxTiles];
  int32_t n_tiles;
};

template <int DH>
struct BwdLay {
  static constexpr uint32_t kChunks = DH / 64;
  static constexpr uint32_t kBox = 128 * 128;        // 128 rows x 64 bf16
  static constexpr uint32_t kTile = kChunks * kBox;  // one 128-row tile
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kTile;
  static constexpr uint32_t kQ = 2 * kTile;                    // [stage] Q then dO
  static constexpr uint32_t kAug = kQ + kBwdStages * 2 * kTile;  // A, then [stage] Bx, By
  static constexpr uint32_t kAugTile = 4096;
  static constexpr uint32_t kBars = kAug + (1 + 2 * kBwdStages) * kAugTile;
  static constexpr uint32_t kMisc = kBars + 16 * 8;
  static constexpr uint32_t kTotal = kMisc + 16;
  static constexpr uint32_t kDynSmem = kTotal + 1024;
};

enum {
  kBKVFull = 0,
  kBKVEmpty = 1,
  kBQFull = 2,    // [stages]
  kBQEmpty = 4,   // [stages]
  kBAugFull = 6,  // [stages], 64 arrivals
  kBSFull = 8,    // [2 warpgroups]
  kBTFree = 10,   // [2 warpgroups], 128 arrivals
  kBDrain = 12,
};

__device__ __forceinline__ uint4 split3(float x) {  // three bf16 parts summing to x
  const __nv_bfloat16 a = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(a);
  const __nv_bfloat16 b = __float2bfloat16_rn(r1);
  const __nv_bfloat16 c = __float2bfloat16_rn(r1 - __bfloat162float(b));
  const __nv_bfloat162 ab = __halves2bfloat162(a, b), c0 = __halves2bfloat162(c, __float2bfloat16_rn(0.0f));
  return make_uint4(*reinterpret_cast<const uint32_t*>(&ab), *reinterpret_cast<const uint32_t*>(&c0),
                    0u, 0u);
}

// Unit of round k on CTA r of g: boustrophedon deal of units sorted by cost.
__device__ __forceinline__ int bwd_snake(int k, int r, int g) {
  return k * g + ((k & 1) ? g - 1 - r : r);
}

template <int DH>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ BwdTcParams P) {
  using L = BwdLay<DH>;
  const BwdParams& p = P.b;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  uint8_t* s_aug = smem + L::kAug;
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_units = P.n_tiles * p.hq;

  if (warp == 0 && lane == 0) {
    mbar_init(bar(kBKVFull), 1);
    mbar_init(bar(kBKVEmpty), 1);
    for (int s = 0; s < kBwdStages; ++s) {
      mbar_init(bar(kBQFull + s), 1);
      mbar_init(bar(kBQEmpty + s), 1);
      mbar_init(bar(kBAugFull + s), 64);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(bar(kBSFull + w), 1);
      mbar_init(bar(kBTFree + w), 128);
    }
    mbar_init(bar(kBDrain), 1);
    *abort_flag = 0;
    mbar_fence_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_do);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  // A rows of the bias step: [1, 1, 1, 0 ...]; all zero halves (k = 8..15)
  for (int i = threadIdx.x; i < static_cast<int>((1 + 2 * kBwdStages) * L::kAugTile / 16);
       i += kBwdThreads)
    reinterpret_cast<uint4*>(s_aug)[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  if (threadIdx.x < 128) {
    const __nv_bfloat162 one2 = __floats2bfloat162_rn(1.0f, 1.0f), one0 = __floats2bfloat162_rn(1.0f, 0.0f);
    reinterpret_cast<uint4*>(s_aug)[threadIdx.x] =
        make_uint4(*reinterpret_cast<const uint32_t*>(&one2), *reinterpret_cast<const uint32_t*>(&one0), 0u, 0u);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dep_wait();  // D and the cleared outputs are in place
  grid_dep_launch();
  const uint32_t tmem = *tmem_slot;
  int kv_loads = 0, q_loads = 0;

  auto unit_of = [&](int round, int& b, int& jt, int& h, int& n_q, int& len, int& kstart) {
    const int u = bwd_snake(round, blockIdx.x, gridDim.x);
    if (u >= n_units) return false;
    const int t = u / p.hq;
    h = u - t * p.hq;
    b = P.tile_b[t];
    jt = P.tile_j[t];
    kstart = p.kept_start[b];
    len = p.kept_start[b + 1] - kstart;
    n_q = (len + 127) / 128 - jt;
    return true;
  };
  if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(104));

  if (warp == 0) {
    if (lane == 0) {
      const int hkv = p.hq / p.group;
      uint32_t kv_ph = 0;
      int qs = 0;
      uint32_t q_ph = 0;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        int b, jt, h, n_q, len, kstart;
        if (!unit_of(round, b, jt, h, n_q, len, kstart)) break;
        const int hk = h / p.group;
        (void)hkv;
        if (!(ok = mbar_wait(bar(kBKVEmpty), kv_ph ^ 1, abort_flag, p.status_word, kDevTimeoutAttn)))
          break;
        kv_ph ^= 1;
        mbar_arrive_expect_tx(bar(kBKVFull), 2 * L::kTile);
        ++kv_loads;
        for (uint32_t c = 0; c < L::kChunks; ++c) {
          tma_load_2d(sb + L::kK + c * L::kBox, &tm_k, hk * DH + c * 64, kstart + jt * 128, bar(kBKVFull));
          tma_load_2d(sb + L::kV + c * L::kBox, &tm_v, hk * DH + c * 64, kstart + jt * 128, bar(kBKVFull));
        }
        for (int r = 0; r < n_q; ++r) {
          if (!(ok = mbar_wait(bar(kBQEmpty + qs), q_ph ^ 1, abort_flag, p.status_word, kDevTimeoutAttn)))
            break;
          const int row = kstart + (jt + r) * 128;
          mbar_arrive_expect_tx(bar(kBQFull + qs), 2 * L::kTile);
          ++q_loads;
          const uint32_t dq = sb + L::kQ + qs * 2 * L::kTile;
          for (uint32_t c = 0; c < L::kChunks; ++c) {
            tma_load_2d(dq + c * L::kBox, &tm_q, h * DH + c * 64, row, bar(kBQFull + qs));
            tma_load_2d(dq + L::kTile + c * L::kBox, &tm_do, h * DH + c * 64, row, bar(kBQFull + qs));
          }
          if (++qs == kBwdStages) {
            qs = 0;
            q_ph ^= 1;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
      const uint64_t d_k = sw128_desc(sb + L::kK, 16, 1024);
      const uint64_t d_v = sw128_desc(sb + L::kV, 16, 1024);
      const uint64_t d_q0 = sw128_desc(sb + L::kQ, 16, 1024);
      const uint64_t d_a = nosw_desc(sb + L::kAug, 2048, 128);
      const uint64_t d_b0 = nosw_desc(sb + L::kAug + L::kAugTile, 2048, 128);
      auto wt = [&](uint32_t b_, uint32_t par) {
        return mbar_wait(b_, par, abort_flag, p.status_word, kDevTimeoutAttn);
      };
      uint32_t kv_ph = 0, q_ph = 0, tf_ph[2] = {1u, 1u};
      int qs = 0;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        int b, jt, h, n_q, len, kstart;
        if (!unit_of(round, b, jt, h, n_q, len, kstart)) break;
        if (!(ok = wt(bar(kBKVFull), kv_ph))) break;
        kv_ph ^= 1;
        for (int r = 0; r < n_q; ++r) {
          const int w = r & 1;
          if (!(ok = wt(bar(kBQFull + qs), q_ph))) break;
          if (!(ok = wt(bar(kBAugFull + qs), q_ph))) break;
          if (!(ok = wt(bar(kBTFree + w), tf_ph[w]))) break;
          tf_ph[w] ^= 1;
          tc_fence_after();
          const uint64_t dq = d_q0 + ((qs * 2 * L::kTile) >> 4);
          const uint64_t ddo = dq + (L::kTile >> 4);
          const uint32_t ts = tmem + w * 256, tp = ts + 128;
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) {
            const uint32_t off = (kk >> 2) * (L::kBox >> 4) + (kk & 3) * 2;
            umma_ss(ts, d_k + off, dq + off, idesc, kk > 0 ? 1u : 0u);
          }
          umma_ss(ts, d_a, d_b0 + ((qs * 2 * L::kAugTile) >> 4), idesc, 1u);
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) {
            const uint32_t off = (kk >> 2) * (L::kBox >> 4) + (kk & 3) * 2;
            umma_ss(tp, d_v + off, ddo + off, idesc, kk > 0 ? 1u : 0u);
          }
          umma_ss(tp, d_a, d_b0 + (((qs * 2 + 1) * L::kAugTile) >> 4), idesc, 1u);
          umma_commit(bar(kBSFull + w));
          umma_commit(bar(kBQEmpty + qs));
          if (++qs == kBwdStages) {
            qs = 0;
            q_ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(bar(kBKVEmpty));
      }
    }
    __syncwarp();
  } else if (warp < 4) {
    // bias rows of each query stage: x_i (for S') and y_i (for dP'), two rows per thread
    const int t = threadIdx.x - 64;
    uint32_t q_ph = 0;
    int qs = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      int b, jt, h, n_q, len, kstart;
      if (!unit_of(round, b, jt, h, n_q, len, kstart)) break;
      const float xs = -sqrtf(static_cast<float>(DH)) * __ldg(p.temp + h);
      for (int r = 0; r < n_q; ++r) {
        ok = mbar_wait(bar(kBQEmpty + qs), q_ph ^ 1, abort_flag, p.status_word, kDevTimeoutAttn);
        if (named_barrier_or(3, 64, !ok)) {
          ok = false;
          break;
        }
        for (int rr = t; rr < 128; rr += 64) {
          const int qi = (jt + r) * 128 + rr;
          float x = 0.0f, y = 0.0f;
          if (qi < len) {
            const int64_t gi = static_cast<int64_t>(h) * p.m_total + kstart + qi;
            x = __ldg(p.lse + gi) * xs;
            y = -p.D[gi];
          }
          reinterpret_cast<uint4*>(s_aug + (1 + 2 * qs) * L::kAugTile)[rr] = split3(x);
          reinterpret_cast<uint4*>(s_aug + (2 + 2 * qs) * L::kAugTile)[rr] = split3(y);
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(kBAugFull + qs));
        if (++qs == kBwdStages) {
          qs = 0;
          q_ph ^= 1;
        }
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(192));
    const int w = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;  // key row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_off + w * 256, t_p = t_s + 128;
    uint32_t s_ph = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      int b, jt, h, n_q, len, kstart;
      if (!unit_of(round, b, jt, h, n_q, len, kstart)) break;
      if (w >= n_q) continue;  // no query tile of this unit for this warpgroup
      const int key = jt * 128 + rl;
      const bool key_ok = key < len;
      const float lj = key_ok ? __ldg(p.logsig + kstart + key) : 0.0f;
      const float g = __ldg(p.gain + h);
      const float scale = kLog2e_b / (sqrtf(static_cast<float>(DH)) * __ldg(p.temp + h));
      const float cj = g * kLog2e_b * lj;
      const float2 sc2 = make_float2(scale, scale), cj2 = make_float2(cj, cj);
      float2 accL = make_float2(0.0f, 0.0f), accT = make_float2(0.0f, 0.0f);
      for (int r = w; r < n_q; r += 2) {
        ok = mbar_wait(bar(kBSFull + w), s_ph, abort_flag, p.status_word, kDevTimeoutAttn);
        s_ph ^= 1;
        if (named_barrier_or(1 + w, 128, !ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int qlim = len - (jt + r) * 128;  // query columns at or past it do not exist
        const int qmin = r == 0 ? rl : 0;       // diagonal tile: queries before the key are masked
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t sv[32], dv[32];
          tmem_ld32(t_s + c * 32, sv);
          tmem_ld32(t_p + c * 32, dv);
          tmem_ld_wait(sv);
          tmem_ld_wait(dv);
          if (c == 3) {
            tc_fence_before();
            mbar_arrive(bar(kBTFree + w));
          }
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int col = c * 32 + e;
            float2 t2 = __ffma2_rn(make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sc2, cj2);
            if (col < qmin || col >= qlim) t2.x = -1e30f;
            if (col + 1 < qmin || col + 1 >= qlim) t2.y = -1e30f;
            const float2 pr = make_float2(exp2_approx(t2.x), exp2_approx(t2.y));
            const float2 dl = __fmul2_rn(pr, make_float2(__uint_as_float(dv[e]), __uint_as_float(dv[e + 1])));
            accL = __fadd2_rn(accL, dl);
            accT = __ffma2_rn(dl, t2, accT);
          }
        }
      }
      if (!ok) break;
      const float sl = accL.x + accL.y;
      if (key_ok) atomicAdd(p.d_logsig + kstart + key, g * sl);
      float G = key_ok ? lj * sl : 0.0f, A = key_ok ? accT.x + accT.y : 0.0f;
      G = warp_sum(G);
      A = warp_sum(A);
      if (lane == 0) {
        atomicAdd(p.d_gain + h, G);
        atomicAdd(p.acc + h, A);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // a wait gave up: let the loads and MMAs already issued finish (bounded)
    if (warp == 0 && lane == 0) {
      if (kv_loads > 0) mbar_drain(bar(kBKVFull), (kv_loads - 1) & 1);
      for (int s = 0; s < kBwdStages && s < q_loads; ++s)
        mbar_drain(bar(kBQFull + s), ((q_loads - 1 - s) / kBwdStages) & 1);
    }
    if (warp == 1 && lane == 0) {
      umma_commit(bar(kBDrain));
      mbar_drain(bar(kBDrain), 0);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
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
                          float* d_temp, void* workspace, int algo, cudaStream_t st) {
  static thread_local BwdTcParams P;
  BwdParams& p = P.b;
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
  p.status_word = device_status_word();
  if (!p.status_word) return set_error(TG_ERR_CUDA, "device status word unavailable");
  // key tiles by decreasing number of query tiles (their units' cost)
  int n_tiles = 0;
  for (int b = 0; b < pt.batch; ++b) n_tiles += (pt.kept_start[b + 1] - pt.kept_start[b] + 127) / 128;
  const bool tc = dt == TG_BF16 && algo != TG_ALGO_SIMT && n_tiles <= kBwdMaxTiles;
  if (tc) {
    int n = 0;
    int max_nt = 0;
    for (int b = 0; b < pt.batch; ++b)
      max_nt = std::max(max_nt, (pt.kept_start[b + 1] - pt.kept_start[b] + 127) / 128);
    for (int cost = max_nt; cost >= 1; --cost)
      for (int b = 0; b < pt.batch; ++b) {
        const int nt = (pt.kept_start[b + 1] - pt.kept_start[b] + 127) / 128;
        if (nt >= cost) {
          P.tile_b[n] = static_cast<int16_t>(b);
          P.tile_j[n] = static_cast<int16_t>(nt - cost);
          ++n;
        }
      }
    P.n_tiles = n;
  }
  const int64_t warps = static_cast<int64_t>(p.m_total) * hq;
  int64_t blocks = (warps + 7) / 8;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (blocks > cap) blocks = cap;
  const dim3 grid(static_cast<unsigned>(blocks)), blk(256);
  tg_status r;
#define TG_BWD_PREP(T, DH)                                                                      \
  r = cuda_check(launch_pdl(bwd_prep_kernel<T, DH>, grid, blk, 0, st,                           \
                            static_cast<const T*>(out), static_cast<const T*>(dout), p),        \
                 "attention backward prep launch")
#define TG_BWD_SIMT(T, DH)                                                                      \
  r = cuda_check(launch_pdl(bwd_simt_kernel<T, DH>, grid, blk, 0, st, static_cast<const T*>(q), \
                            static_cast<const T*>(k), static_cast<const T*>(v),                 \
                            static_cast<const T*>(dout), p),                                    \
                 "attention backward launch")
  if (dt == TG_BF16) {
    if (dh == 64) TG_BWD_PREP(__nv_bfloat16, 64);
    else TG_BWD_PREP(__nv_bfloat16, 128);
  } else {
    if (dh == 64) TG_BWD_PREP(float, 64);
    else TG_BWD_PREP(float, 128);
  }
  if (r != TG_OK) return r;
  if (tc) {
    CUtensorMap tq, tk, tv, tdo;
    const uint64_t M = static_cast<uint64_t>(p.m_total);
    if (!encode_tmap_2d_bf16(&tq, q, static_cast<uint64_t>(hq) * dh, M,
                             static_cast<uint64_t>(hq) * dh * 2, 64, 128) ||
        !encode_tmap_2d_bf16(&tdo, dout, static_cast<uint64_t>(hq) * dh, M,
                             static_cast<uint64_t>(hq) * dh * 2, 64, 128) ||
        !encode_tmap_2d_bf16(&tk, k, static_cast<uint64_t>(hkv) * dh, M,
                             static_cast<uint64_t>(hkv) * dh * 2, 64, 128) ||
        !encode_tmap_2d_bf16(&tv, v, static_cast<uint64_t>(hkv) * dh, M,
                             static_cast<uint64_t>(hkv) * dh * 2, 64, 128))
      return set_error(TG_ERR_CUDA, "cuTensorMapEncodeTiled failed for the backward");
    const int n_units = P.n_tiles * hq;
    const int g = std::min(num_sms(), n_units);
    auto launch = [&](auto kern, uint32_t smem) {
      tg_status rr = cuda_check(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     static_cast<int>(smem)),
                                "attention backward smem attribute");
      if (rr != TG_OK) return rr;
      return cuda_check(launch_pdl(kern, dim3(g), dim3(kBwdThreads), smem, st, tq, tk, tv, tdo, P),
                        "attention backward launch");
    };
    r = dh == 64 ? launch(bwd_tc_kernel<64>, BwdLay<64>::kDynSmem)
                 : launch(bwd_tc_kernel<128>, BwdLay<128>::kDynSmem);
  } else if (dt == TG_BF16) {
    if (dh == 64) TG_BWD_SIMT(__nv_bfloat16, 64);
    else TG_BWD_SIMT(__nv_bfloat16, 128);
  } else {
    if (dh == 64) TG_BWD_SIMT(float, 64);
    else TG_BWD_SIMT(float, 128);
  }
#undef TG_BWD_PREP
#undef TG_BWD_SIMT
  if (r != TG_OK) return r;
  unsigned fb = static_cast<unsigned>((p.m_total + 255) / 256);
  if (fb == 0) fb = 1;
  return cuda_check(launch_pdl(bwd_finish_kernel, dim3(fb), blk, 0, st, p, tc ? 1 : 0),
                    "attention backward finish launch");
}

}  // namespace tg
