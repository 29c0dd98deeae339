// Gate MLP score (TokenGate: "at layer L a small MLP scores each token from its
// post-attention residual"):  z[j] = w2 . GELU(W1 h[j] + b1) + b2.
//
// gate_tc_kernel (bf16, the hot path) is a persistent tcgen05 GEMM whose
// epilogue is the rest of the MLP, so the [n, d_hidden] hidden activation never
// reaches HBM:
//   warp 0     TMA producer: 128 x 64 residual tile + d_hidden x 64 W1 tile per
//              stage, 128-byte swizzle, 4-stage ring (residual streamed with an
//              evict-first hint, W1 kept in L2 with evict-last)
//   warp 1     allocates 512 TMEM columns and issues tcgen05.mma (M=128,
//              N=d_hidden, K=16) into one of two accumulators
//   warps 2-5  epilogue: tcgen05.ld of its 32 rows, +b1, erf-GELU, *w2, row sum,
//              +b2, one fp32 store per token; the accumulator is then released so
//              the next tile's MMAs overlap this epilogue.
// gate_simt_kernel is the CUDA-core path for fp32 and for shapes the tensor-core
// kernel does not take.
//
// With a top-K workspace (tg_gate_score_hist) every kernel's epilogue also
// counts each document token's score into its prompt's first radix-pass
// histogram (top 11 bits of the order key), so the top-K select starts at its
// second pass: the scores are in registers here anyway, and the histogram costs
// one global atomic per distinct bin of a warp's rows.
#include "tg_internal.cuh"

namespace tg {
namespace {

__device__ __forceinline__ float gelu_erf(float a) {
  return 0.5f * a * (1.0f + erff(a * 0.70710678118654752f));
}

// GELU for the tensor-core epilogues: GELU(a) = a Phi(a), Phi(a) = (1 + erf(a/sqrt2)) / 2,
// with erf from the rational-exponential approximation of Abramowitz & Stegun
// (Handbook of Mathematical Functions, 7.1.26, after C. Hastings): for x >= 0,
//   1 - erf(x) = t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) e^(-x^2),  t = 1 / (1 + p x),
// absolute error <= 1.5e-7.  With h = a (1 - erf(|a|/sqrt2)) / 2, GELU(a) is a - h for
// a >= 0 and h for a < 0.  One reciprocal and one exponential on the special-function
// unit, seven FMA-pipe operations.
__device__ __forceinline__ float gelu_as(float a) {
  const float x = fabsf(a) * 0.70710678118654752f;
  float t;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t) : "f"(fmaf(0.3275911f, x, 1.0f)));
  float q = fmaf(t, 1.061405429f, -1.453152027f);
  q = fmaf(q, t, 1.421413741f);
  q = fmaf(q, t, -0.284496736f);
  q = fmaf(q, t, 0.254829592f);
  q *= t;
  const float e = exp2_approx(-1.4426950408889634f * x * x);
  const float h = 0.5f * a * (q * e);
  return a >= 0.0f ? a - h : h;
}
// w2 . GELU(acc + b1) over 32 accumulator columns (b1, w2 in shared memory,
// 16-byte aligned), two partial sums
__device__ __forceinline__ float gelu_dot32(const uint32_t (&r)[32], const float* b1, const float* w2,
                                            float sum) {
  float s2 = 0.0f;
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const float4 bb = *reinterpret_cast<const float4*>(b1 + j);
    const float4 ww = *reinterpret_cast<const float4*>(w2 + j);
    sum = fmaf(ww.x, gelu_as(__uint_as_float(r[j]) + bb.x), sum);
    s2 = fmaf(ww.y, gelu_as(__uint_as_float(r[j + 1]) + bb.y), s2);
    sum = fmaf(ww.z, gelu_as(__uint_as_float(r[j + 2]) + bb.z), sum);
    s2 = fmaf(ww.w, gelu_as(__uint_as_float(r[j + 3]) + bb.w), s2);
  }
  return sum + s2;
}

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// ---- CUDA-core path: one warp per token -----------------------------------
template <typename T>
__global__ void __launch_bounds__(256) gate_simt_kernel(const T* __restrict__ h, int64_t n, int d,
                                                        const T* __restrict__ W1,
                                                        const float* __restrict__ b1, int dg,
                                                        const float* __restrict__ w2, float b2,
                                                        float* __restrict__ z,
                                                        const __grid_constant__ GateHist gh) {
  const int lane = threadIdx.x & 31;
  grid_dep_wait();
  grid_dep_launch();
  gate_hist_tags(gh, 0, blockDim.x);
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       j < n; j += warps) {
    const T* hj = h + j * d;
    float zsum = 0.0f;
    for (int u = 0; u < dg; ++u) {
      const T* wu = W1 + static_cast<int64_t>(u) * d;
      float acc = 0.0f;
      for (int c = lane; c < d; c += 32) acc = fmaf(to_f(__ldg(wu + c)), to_f(hj[c]), acc);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      zsum = fmaf(__ldg(w2 + u), gelu_erf(acc + __ldg(b1 + u)), zsum);
    }
    if (lane == 0) z[j] = zsum + b2;
    if (gh.hist) gate_hist_add(gh, static_cast<int>(j), zsum + b2, lane == 0);
  }
}

// ---- tensor-core path -------------------------------------------------------
constexpr int kBM = 128;
constexpr int kBK = 64;  // 64 bf16 = one 128-byte swizzle row
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr uint32_t kAccCols = 256;  // columns per accumulator (d_hidden <= 256)
constexpr uint32_t kTmemCols = 512;

struct GateTcParams {
  const float* b1;
  const float* w2;
  float* z;
  uint32_t* status;
  float b2;
  int32_t n;
  int32_t d;
  int32_t dg;
  int32_t num_tiles;
};

struct GateSmemLayout {
  uint32_t stage_bytes, a_bytes;
  uint32_t bars_off, misc_off, b1_off, w2_off, total;
  __host__ __device__ GateSmemLayout(int dg) {
    a_bytes = kBM * kBK * 2;
    stage_bytes = a_bytes + static_cast<uint32_t>(dg) * kBK * 2;
    bars_off = kStages * stage_bytes;
    misc_off = bars_off + 16 * 8;
    b1_off = misc_off + 16;
    w2_off = b1_off + 256 * 4;
    total = w2_off + 256 * 4;
  }
};

__global__ void __launch_bounds__(kThreads, 1)
    gate_tc_kernel(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ GateTcParams p, const __grid_constant__ GateHist gh) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const GateSmemLayout L(p.dg);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars_off);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc_off + 4);
  float* s_b1 = reinterpret_cast<float*>(smem + L.b1_off);
  float* s_w2 = reinterpret_cast<float*>(smem + L.w2_off);
  // barrier indices: full[0..3], empty[4..7], tmem_full[8..9], tmem_empty[10..11]
  auto bar = [&](int i) { return smem_u32(bars + i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = p.d / kBK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(s), 1);
      mbar_init(bar(4 + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(8 + a), 1);
      mbar_init(bar(10 + a), 128);
    }
    *abort_flag = 0;
    mbar_fence_init();
    prefetch_tmap(&tm_h);
    prefetch_tmap(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (warp >= 2) {
    for (int i = threadIdx.x - 64; i < p.dg; i += 128) {
      s_b1[i] = p.b1[i];
      s_w2[i] = p.w2[i];
    }
    gate_hist_tags(gh, 64, 128);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dep_wait();  // (launched in stream order: returns at once)
  grid_dep_launch();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!(ok = mbar_wait(bar(4 + stage), phase ^ 1, abort_flag, p.status, kDevTimeoutGate)))
            break;
          const uint32_t sa = smem_u32(smem + stage * L.stage_bytes);
          mbar_arrive_expect_tx(bar(stage), L.stage_bytes);
          tma_load_2d_hint(sa, &tm_h, kb * kBK, tile * kBM, bar(stage), pol_stream);
          tma_load_2d_hint(sa + L.a_bytes, &tm_w, kb * kBK, 0, bar(stage), pol_keep);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, p.dg, false, false);
      int stage = 0;
      uint32_t phase = 0, acc = 0, acc_phase = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
        if (!mbar_wait(bar(10 + acc), acc_phase ^ 1, abort_flag, p.status, kDevTimeoutGate)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!(ok = mbar_wait(bar(stage), phase, abort_flag, p.status, kDevTimeoutGate))) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * L.stage_bytes);
          const uint32_t sb = sa + L.a_bytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            umma_ss(d_tmem, sw128_desc(sa + k * 32, 16, 1024), sw128_desc(sb + k * 32, 16, 1024),
                    idesc, (kb | k) != 0);
          }
          umma_commit(bar(4 + stage));  // stage free once these MMAs have read it
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(bar(8 + acc));  // accumulator ready for the epilogue
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int row_local = quarter * 32 + lane;
    uint32_t acc = 0, acc_phase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      if (!mbar_wait(bar(8 + acc), acc_phase, abort_flag, p.status, kDevTimeoutGate)) break;
      tc_fence_after();
      const uint32_t t_addr =
          tmem_base + acc * kAccCols + (static_cast<uint32_t>(quarter * 32) << 16);
      float sum = 0.0f;
      for (int c = 0; c < p.dg; c += 32) {
        uint32_t r[32];
        tmem_ld32(t_addr + c, r);
        tmem_ld_wait(r);
        sum = gelu_dot32(r, s_b1 + c, s_w2 + c, sum);
      }
      tc_fence_before();
      mbar_arrive(bar(10 + acc));
      const int row = tile * kBM + row_local;
      if (row < p.n) p.z[row] = sum + p.b2;
      if (gh.hist) gate_hist_add(gh, row, sum + p.b2, row < p.n);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---- tensor-core path on CTA pairs (tcgen05 cta_group::2) ---------------------
// Same dataflow as gate_tc_kernel, but a cluster of two CTAs computes one
// 256-row tile with M=256 MMAs: each CTA stages its own 128 residual rows and
// only half of W1 (d_hidden/2 rows), so every SM streams 32 KB per k-block
// instead of 48 KB and the W1 re-read from L2 per residual row halves.  The
// even CTA issues the MMAs for both; its barriers count both CTAs' TMA bytes and
// both epilogues' releases, and it signals the odd CTA's barriers with a second
// commit.
// A stage covers 128 columns of the residual (two adjacent 128-byte swizzle boxes
// per row), so each row contributes 256 contiguous bytes per TMA round.
constexpr int kStages2 = 3;
constexpr int kThreads2 = 320;  // TMA warp, MMA warp, 8 epilogue warps (2 per TMEM lane quarter)
constexpr int kBK2 = 128;

struct Gate2Layout {
  uint32_t stage_bytes, a_bytes, a_box, b_box;
  uint32_t bars_off, misc_off, b1_off, w2_off, part_off, total;
  __host__ __device__ Gate2Layout(int dg) {
    a_box = kBM * kBK * 2;                             // 128 rows x 64 cols
    b_box = static_cast<uint32_t>(dg / 2) * kBK * 2;   // dg/2 rows x 64 cols
    a_bytes = (kBK2 / kBK) * a_box;
    stage_bytes = a_bytes + (kBK2 / kBK) * b_box;
    bars_off = kStages2 * stage_bytes;
    misc_off = bars_off + 24 * 8;
    b1_off = misc_off + 16;
    w2_off = b1_off + 256 * 4;
    part_off = w2_off + 256 * 4;  // [2 accumulators][128 rows] partial row sums
    total = part_off + 2 * 128 * 4;
  }
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads2, 1)
    gate_tc2_kernel(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w,
                    const __grid_constant__ GateTcParams p, const __grid_constant__ GateHist gh) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const Gate2Layout L(p.dg);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars_off);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc_off + 4);
  float* s_b1 = reinterpret_cast<float*>(smem + L.b1_off);
  float* s_w2 = reinterpret_cast<float*>(smem + L.w2_off);
  // barrier indices: full[0..5], empty[6..11], tmem_full[12..13], tmem_empty[14..15]
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  auto leader_bar = [&](int i) { return mapa_shared(bar(i), 0); };
  auto peer_bar = [&](int i) { return mapa_shared(bar(i), 1); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = p.d / kBK2;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages2; ++s) {
      mbar_init(bar(s), 1);
      mbar_init(bar(6 + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(12 + a), 1);
      mbar_init(bar(14 + a), 512);  // both CTAs' epilogue threads
    }
    *abort_flag = 0;
    mbar_fence_init();
    prefetch_tmap(&tm_h);
    prefetch_tmap(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers and TMEM of both CTAs are ready
  tc_fence_after();
  grid_dep_wait();  // (launched in stream order: returns at once)
  grid_dep_launch();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = pair; tile < p.num_tiles; tile += npairs) {
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!(ok = mbar_wait(bar(6 + stage), phase ^ 1, abort_flag, p.status, kDevTimeoutGate)))
            break;
          const uint32_t sa = smem_u32(smem + stage * L.stage_bytes);
          if (leader) mbar_arrive_expect_tx(bar(stage), 2 * L.stage_bytes);
          for (int c = 0; c < kBK2 / kBK; ++c)
            tma_load_2d_pair(sa + c * L.a_box, &tm_h, kb * kBK2 + c * kBK,
                             tile * 2 * kBM + rank * kBM, leader_bar(stage), pol_stream);
          for (int c = 0; c < kBK2 / kBK; ++c)
            tma_load_2d_pair(sa + L.a_bytes + c * L.b_box, &tm_w, kb * kBK2 + c * kBK,
                             rank * (p.dg / 2), leader_bar(stage), pol_keep);
          if (++stage == kStages2) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      const uint32_t idesc = idesc_bf16_f32(2 * kBM, p.dg, false, false);
      int stage = 0;
      uint32_t phase = 0, acc = 0, acc_phase = 0;
      for (int tile = pair; tile < p.num_tiles; tile += npairs) {
        if (!mbar_wait(bar(14 + acc), acc_phase ^ 1, abort_flag, p.status, kDevTimeoutGate)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!(ok = mbar_wait(bar(stage), phase, abort_flag, p.status, kDevTimeoutGate))) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * L.stage_bytes);
          const uint32_t sb = sa + L.a_bytes;
#pragma unroll
          for (int k = 0; k < kBK2 / 16; ++k) {
            const uint32_t c = k >> 2, kx = (k & 3) * 32;
            umma_ss_pair(d_tmem, sw128_desc(sa + c * L.a_box + kx, 16, 1024),
                         sw128_desc(sb + c * L.b_box + kx, 16, 1024), idesc, (kb | k) != 0);
          }
          umma_commit_pair(leader_bar(6 + stage));  // both CTAs may refill this stage
          umma_commit_pair(peer_bar(6 + stage));
          if (++stage == kStages2) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_pair(leader_bar(12 + acc));  // both accumulator halves are ready
        umma_commit_pair(peer_bar(12 + acc));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
    }
    __syncwarp();
  } else {
    // warps 2-5 take the first half of the hidden columns, warps 6-9 the rest
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row_local = quarter * 32 + lane;
    const int c_split = ((p.dg / 32) / 2) * 32;
    const int c_lo = half ? c_split : 0, c_hi = half ? p.dg : c_split;
    float* s_part = reinterpret_cast<float*>(smem + L.part_off);
    // b1 and w2 into shared memory while the first tile's MMAs run
    for (int i = threadIdx.x - 64; i < p.dg; i += 256) {
      s_b1[i] = p.b1[i];
      s_w2[i] = p.w2[i];
    }
    gate_hist_tags(gh, 64, 256);
    named_barrier(2, 256);
    uint32_t acc = 0, acc_phase = 0;
    for (int tile = pair; tile < p.num_tiles; tile += npairs) {
      if (!mbar_wait(bar(12 + acc), acc_phase, abort_flag, p.status, kDevTimeoutGate)) break;
      tc_fence_after();
      const uint32_t t_addr =
          tmem_base + acc * kAccCols + (static_cast<uint32_t>(quarter * 32) << 16);
      float sum = 0.0f;
      for (int c = c_lo; c < c_hi; c += 32) {
        uint32_t r[32];
        tmem_ld32(t_addr + c, r);
        tmem_ld_wait(r);
        sum = gelu_dot32(r, s_b1 + c, s_w2 + c, sum);
      }
      tc_fence_before();
      mbar_arrive_cluster(leader_bar(14 + acc));
      if (half) s_part[acc * 128 + row_local] = sum;
      named_barrier(1, 256);  // both halves of every row are summed
      const int row = tile * 2 * kBM + static_cast<int>(rank) * kBM + row_local;
      if (!half) {
        const float zr = sum + s_part[acc * 128 + row_local] + p.b2;
        if (row < p.n) p.z[row] = zr;
        if (gh.hist) gate_hist_add(gh, row, zr, row < p.n);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no commit or arrival can still target the other CTA
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace

tg_status launch_gate_simt(const void* h, tg_dtype dt, int64_t n, int d, const void* W1,
                           const float* b1, int dg, const float* w2, float b2, float* z,
                           const GateHist& gh, cudaStream_t st) {
  const int64_t warps_needed = n;
  int64_t blocks = (warps_needed + 7) / 8;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  if (dt == TG_BF16)
    gate_simt_kernel<__nv_bfloat16><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(h), n, d, static_cast<const __nv_bfloat16*>(W1), b1, dg,
        w2, b2, z, gh);
  else
    gate_simt_kernel<float><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const float*>(h), n, d, static_cast<const float*>(W1), b1, dg, w2, b2, z, gh);
  return cuda_check(cudaGetLastError(), "gate_simt launch");
}

tg_status launch_gate_tc(const void* h, int64_t n, int d, const void* W1, const float* b1, int dg,
                         const float* w2, float b2, float* z, const GateHist& gh,
                         cudaStream_t st) {
  CUtensorMap tm_h, tm_w;
  // CTA-pair kernel (each CTA stages half of W1) when the 128-column stages tile d
  const bool pairs = num_sms() >= 2 && d % kBK2 == 0;
  if (!encode_tmap_2d_bf16(&tm_h, h, static_cast<uint64_t>(d), static_cast<uint64_t>(n),
                           static_cast<uint64_t>(d) * 2, kBK, kBM) ||
      !encode_tmap_2d_bf16(&tm_w, W1, static_cast<uint64_t>(d), static_cast<uint64_t>(dg),
                           static_cast<uint64_t>(d) * 2, kBK,
                           static_cast<uint32_t>(pairs ? dg / 2 : dg)))
    return set_error(TG_ERR_CUDA, "cuTensorMapEncodeTiled failed for the gate operands");
  GateTcParams p;
  p.b1 = b1;
  p.w2 = w2;
  p.z = z;
  p.status = device_status_word();
  if (!p.status) return set_error(TG_ERR_CUDA, "device status word unavailable");
  p.b2 = b2;
  p.n = static_cast<int32_t>(n);
  p.d = d;
  p.dg = dg;
  if (pairs) {
    p.num_tiles = static_cast<int32_t>((n + 2 * kBM - 1) / (2 * kBM));  // 256-row tiles
    const Gate2Layout L2(dg);
    const size_t smem2 = L2.total + 1024;
    tg_status r2 = cuda_check(cudaFuncSetAttribute(gate_tc2_kernel,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   static_cast<int>(smem2)),
                              "gate pair smem attribute");
    if (r2 != TG_OK) return r2;
    int npairs = num_sms() / 2;
    if (npairs > p.num_tiles) npairs = p.num_tiles;
    gate_tc2_kernel<<<2 * npairs, kThreads2, smem2, st>>>(tm_h, tm_w, p, gh);
    return cuda_check(cudaGetLastError(), "gate_tc2 launch");
  }
  p.num_tiles = static_cast<int32_t>((n + kBM - 1) / kBM);
  const GateSmemLayout L(dg);
  const size_t smem = L.total + 1024;
  tg_status r = cuda_check(cudaFuncSetAttribute(gate_tc_kernel,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                static_cast<int>(smem)),
                           "gate smem attribute");
  if (r != TG_OK) return r;
  int grid = num_sms();
  if (grid > p.num_tiles) grid = p.num_tiles;
  gate_tc_kernel<<<grid, kThreads, smem, st>>>(tm_h, tm_w, p, gh);
  return cuda_check(cudaGetLastError(), "gate_tc launch");
}

}  // namespace tg
