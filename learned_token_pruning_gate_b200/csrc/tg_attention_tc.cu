// Token-gated causal GQA attention, tensor-core path (bf16, head_dim 64/128).
//
// TokenGate adds each kept key's gate score to the attention logits above the
// gate as a bias scaled by a per-head learned gain (the Mixture-of-Experts
// router trick) and divides q.k by a per-head learned temperature:
//     logit_ij = q_i.k_j / (sqrt(d) tau_h) + g_h l_j,     j <= i in the prompt.
// In the log2 domain t = s * log2e/(sqrt(d) tau_h) + g_h log2e l_j, so bias
// and temperature cost one FMA per logit.
//
// Work item = (prompt, 128-query tile, pair of query heads sharing one KV
// head).  Both heads of a pair need exactly the same K/V tiles (0..tile), so a
// K/V tile is loaded once and feeds two independent softmax warpgroups that
// take turns with the tensor core (while one computes softmax, the tensor core
// runs the other's P.V and next Q.K^T).  The kernel is persistent: one CTA per
// SM.  Work units are items, or for small problems chunks of an item's key
// range, sorted longest first and dealt to the CTAs in boustrophedon order
// (0..G-1, then G-1..0, ...), which evens out the causal imbalance.  When an
// item is split, every chunk writes its normalised partial output and
// log-sum-exp to the caller's workspace; the chunk that finishes last (a
// counter per item and head, no waiting) merges all partials in chunk order,
// so the result does not depend on which chunk finishes last.
//
//   warp 0     TMA: both Q tiles of an item, then K and V tiles (128 keys)
//              into a ring of shared-memory stages (128-byte swizzle)
//   warp 1     TMEM owner (512 columns: S_a, S_b, O_a, O_b) and the single
//              tcgen05.mma issuer: S_x = Q_x K^T, O_x += P_x V with P_x read
//              from TMEM (bf16 written over S_x) and V MN-major from smem.
//              Issue order S_a0 S_b0 | PV_a0 S_a1 | PV_b0 S_b1 | ... relies on
//              tcgen05.mma executing in issue order.
//   warps 2-3  idle (they only complete warpgroup 0 for the register split)
//   warps 4-7  softmax for head a, warps 8-11 for head b: one query row per
//              thread; packed fp32x2 math; causal mask on the diagonal tile;
//              lazy rescaling: O is rescaled in TMEM only when a row's max
//              grows by more than 2^8 (the P.V of the previous tile is known
//              complete then, because this tile's S commit tracks it).
//              Epilogue: O / l -> bf16 -> global, LSE.
#include "tg_internal.cuh"

namespace tg {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kThreads = 384;  // 3 warpgroups
// Register split (launch: 384 threads x 168 = 64512): warpgroup 0 (TMA, MMA and
// two idle warps) shrinks to 104 per thread, the two softmax warpgroups grow to
// 192: 128*104 + 256*192 = 62464 <= 64512.
constexpr int kRegsProducer = 104;
constexpr int kRegsSoftmax = 192;
static_assert(128 * kRegsProducer + 256 * kRegsSoftmax <= kThreads * 168, "register split");
constexpr int kBM = 128;       // queries per tile
constexpr int kBN = 128;       // keys per tile
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;

constexpr int kMaxUnits = 2048;  // work units listed explicitly when items are split
constexpr int kMaxChunks = 4;    // chunks per split item

struct TcParams {
  int32_t kept_start[kMaxBatch + 1];
  int32_t order[kMaxBatch];      // prompts by query-tile count, descending
  int32_t nt_sorted[kMaxBatch];  // their query-tile counts
  const float* logsig;
  const float* gain;
  const float* temp;
  __nv_bfloat16* out;
  float* lse;
  uint32_t* status;
  int32_t batch;
  int32_t m_total;
  int32_t hq;
  int32_t group;          // query heads per KV head
  int32_t pairs_per_kvh;  // ceil(group / 2)
  int32_t pairs;          // head pairs per (prompt, query tile) = hkv * pairs_per_kvh
  int32_t n_items;
  int32_t n_units;        // = n_items unless items are split
  // split items: per slot and head, [DH/4][128] float4 (a warp's rows contiguous),
  // the rows' log2-domain log-sum-exp, and one arrival counter per item and head
  float4* part_o;
  float* part_lse;
  int32_t* part_cnt;
};

// Explicit unit list (split plans only): .x item rank, .y = slot << 8 | chunk << 4 | chunks.
template <bool kSplit>
struct UnitTable {
  int32_t unused;
};
template <>
struct UnitTable<true> {
  int2 unit[kMaxUnits];
};

template <int DH>
struct Lay {
  static constexpr uint32_t kChunks = DH / 64;
  static constexpr uint32_t kBox = 128 * 128;           // 128 rows x 64 bf16 (16 KB)
  static constexpr uint32_t kTile = kChunks * kBox;     // one 128-row Q/K/V tile
  static constexpr int kStages = DH == 64 ? 4 : 2;
  static constexpr uint32_t kQa = 0;
  static constexpr uint32_t kQb = kTile;
  static constexpr uint32_t kK = 2 * kTile;
  static constexpr uint32_t kV = kK + kStages * kTile;
  // operands of the bias step of S: A_a, A_b (per head) and B_0, B_1 (per key
  // tile, by tile parity), each 128 rows x 16 bf16, K-major without swizzle:
  // rows of 16 bytes for k = 0..7, then 2 KB of zeros for k = 8..15
  static constexpr uint32_t kAugTile = 4096;
  static constexpr uint32_t kAug = kV + kStages * kTile;
  static constexpr uint32_t kBars = kAug + 4 * kAugTile;
  static constexpr uint32_t kMisc = kBars + 32 * 8;
  static constexpr uint32_t kTotal = kMisc + 16;  // tmem slot, abort flag, last-chunk flags[2]
  static constexpr uint32_t kDynSmem = kTotal + 1024;
};

// barrier slots
enum {
  kQFull = 0,
  kQEmpty = 1,
  kSFull = 2,   // [2]
  kPFull = 4,   // [2]
  kOFull = 6,   // [2]
  kOFree = 8,   // [2]
  kKFull = 10,  // [stages]
  kAugFull = 22,  // [2] bias operands of an item's first tile written
  kDrain = 31,  // MMA completion on the way out after an abort
};

struct Item {
  int b, t, ha, hb, hk;
  bool has_b;
};

// Number of items at query-tile levels >= t.
__device__ __forceinline__ int items_at_or_above(const TcParams& p, int t) {
  int s = 0;
  for (int k = 0; k < p.batch; ++k) {
    const int d = p.nt_sorted[k] - t;
    if (d <= 0) break;
    s += d;
  }
  return s * p.pairs;
}

// Item of rank r in longest-first order: levels (query tile index) descending,
// then prompts (longest first), then head pairs.
__device__ __forceinline__ Item decode_item(const TcParams& p, int r) {
  int lo = 0, hi = p.nt_sorted[0] - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (items_at_or_above(p, mid) > r) lo = mid; else hi = mid - 1;
  }
  const int idx = r - items_at_or_above(p, lo + 1);
  const int k = idx / p.pairs, pr = idx - k * p.pairs;
  Item it;
  it.b = p.order[k];
  it.t = lo;
  const int g = pr / p.pairs_per_kvh, pp = pr - g * p.pairs_per_kvh;
  it.hk = g;
  it.ha = g * p.group + 2 * pp;
  it.hb = it.ha + 1;
  it.has_b = 2 * pp + 1 < p.group;
  return it;
}

struct Unit {
  Item it;
  int j0, j1;     // key tiles [j0, j1) of the item's 0..t
  int c, n;       // chunk c of n (n = 1: the whole item)
  int slot;       // first partial slot of a split item
};

template <bool kSplit>
__device__ __forceinline__ Unit decode_unit(const TcParams& p, const UnitTable<kSplit>& tab, int u) {
  Unit w;
  if constexpr (kSplit) {
    const int2 e = tab.unit[u];
    w.it = decode_item(p, e.x);
    w.n = e.y & 15;
    w.c = (e.y >> 4) & 15;
    w.slot = e.y >> 8;
    const int nkv = w.it.t + 1;
    w.j0 = w.c * nkv / w.n;
    w.j1 = (w.c + 1) * nkv / w.n;
  } else {
    w.it = decode_item(p, u);
    w.n = 1;
    w.c = 0;
    w.slot = 0;
    w.j0 = 0;
    w.j1 = w.it.t + 1;
  }
  return w;
}

// Unit of round k for CTA r of G: boustrophedon order over the sorted units.
__device__ __forceinline__ int snake_unit(int k, int r, int g) {
  return k * g + ((k & 1) ? g - 1 - r : r);
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

template <int DH, bool kSplit>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ TcParams p,
                   const __grid_constant__ UnitTable<kSplit> tab) {
  using L = Lay<DH>;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);
  static_assert(kKFull + 3 * S <= kAugFull, "barrier slots");
  uint8_t* s_aug = smem + L::kAug;
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  auto k_full = [&](int s) { return bar(kKFull + s); };
  auto v_full = [&](int s) { return bar(kKFull + S + s); };
  auto kv_empty = [&](int s) { return bar(kKFull + 2 * S + s); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    mbar_init(bar(kQFull), 1);
    mbar_init(bar(kQEmpty), 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(kSFull + x), 1);
      mbar_init(bar(kPFull + x), 128);
      mbar_init(bar(kOFull + x), 1);
      mbar_init(bar(kOFree + x), 128);
      mbar_init(bar(kAugFull + x), 128);
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    mbar_init(bar(kDrain), 1);
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
  // the zero halves (k = 8..15) of the bias operands are never written again
  for (int i = threadIdx.x; i < static_cast<int>(4 * L::kAugTile / 16); i += kThreads)
    reinterpret_cast<uint4*>(s_aug)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dep_wait();  // q', k', v' and the log-gates are complete
  grid_dep_launch();
  const uint32_t tmem = *tmem_slot;

  int q_loads = 0, tiles_loaded = 0;  // producer thread: loads issued (for the abort drain)
  if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsProducer));
  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int rs = 0;
      uint32_t rph = 0, q_waits = 0;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int u = snake_unit(round, blockIdx.x, gridDim.x);
        if (u >= p.n_units) break;
        const Unit w = decode_unit<kSplit>(p, tab, u);
        const Item& it = w.it;
        const int32_t kstart = p.kept_start[it.b];
        if (!(ok = mbar_wait(bar(kQEmpty), (q_waits++ & 1) ^ 1, abort_flag, p.status,
                             kDevTimeoutAttn)))
          break;
        mbar_arrive_expect_tx(bar(kQFull), L::kTile * (it.has_b ? 2 : 1));
        ++q_loads;
        for (uint32_t c = 0; c < L::kChunks; ++c) {
          tma_load_2d(sb + L::kQa + c * L::kBox, &tm_q, it.ha * DH + c * 64, kstart + it.t * kBM,
                      bar(kQFull));
          if (it.has_b)
            tma_load_2d(sb + L::kQb + c * L::kBox, &tm_q, it.hb * DH + c * 64,
                        kstart + it.t * kBM, bar(kQFull));
        }
        for (int j = w.j0; j < w.j1; ++j) {
          if (!(ok = mbar_wait(kv_empty(rs), rph ^ 1, abort_flag, p.status, kDevTimeoutAttn)))
            break;
          const int krow = kstart + j * kBN;
          ++tiles_loaded;
          mbar_arrive_expect_tx(k_full(rs), L::kTile);
          for (uint32_t c = 0; c < L::kChunks; ++c)
            tma_load_2d(sb + L::kK + rs * L::kTile + c * L::kBox, &tm_k, it.hk * DH + c * 64, krow,
                        k_full(rs));
          mbar_arrive_expect_tx(v_full(rs), L::kTile);
          for (uint32_t c = 0; c < L::kChunks; ++c)
            tma_load_2d(sb + L::kV + rs * L::kTile + c * L::kBox, &tm_v, it.hk * DH + c * 64, krow,
                        v_full(rs));
          if (++rs == S) {
            rs = 0;
            rph ^= 1;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, DH, false, true);
      auto wt = [&](uint32_t b, uint32_t par) {
        return mbar_wait(b, par, abort_flag, p.status, kDevTimeoutAttn);
      };
      // S_x = Q_x K^T for head x with the K tile in stage s
      // Descriptors are built once; a k-step or a stage only moves the start
      // address, which is the low field (address >> 4) of the descriptor, so each
      // MMA costs one add.  (Shared memory stays below 256 KB: no carry out.)
      const uint64_t d_q[2] = {sw128_desc(sb + L::kQa, 16, 1024), sw128_desc(sb + L::kQb, 16, 1024)};
      const uint64_t d_k0 = sw128_desc(sb + L::kK, 16, 1024);
      const uint64_t d_v0 = sw128_desc(sb + L::kV, L::kBox, 1024);
      const uint64_t d_aug_a = nosw_desc(sb + L::kAug, 2048, 128);
      const uint64_t d_aug_b = nosw_desc(sb + L::kAug + 2 * L::kAugTile, 2048, 128);
      constexpr uint32_t kAug16 = L::kAugTile >> 4;
      // S_x = Q_x K^T + A_x B^T for head x, K tile in stage s, bias operand B of
      // tile parity tp
      auto issue_s = [&](int x, int s, uint32_t tp) {
        const uint64_t dq = d_q[x];
        const uint64_t dk = d_k0 + ((s * L::kTile) >> 4);
        const uint32_t ts = tmem + x * 128;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          constexpr uint32_t kBox16 = L::kBox >> 4;
          const uint32_t off = (kk >> 2) * kBox16 + (kk & 3) * 2;
          umma_ss(ts, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_ss(ts, d_aug_a + x * kAug16, d_aug_b + tp * kAug16, idesc_qk, 1u);
        umma_commit(bar(kSFull + x));
      };
      // O_x (+)= P_x V with the V tile in stage s
      auto issue_pv = [&](int x, int s, bool acc) {
        const uint64_t dv = d_v0 + ((s * L::kTile) >> 4);
        const uint32_t to = tmem + 256 + x * 128, tp = tmem + x * 128;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          umma_ts(to, tp + kk * 8, dv + kk * (2048 >> 4), idesc_pv, (acc || kk > 0) ? 1u : 0u);
      };
      int rs = 0;
      uint32_t rph = 0, q_waits = 0, p_waits[2] = {0, 0}, of_waits[2] = {0, 0};
      uint32_t aug_waits[2] = {0, 0}, tile_base = 0;  // tiles of earlier units
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int u = snake_unit(round, blockIdx.x, gridDim.x);
        if (u >= p.n_units) break;
        const Unit w = decode_unit<kSplit>(p, tab, u);
        const Item& it = w.it;
        const int n_kv = w.j1 - w.j0;
        if (!(ok = wt(bar(kQFull), q_waits++ & 1))) break;
        if (!(ok = wt(k_full(rs), rph))) break;
        if (!(ok = wt(bar(kAugFull + 0), aug_waits[0]++ & 1))) break;
        tc_fence_after();
        issue_s(0, rs, tile_base & 1);
        if (it.has_b) {
          if (!(ok = wt(bar(kAugFull + 1), aug_waits[1]++ & 1))) break;
          tc_fence_after();
          issue_s(1, rs, tile_base & 1);
        }
        if (n_kv == 1) umma_commit(bar(kQEmpty));
        for (int j = 0; ok && j < n_kv; ++j) {
          int ns = rs + 1;
          uint32_t nph = rph;
          if (ns == S) {
            ns = 0;
            nph ^= 1;
          }
          const bool more = j + 1 < n_kv;
          // head a: P_a(j) V_j, then S_a(j+1); the tiles are waited for first, so once
          // P_a arrives both groups of MMAs issue back to back
          if (!(ok = wt(v_full(rs), rph))) break;
          if (more && !(ok = wt(k_full(ns), nph))) break;
          if (!(ok = wt(bar(kPFull + 0), p_waits[0]++ & 1))) break;
          if (j == 0 && !(ok = wt(bar(kOFree + 0), (of_waits[0]++ & 1) ^ 1))) break;
          tc_fence_after();
          issue_pv(0, rs, j > 0);
          if (!more) umma_commit(bar(kOFull + 0));
          if (more) {
            issue_s(0, ns, (tile_base + j + 1) & 1);
            if (!it.has_b && j + 2 == n_kv) umma_commit(bar(kQEmpty));
          }
          // head b: P_b(j) V_j, then S_b(j+1)
          if (it.has_b) {
            if (!(ok = wt(bar(kPFull + 1), p_waits[1]++ & 1))) break;
            if (j == 0 && !(ok = wt(bar(kOFree + 1), (of_waits[1]++ & 1) ^ 1))) break;
            tc_fence_after();
            issue_pv(1, rs, j > 0);
            if (!more) umma_commit(bar(kOFull + 1));
          }
          umma_commit(kv_empty(rs));  // V_j (and K_j) no longer needed once these finish
          if (more && it.has_b) {
            issue_s(1, ns, (tile_base + j + 1) & 1);
            if (j + 2 == n_kv) umma_commit(bar(kQEmpty));
          }
          rs = ns;
          rph = nph;
        }
        tile_base += n_kv;
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------- softmax warpgroups ----------------
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    const int x = (warp - 4) >> 2;  // 0: head a (warps 4-7), 1: head b (warps 8-11)
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;  // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_off + x * 128;
    const uint32_t t_o = tmem + lane_off + 256 + x * 128;
    uint32_t s_waits = 0, o_waits = 0, tile_ctr = 0;
    bool ok = true;
    // A unit's output is packed in registers and stored only after the next
    // unit's bias operands are published: a release arrival waits for the
    // thread's earlier global stores, and the O-free and bias arrivals gate the
    // tensor core, so the stores must not precede them.
    uint32_t pend[DH / 32][16];
    uint4* pend_dst = nullptr;
    float* pend_lse = nullptr;
    float pend_lse_v = 0.0f;
    auto flush = [&]() {
      if (pend_dst) {
#pragma unroll
        for (int c = 0; c < DH / 32; ++c)
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            pend_dst[c * 4 + v4] = make_uint4(pend[c][4 * v4], pend[c][4 * v4 + 1],
                                              pend[c][4 * v4 + 2], pend[c][4 * v4 + 3]);
        pend_dst = nullptr;
      }
      if (pend_lse) {
        *pend_lse = pend_lse_v;
        pend_lse = nullptr;
      }
    };
    for (int round = 0; ok; ++round) {
      const int u = snake_unit(round, blockIdx.x, gridDim.x);
      if (u >= p.n_units) break;
      const Unit w = decode_unit<kSplit>(p, tab, u);
      const Item& it = w.it;
      if (x == 1 && !it.has_b) continue;
      const int head = x ? it.hb : it.ha;
      const int32_t kstart = p.kept_start[it.b];
      const int32_t len = p.kept_start[it.b + 1] - kstart;
      const int n_kv = w.j1 - w.j0;
      const float scale = kLog2e / (sqrtf(static_cast<float>(DH)) * __ldg(p.temp + head));
      const float2 sc2 = make_float2(scale, scale);
      // Bias operands.  S = Q K^T + A B^T with A row = [c_hi, c_lo, c_hi, c_lo] and
      // B row j = [l_hi, l_hi, l_lo, l_lo] (bf16 halves of c = g_h log2e / scale and
      // of the key's log-gate l_j), so S_ij = q.k + c l_j to about 2^-16 relative
      // and scale * S is the log2-domain logit.  Key rows beyond the prompt and
      // question keys carry l = 0.
      {
        const float cb = p.logsig ? __ldg(p.gain + head) * kLog2e / scale : 0.0f;
        const __nv_bfloat16 c_hi = __float2bfloat16_rn(cb);
        const __nv_bfloat16 c_lo = __float2bfloat16_rn(cb - __bfloat162float(c_hi));
        const __nv_bfloat162 ca = __halves2bfloat162(c_hi, c_lo);
        const uint32_t cw = *reinterpret_cast<const uint32_t*>(&ca);
        *reinterpret_cast<uint4*>(s_aug + x * L::kAugTile + rl * 16) = make_uint4(cw, cw, 0u, 0u);
      }
      auto load_l = [&](int key) {  // the key's log-gate (key index in the prompt)
        return (p.logsig && key < len) ? __ldg(p.logsig + kstart + key) : 0.0f;
      };
      auto aug_row = [](float lj) {  // bias operand row of a key
        lj = fmaxf(lj, -1e30f);
        const __nv_bfloat16 l_hi = __float2bfloat16_rn(lj);
        const __nv_bfloat16 l_lo = __float2bfloat16_rn(lj - __bfloat162float(l_hi));
        const __nv_bfloat162 h2 = __halves2bfloat162(l_hi, l_hi), o2 = __halves2bfloat162(l_lo, l_lo);
        return make_uint4(*reinterpret_cast<const uint32_t*>(&h2), *reinterpret_cast<const uint32_t*>(&o2),
                          0u, 0u);
      };
      auto aug_b_row = [&](uint32_t tile) {
        return reinterpret_cast<uint4*>(s_aug + (2 + (tile & 1)) * L::kAugTile + rl * 16);
      };
      // head a's warpgroup writes B for every tile: the first one now, tile j + 1
      // while tile j is in softmax (after S_j is complete, so both heads' S of the
      // tile that used the same parity are done); the log-gates are loaded one
      // tile ahead of their use
      float next_l = 0.0f;
      if (x == 0) {
        *aug_b_row(tile_ctr) = aug_row(load_l(w.j0 * kBN + rl));
        if (n_kv > 1) next_l = load_l((w.j0 + 1) * kBN + rl);
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(kAugFull + x));
      flush();  // the previous unit's output, now that its successor may start
      float m = -INFINITY, l = 0.0f;
      for (int j = 0; j < n_kv; ++j) {
        const int jabs = w.j0 + j;
        ok = mbar_wait(bar(kSFull + x), s_waits++ & 1, abort_flag, p.status, kDevTimeoutAttn);
        // one outcome for the whole warpgroup
        if (named_barrier_or(1 + x, 128, !ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(t_s + c * 32, sr[c]);
        if (x == 0 && j + 1 < n_kv) {
          *aug_b_row(tile_ctr + j + 1) = aug_row(next_l);
          fence_proxy_async_smem();  // ordered before this thread's P arrival below
          if (j + 2 < n_kv) next_l = load_l((jabs + 2) * kBN + rl);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_wait(sr[c]);
        // tile max of S (scale > 0, so it is the max of the logits), four
        // independent chains; on the diagonal tile key column c is visible to
        // row rl iff c <= rl
        float mxv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (jabs != it.t) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int e = 0; e < 32; e += 2)
              mxv[(c & 1) * 2 + ((e >> 1) & 1)] =
                  max3f(mxv[(c & 1) * 2 + ((e >> 1) & 1)], __uint_as_float(sr[c][e]),
                        __uint_as_float(sr[c][e + 1]));
          }
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const int col = c * 32 + e;
              if (col > rl) sr[c][e] = __float_as_uint(-INFINITY);
              if (col + 1 > rl) sr[c][e + 1] = __float_as_uint(-INFINITY);
              mxv[(c & 1) * 2 + ((e >> 1) & 1)] =
                  max3f(mxv[(c & 1) * 2 + ((e >> 1) & 1)], __uint_as_float(sr[c][e]),
                        __uint_as_float(sr[c][e + 1]));
            }
          }
        }
        const float mx = fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3])) * scale;
        // lazy rescale: move the reference max only when it grows by > 2^8
        float alpha = 1.0f;
        const bool grow = mx > m + kRescaleLog2;
        if (grow) {
          alpha = exp2_approx(m - mx);
          m = mx;
        }
        // p = 2^(t - m), row sum, and P (bf16 pairs) over the first 64 columns of S,
        // 32 keys (16 columns) at a time
        const float2 nm2 = make_float2(-m, -m);
        float2 acc[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 a2 = __ffma2_rn(
                make_float2(__uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1])), sc2, nm2);
            const float2 p2 = make_float2(exp2_approx(a2.x), exp2_approx(a2.y));
            acc[(e >> 1) & 1] = __fadd2_rn(acc[(e >> 1) & 1], p2);
            __nv_bfloat162 pp = __floats2bfloat162_rn(p2.x, p2.y);
            pk[e >> 1] = *reinterpret_cast<uint32_t*>(&pp);
          }
          tmem_st16(t_s + c * 16, pk);
        }
        l = fmaf(l, alpha, (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y));
        // The previous tile's P.V is complete (this tile's S commit tracked it) and
        // this tile's is not issued before P is marked full, so O may be rescaled
        // in place: done after the exponentials, when S holds no registers.
        // Warp-uniform: tcgen05.ld/st are collective.
        if (j > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll
          for (int c = 0; c < DH / 32; ++c) {
            uint32_t orow[32];
            tmem_ld32(t_o + c * 32, orow);
            tmem_ld_wait(orow);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 v2 = __fmul2_rn(
                  make_float2(__uint_as_float(orow[e]), __uint_as_float(orow[e + 1])),
                  make_float2(alpha, alpha));
              orow[e] = __float_as_uint(v2.x);
              orow[e + 1] = __float_as_uint(v2.y);
            }
            tmem_st32(t_o + c * 32, orow);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(kPFull + x));
      }
      if (!ok) break;
      tile_ctr += n_kv;
      // epilogue: O / l
      ok = mbar_wait(bar(kOFull + x), o_waits++ & 1, abort_flag, p.status, kDevTimeoutAttn);
      if (named_barrier_or(1 + x, 128, !ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int qi = it.t * kBM + rl;
      const float inv = 1.0f / l;
      __nv_bfloat16* out = p.out + (static_cast<int64_t>(kstart + qi) * p.hq + head) * DH;
      if (!kSplit || w.n == 1) {
#pragma unroll
        for (int c = 0; c < DH / 32; ++c) {
          uint32_t orow[32];
          tmem_ld32(t_o + c * 32, orow);
          tmem_ld_wait(orow);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            __nv_bfloat162 pp = __floats2bfloat162_rn(__uint_as_float(orow[2 * e]) * inv,
                                                      __uint_as_float(orow[2 * e + 1]) * inv);
            pend[c][e] = *reinterpret_cast<uint32_t*>(&pp);
          }
        }
        tc_fence_before();
        mbar_arrive(bar(kOFree + x));
        if (qi < len) pend_dst = reinterpret_cast<uint4*>(out);
        if (p.lse && qi < len) {
          pend_lse = p.lse + static_cast<int64_t>(head) * p.m_total + kstart + qi;
          pend_lse_v = (m + log2f(l)) * kLn2;
        }
      } else {
        // chunk of a split item: store the normalised partial and its log2 LSE
        constexpr int kV4 = DH / 4;
        float4* po = p.part_o + static_cast<int64_t>((w.slot + w.c) * 2 + x) * kV4 * 128 + rl;
#pragma unroll
        for (int c = 0; c < DH / 32; ++c) {
          uint32_t orow[32];
          tmem_ld32(t_o + c * 32, orow);
          tmem_ld_wait(orow);
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            __stcg(po + (c * 8 + v4) * 128,
                   make_float4(__uint_as_float(orow[4 * v4]) * inv, __uint_as_float(orow[4 * v4 + 1]) * inv,
                               __uint_as_float(orow[4 * v4 + 2]) * inv,
                               __uint_as_float(orow[4 * v4 + 3]) * inv));
        }
        const float lse_own = m + log2f(l);
        __stcg(p.part_lse + ((w.slot + w.c) * 2 + x) * 128 + rl, lse_own);
        // publish, then count arrivals; the last chunk to arrive merges.  O stays
        // in TMEM until then: the merge reads this chunk's own part from there.
        __threadfence();
        named_barrier(1 + x, 128);
        if (rl == 0) last_flag[x] = atomicAdd(p.part_cnt + w.slot * 2 + x, 1) == w.n - 1;
        named_barrier(1 + x, 128);
        if (last_flag[x]) {
          __threadfence();
          // weights in chunk order (the own LSE is the value stored above)
          float lc[kMaxChunks], wc[kMaxChunks];
          float mx = -INFINITY;
#pragma unroll
          for (int cc = 0; cc < kMaxChunks; ++cc) {
            lc[cc] = cc >= w.n ? -INFINITY
                     : cc == w.c ? lse_own
                                 : __ldcg(p.part_lse + ((w.slot + cc) * 2 + x) * 128 + rl);
            mx = fmaxf(mx, lc[cc]);
          }
          float wsum = 0.0f;
#pragma unroll
          for (int cc = 0; cc < kMaxChunks; ++cc) {
            wc[cc] = cc < w.n ? exp2f(lc[cc] - mx) : 0.0f;
            wsum += wc[cc];
          }
          const float winv = 1.0f / wsum;
#pragma unroll
          for (int cc = 0; cc < kMaxChunks; ++cc) wc[cc] *= winv;
          const float4* pb = p.part_o + static_cast<int64_t>(w.slot * 2 + x) * kV4 * 128 + rl;
          const int64_t slot_stride = 2 * kV4 * 128;
          // The sum runs over the chunks in index order with the very values
          // each chunk stored, so it does not depend on which chunk is last.
          // Two 32-column blocks per round: every partial read of a round is in
          // flight at once.
#pragma unroll 1
          for (int c2 = 0; c2 < DH / 32; c2 += 2) {
            float acc[2][32];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int e = 0; e < 32; ++e) acc[h][e] = 0.0f;
#pragma unroll 1
            for (int cc = 0; cc < w.n; ++cc) {
              if (cc == w.c) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  uint32_t orow[32];
                  tmem_ld32(t_o + (c2 + h) * 32, orow);
                  tmem_ld_wait(orow);
#pragma unroll
                  for (int e = 0; e < 32; ++e)
                    acc[h][e] = fmaf(wc[cc], __uint_as_float(orow[e]) * inv, acc[h][e]);
                }
              } else {
                float4 a[2][8];
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                  for (int v4 = 0; v4 < 8; ++v4)
                    a[h][v4] = __ldcg(pb + cc * slot_stride + ((c2 + h) * 8 + v4) * 128);
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                  for (int v4 = 0; v4 < 8; ++v4) {
                    acc[h][4 * v4] = fmaf(wc[cc], a[h][v4].x, acc[h][4 * v4]);
                    acc[h][4 * v4 + 1] = fmaf(wc[cc], a[h][v4].y, acc[h][4 * v4 + 1]);
                    acc[h][4 * v4 + 2] = fmaf(wc[cc], a[h][v4].z, acc[h][4 * v4 + 2]);
                    acc[h][4 * v4 + 3] = fmaf(wc[cc], a[h][v4].w, acc[h][4 * v4 + 3]);
                  }
              }
            }
            if (qi < len) {
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                uint32_t pkd[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                  __nv_bfloat162 pp = __floats2bfloat162_rn(acc[h][2 * e], acc[h][2 * e + 1]);
                  pkd[e] = *reinterpret_cast<uint32_t*>(&pp);
                }
                uint4* dst = reinterpret_cast<uint4*>(out + (c2 + h) * 32);
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4)
                  dst[v4] = make_uint4(pkd[4 * v4], pkd[4 * v4 + 1], pkd[4 * v4 + 2], pkd[4 * v4 + 3]);
              }
            }
          }
          if (p.lse && qi < len)
            p.lse[static_cast<int64_t>(head) * p.m_total + kstart + qi] = (mx + log2f(wsum)) * kLn2;
        }
        tc_fence_before();
        mbar_arrive(bar(kOFree + x));  // O may now be overwritten by the next unit
      }
    }
    flush();
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // a wait gave up: let the loads and MMAs already issued finish (bounded)
    // before the shared memory and TMEM are released
    if (warp == 0 && lane == 0) {
      if (q_loads > 0) mbar_drain(bar(kQFull), (q_loads - 1) & 1);
      for (int s = 0; s < S && s < tiles_loaded; ++s) {
        const uint32_t par = ((tiles_loaded - 1 - s) / S) & 1;
        mbar_drain(k_full(s), par);
        mbar_drain(v_full(s), par);
      }
    }
    if (warp == 1 && lane == 0) {
      umma_commit(bar(kDrain));
      mbar_drain(bar(kDrain), 0);
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Pair kernel (tcgen05 cta_group::2, head_dim 128, even GQA groups).
//
// A cluster of two CTAs takes one work unit: CTA 0 the unit's head a, CTA 1
// head b; the two query tiles form the M = 256 rows of every MMA.  Both heads
// read the same K and V tiles, so each CTA stages only half of them (K: 64 of
// the 128 keys, V: 64 of the 128 dims) and the pair's MMAs read the other half
// from the peer: per SM, Q.K^T reads 6 KB instead of 8 KB of shared memory per
// k-step.  With one head per CTA, TMEM holds two S buffers and two output
// accumulators (4 x 128 columns): the key tiles of a unit alternate between
// two softmax warpgroups, each with its own S buffer, running max, row sum and
// O, so one warpgroup's softmax overlaps the other's and the tensor core's
// work, and no tile waits for the previous tile's softmax.  The epilogue
// merges the two partial results (the same rule as merging key-range chunks).
//
//   warp 0     TMA (each CTA): its Q tile, its halves of K and V tiles into
//              two rings; the bytes of both CTAs are counted on CTA 0's barriers
//   warp 1     CTA 0 only: TMEM allocation for the pair and the single MMA
//              issuer: S(0) S(1) | P(j).V_j -> O_(j mod 2), S(j+2) | ...;
//              commits go to the barriers of both CTAs
//   warps 2-3  idle (they complete warpgroup 0 for the register split)
//   warps 4-7  softmax of the even key tiles of this CTA's head, warps 8-11 of
//              the odd ones; one query row per thread.  Epilogue: the two
//              warpgroups merge O_0 and O_1, each for half of the columns.
// ---------------------------------------------------------------------------
constexpr int kPairThreads = 384;
// Three stages each: at a unit boundary the rings refill at once, and those TMA
// writes compete with the first MMAs of the next unit for shared memory; five
// stages were measured 1-6 % slower.
constexpr int kPKStages = 3, kPVStages = 3;

struct PairLay {
  static constexpr uint32_t kQBox = kBM * 128;          // 128 rows x 64 bf16
  static constexpr uint32_t kQ = 0;                     // 2 boxes (dims 0-63, 64-127)
  static constexpr uint32_t kKBox = 64 * 128;           // 64 keys x 64 bf16
  static constexpr uint32_t kKStage = 2 * kKBox;        // this CTA's 64 keys, all dims
  static constexpr uint32_t kVStage = 128 * 128;        // 128 keys x this CTA's 64 dims
  static constexpr uint32_t kK = 2 * kQBox;
  static constexpr uint32_t kV = kK + kPKStages * kKStage;
  // bias operands of S (as in the single-CTA kernel): A (this CTA's head),
  // B_0, B_1 (this CTA's 64 keys of the tiles in S buffer 0 / 1)
  static constexpr uint32_t kAugTile = 4096;
  static constexpr uint32_t kAug = kV + kPVStages * kVStage;
  static constexpr uint32_t kML = kAug + 3 * kAugTile;  // [2 warpgroups][128] float2 (m, l)
  static constexpr uint32_t kBars = kML + 2 * 128 * 8;
  static constexpr uint32_t kMisc = kBars + 48 * 8;
  static constexpr uint32_t kTotal = kMisc + 16;
  static constexpr uint32_t kDynSmem = kTotal + 1024;
  static_assert(kDynSmem <= 227 * 1024, "shared memory");
};

// barrier slots (same offsets in both CTAs)
enum {
  kPQFull = 0,     // CTA 0: Q bytes of both CTAs
  kPQEmpty = 1,    // each CTA
  kPSFull = 2,     // [2 buffers], each CTA
  kPPFull = 4,     // [2 buffers], CTA 0: 256 softmax threads
  kPOFull = 6,     // each CTA
  kPOFree = 7,     // CTA 0: 512 softmax threads
  kPAugFull = 8,   // CTA 0: 512 softmax threads, bias operands of a unit's first tiles
  kPDrain = 9,     // CTA 0
  kPKFull = 10,    // [K stages], CTA 0: both halves
  kPKEmpty = kPKFull + kPKStages,   // [K stages], each CTA
  kPVFull = kPKEmpty + kPKStages,   // [V stages], CTA 0
  kPVEmpty = kPVFull + kPVStages,   // [V stages], each CTA
  kPBarCount = kPVEmpty + kPVStages,
};
static_assert(kPBarCount <= 48, "barrier slots");

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ TcParams p) {
  constexpr int DH = 128;
  constexpr bool kSplit = false;  // units are whole items (the pair plan never splits)
  const UnitTable<false> tab{0};
  using L = PairLay;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  uint8_t* s_aug = smem + L::kAug;
  float2* s_ml = reinterpret_cast<float2*>(smem + L::kML);
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  auto leader_bar = [&](int i) { return mapa_shared(bar(i), 0); };
  // commit to the same barrier in both CTAs
  auto commit_both = [&](int i) { umma_commit_pair_both(bar(i)); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cl = blockIdx.x >> 1, ncl = gridDim.x >> 1;

  if (warp == 0 && lane == 0) {
    mbar_init(bar(kPQFull), 1);
    mbar_init(bar(kPQEmpty), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(kPSFull + b), 1);
      mbar_init(bar(kPPFull + b), 256);
    }
    mbar_init(bar(kPOFull), 1);
    mbar_init(bar(kPOFree), 512);
    mbar_init(bar(kPAugFull), 512);
    mbar_init(bar(kPDrain), 1);
    for (int s = 0; s < kPKStages; ++s) {
      mbar_init(bar(kPKFull + s), 1);
      mbar_init(bar(kPKEmpty + s), 1);
    }
    for (int s = 0; s < kPVStages; ++s) {
      mbar_init(bar(kPVFull + s), 1);
      mbar_init(bar(kPVEmpty + s), 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  // the zero halves (k = 8..15) of the bias operands are never written again
  for (int i = threadIdx.x; i < static_cast<int>(3 * L::kAugTile / 16); i += kPairThreads)
    reinterpret_cast<uint4*>(s_aug)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  tc_fence_before();
  cluster_sync_all();  // barriers and TMEM of both CTAs are ready
  tc_fence_after();
  grid_dep_wait();  // q', k', v' and the log-gates are complete
  grid_dep_launch();
  const uint32_t tmem = *tmem_slot;
  int q_loads = 0, k_loads = 0, v_loads = 0;  // CTA 0's TMA thread: for the abort drain

  if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsProducer));
  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();  // K/V tiles are re-read by later units
      int ks = 0, vs = 0;
      uint32_t kph = 0, vph = 0, q_waits = 0;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int u = snake_unit(round, cl, ncl);
        if (u >= p.n_units) break;
        const Unit w = decode_unit<kSplit>(p, tab, u);
        const Item& it = w.it;
        const int32_t kstart = p.kept_start[it.b];
        const int head = rank ? it.hb : it.ha;
        if (!(ok = mbar_wait(bar(kPQEmpty), (q_waits++ & 1) ^ 1, abort_flag, p.status,
                             kDevTimeoutAttn)))
          break;
        if (leader) {
          mbar_arrive_expect_tx(bar(kPQFull), 2 * 2 * L::kQBox);
          ++q_loads;
        }
        for (int c = 0; c < 2; ++c)
          tma_load_2d_pair(sb + L::kQ + c * L::kQBox, &tm_q, head * DH + c * 64, kstart + it.t * kBM,
                           leader_bar(kPQFull), pol);
        for (int j = w.j0; j < w.j1; ++j) {
          if (!(ok = mbar_wait(bar(kPKEmpty + ks), kph ^ 1, abort_flag, p.status, kDevTimeoutAttn)))
            break;
          if (leader) {
            mbar_arrive_expect_tx(bar(kPKFull + ks), 2 * L::kKStage);
            ++k_loads;
          }
          for (int c = 0; c < 2; ++c)
            tma_load_2d_pair(sb + L::kK + ks * L::kKStage + c * L::kKBox, &tm_k, it.hk * DH + c * 64,
                             kstart + j * kBN + static_cast<int>(rank) * 64, leader_bar(kPKFull + ks),
                             pol);
          if (++ks == kPKStages) {
            ks = 0;
            kph ^= 1;
          }
          if (!(ok = mbar_wait(bar(kPVEmpty + vs), vph ^ 1, abort_flag, p.status, kDevTimeoutAttn)))
            break;
          if (leader) {
            mbar_arrive_expect_tx(bar(kPVFull + vs), 2 * L::kVStage);
            ++v_loads;
          }
          tma_load_2d_pair(sb + L::kV + vs * L::kVStage, &tm_v,
                           it.hk * DH + static_cast<int>(rank) * 64, kstart + j * kBN,
                           leader_bar(kPVFull + vs), pol);
          if (++vs == kPVStages) {
            vs = 0;
            vph ^= 1;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer (CTA 0) ----------------
    if (lane == 0 && leader) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(2 * kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(2 * kBM, DH, false, true);
      uint32_t ph = 1u << kPOFree;  // bit i: parity to wait for on slot i ("free" starts passed)
      bool ok = true;
      auto wait_slot = [&](int slot) {
        ok = mbar_wait(bar(slot), (ph >> slot) & 1u, abort_flag, p.status, kDevTimeoutAttn);
        ph ^= 1u << slot;
        return ok;
      };
      const uint64_t dq = sw128_desc(sb + L::kQ, 16, 1024);
      const uint64_t dk0 = sw128_desc(sb + L::kK, 16, 1024);
      const uint64_t dv0 = sw128_desc(sb + L::kV, L::kVStage, 1024);
      const uint64_t d_aug_a = nosw_desc(sb + L::kAug, 2048, 128);
      const uint64_t d_aug_b = nosw_desc(sb + L::kAug + L::kAugTile, 2048, 128);
      // S(bf) = Q K^T + A B_bf^T (the second operand: 64 keys from each CTA)
      auto issue_s = [&](int bf, int ks) {
        const uint64_t dk = dk0 + ((ks * L::kKStage) >> 4);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk)
          umma_ss_pair(tmem + bf * 128, dq + (kk >> 2) * (L::kQBox >> 4) + (kk & 3) * 2,
                       dk + (kk >> 2) * (L::kKBox >> 4) + (kk & 3) * 2, idesc_qk, kk > 0 ? 1u : 0u);
        umma_ss_pair(tmem + bf * 128, d_aug_a, d_aug_b + bf * (L::kAugTile >> 4), idesc_qk, 1u);
      };
      int ks = 0, vs = 0;
      uint32_t kph = 0, vph = 0;
      for (int round = 0; ok; ++round) {
        const int u = snake_unit(round, cl, ncl);
        if (u >= p.n_units) break;
        const Unit w = decode_unit<kSplit>(p, tab, u);
        const int n_kv = w.j1 - w.j0;
        if (!wait_slot(kPQFull)) break;
        if (!wait_slot(kPAugFull)) break;
        const int pro = n_kv < 2 ? n_kv : 2;
        for (int j = 0; j < pro; ++j) {
          if (!(ok = mbar_wait(bar(kPKFull + ks), kph, abort_flag, p.status, kDevTimeoutAttn))) break;
          tc_fence_after();
          issue_s(j, ks);
          commit_both(kPSFull + j);
          commit_both(kPKEmpty + ks);
          if (++ks == kPKStages) {
            ks = 0;
            kph ^= 1;
          }
        }
        if (!ok) break;
        if (n_kv <= 2) commit_both(kPQEmpty);
        for (int j = 0; j < n_kv; ++j) {
          const int bf = j & 1;
          // the tiles first, so once P(j) arrives P.V and the next Q.K^T issue back to back
          if (!(ok = mbar_wait(bar(kPVFull + vs), vph, abort_flag, p.status, kDevTimeoutAttn))) break;
          if (j + 2 < n_kv &&
              !(ok = mbar_wait(bar(kPKFull + ks), kph, abort_flag, p.status, kDevTimeoutAttn)))
            break;
          if (!wait_slot(kPPFull + bf)) break;
          if (j == 0 && !wait_slot(kPOFree)) break;
          tc_fence_after();
          const uint64_t dv = dv0 + ((vs * L::kVStage) >> 4);
          // P(j) V_j into O_bf: the softmax warpgroup of this parity owns both
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            umma_ts_pair(tmem + 256 + bf * 128, tmem + bf * 128 + kk * 8, dv + kk * (2048 >> 4),
                         idesc_pv, (j > 1 || kk > 0) ? 1u : 0u);
          if (j + 1 == n_kv) commit_both(kPOFull);
          commit_both(kPVEmpty + vs);
          if (++vs == kPVStages) {
            vs = 0;
            vph ^= 1;
          }
          if (j + 2 < n_kv) {
            issue_s(bf, ks);  // P(j) in this buffer was read by the P.V above: in order
            commit_both(kPSFull + bf);
            commit_both(kPKEmpty + ks);
            if (++ks == kPKStages) {
              ks = 0;
              kph ^= 1;
            }
            if (j + 3 == n_kv) commit_both(kPQEmpty);  // that was the unit's last S
          }
        }
      }
    }
    __syncwarp();
  } else {
    // ---------------- softmax (warps 4-11, this CTA's head) ----------------
    if (warp < 4) {
      // warps 2-3: no role
    } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    const int x = static_cast<int>(rank);  // head slot within the pair
    const int wg = (warp - 4) >> 2;       // key tiles j with j mod 2 == wg, S buffer wg, O_wg
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_off + wg * 128;
    const uint32_t t_o = tmem + lane_off + 256 + wg * 128;
    uint32_t s_ph = 0, o_waits = 0;
    bool ok = true;
    // The output of a unit is packed in registers and stored only after the next
    // unit's bias operands are published, so no store of this thread is still
    // outstanding when it makes the O-free and bias arrivals that gate the
    // tensor core.
    uint32_t pend[2][16];
    uint4* pend_dst = nullptr;  // this thread's output row (columns of its warpgroup), or null
    float* pend_lse = nullptr;
    float pend_lse_v = 0.0f;
    auto flush = [&]() {
      if (pend_dst) {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc)
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            pend_dst[cc * 4 + v4] = make_uint4(pend[cc][4 * v4], pend[cc][4 * v4 + 1],
                                               pend[cc][4 * v4 + 2], pend[cc][4 * v4 + 3]);
        pend_dst = nullptr;
      }
      if (pend_lse) {
        *pend_lse = pend_lse_v;
        pend_lse = nullptr;
      }
    };
    for (int round = 0; ok; ++round) {
      const int u = snake_unit(round, cl, ncl);
      if (u >= p.n_units) break;
      const Unit w = decode_unit<kSplit>(p, tab, u);
      const Item& it = w.it;
      const int head = x ? it.hb : it.ha;
      const int32_t kstart = p.kept_start[it.b];
      const int32_t len = p.kept_start[it.b + 1] - kstart;
      const int n_kv = w.j1 - w.j0;
      const float scale = kLog2e / (sqrtf(static_cast<float>(DH)) * __ldg(p.temp + head));
      const float2 sc2 = make_float2(scale, scale);
      // bias operands: A (warpgroup 0) and this warpgroup's first B; this CTA holds
      // keys 64 * rank .. 64 * rank + 63 of each tile, one row per thread rl < 64
      if (wg == 0) {
        const float cb = p.logsig ? __ldg(p.gain + head) * kLog2e / scale : 0.0f;
        const __nv_bfloat16 c_hi = __float2bfloat16_rn(cb);
        const __nv_bfloat16 c_lo = __float2bfloat16_rn(cb - __bfloat162float(c_hi));
        const __nv_bfloat162 ca = __halves2bfloat162(c_hi, c_lo);
        const uint32_t cw = *reinterpret_cast<const uint32_t*>(&ca);
        *reinterpret_cast<uint4*>(s_aug + rl * 16) = make_uint4(cw, cw, 0u, 0u);
      }
      auto load_l = [&](int j) {  // log-gate of this thread's key in tile w.j0 + j
        const int key = (w.j0 + j) * kBN + static_cast<int>(rank) * 64 + rl;
        return (p.logsig && rl < 64 && key < len) ? __ldg(p.logsig + kstart + key) : 0.0f;
      };
      auto aug_row = [](float lj) {
        lj = fmaxf(lj, -1e30f);
        const __nv_bfloat16 l_hi = __float2bfloat16_rn(lj);
        const __nv_bfloat16 l_lo = __float2bfloat16_rn(lj - __bfloat162float(l_hi));
        const __nv_bfloat162 h2 = __halves2bfloat162(l_hi, l_hi), o2 = __halves2bfloat162(l_lo, l_lo);
        return make_uint4(*reinterpret_cast<const uint32_t*>(&h2), *reinterpret_cast<const uint32_t*>(&o2),
                          0u, 0u);
      };
      uint4* b_row = reinterpret_cast<uint4*>(s_aug + (1 + wg) * L::kAugTile + rl * 16);
      float next_l = 0.0f;
      if (wg < n_kv && rl < 64) *b_row = aug_row(load_l(wg));
      if (wg + 2 < n_kv) next_l = load_l(wg + 2);
      fence_proxy_async_smem();
      mbar_arrive_cluster(leader_bar(kPAugFull));
      flush();  // the previous unit's output, now that its successor may start
      float m = -INFINITY, l = 0.0f;
      for (int j = wg; j < n_kv; j += 2) {
        const int jabs = w.j0 + j;
        ok = mbar_wait(bar(kPSFull + wg), s_ph & 1u, abort_flag, p.status, kDevTimeoutAttn);
        s_ph ^= 1u;
        if (named_barrier_or(1 + wg, 128, !ok)) {  // one outcome for the warpgroup
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(t_s + c * 32, sr[c]);
        // B of tile j + 2 (same buffer): S(j) is complete, S(j + 2) waits for P(j)
        if (j + 2 < n_kv) {
          if (rl < 64) *b_row = aug_row(next_l);
          fence_proxy_async_smem();
          if (j + 4 < n_kv) next_l = load_l(j + 4);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_wait(sr[c]);
        float mxv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (jabs != it.t) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int e = 0; e < 32; e += 2)
              mxv[(c & 1) * 2 + ((e >> 1) & 1)] =
                  max3f(mxv[(c & 1) * 2 + ((e >> 1) & 1)], __uint_as_float(sr[c][e]),
                        __uint_as_float(sr[c][e + 1]));
          }
        } else {  // diagonal tile: key column c is visible to row rl iff c <= rl
#pragma unroll
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const int col = c * 32 + e;
              if (col > rl) sr[c][e] = __float_as_uint(-INFINITY);
              if (col + 1 > rl) sr[c][e + 1] = __float_as_uint(-INFINITY);
              mxv[(c & 1) * 2 + ((e >> 1) & 1)] =
                  max3f(mxv[(c & 1) * 2 + ((e >> 1) & 1)], __uint_as_float(sr[c][e]),
                        __uint_as_float(sr[c][e + 1]));
            }
          }
        }
        const float mx = fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3])) * scale;
        float alpha = 1.0f;
        const bool grow = mx > m + kRescaleLog2;
        if (grow) {
          alpha = exp2_approx(m - mx);
          m = mx;
        }
        const float2 nm2 = make_float2(-m, -m);
        float2 acc[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 a2 = __ffma2_rn(
                make_float2(__uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1])), sc2, nm2);
            const float2 p2 = make_float2(exp2_approx(a2.x), exp2_approx(a2.y));
            acc[(e >> 1) & 1] = __fadd2_rn(acc[(e >> 1) & 1], p2);
            __nv_bfloat162 pp = __floats2bfloat162_rn(p2.x, p2.y);
            pk[e >> 1] = *reinterpret_cast<uint32_t*>(&pp);
          }
          tmem_st16(t_s + c * 16, pk);
        }
        l = fmaf(l, alpha, (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y));
        // O_wg holds P.V of this warpgroup's earlier tiles; the last of them was
        // issued before S(j), which is complete, and P(j).V is not issued before
        // P is marked full: O_wg may be rescaled in place (warp-uniform)
        if (j > wg && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
          for (int c = 0; c < DH / 32; ++c) {
            uint32_t orow[32];
            tmem_ld32(t_o + c * 32, orow);
            tmem_ld_wait(orow);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 v2 = __fmul2_rn(
                  make_float2(__uint_as_float(orow[e]), __uint_as_float(orow[e + 1])),
                  make_float2(alpha, alpha));
              orow[e] = __float_as_uint(v2.x);
              orow[e + 1] = __float_as_uint(v2.y);
            }
            tmem_st32(t_o + c * 32, orow);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive_cluster(leader_bar(kPPFull + wg));
      }
      // both warpgroups take the same way out of the unit
      if (named_barrier_or(1 + wg, 128, !ok)) ok = false;
      if (ok) ok = mbar_wait(bar(kPOFull), o_waits++ & 1, abort_flag, p.status, kDevTimeoutAttn);
      s_ml[wg * 128 + rl] = make_float2(m, l);
      if (named_barrier_or(3, 256, !ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // merge: O = (2^(m0-M) O_0 + 2^(m1-M) O_1) / (2^(m0-M) l_0 + 2^(m1-M) l_1);
      // warpgroup 0 writes columns 0-63, warpgroup 1 columns 64-127
      const float2 ml0 = s_ml[rl], ml1 = s_ml[128 + rl];
      const bool two = n_kv > 1;
      const float mm = two ? fmaxf(ml0.x, ml1.x) : ml0.x;
      const float f0 = exp2f(ml0.x - mm), f1 = two ? exp2f(ml1.x - mm) : 0.0f;
      const float lsum = f0 * ml0.y + f1 * ml1.y;
      const float inv = 1.0f / lsum;
      const float g0 = f0 * inv, g1 = f1 * inv;
      const int qi = it.t * kBM + rl;
      __nv_bfloat16* out = p.out + (static_cast<int64_t>(kstart + qi) * p.hq + head) * DH;
      const uint32_t t_o0 = tmem + lane_off + 256, t_o1 = tmem + lane_off + 384;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = wg * 2 + cc;
        uint32_t o0[32], o1[32];
        tmem_ld32(t_o0 + c * 32, o0);
        if (two) tmem_ld32(t_o1 + c * 32, o1);
        tmem_ld_wait(o0);
        if (two) {
          tmem_ld_wait(o1);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o1[e] = 0u;
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float v0 = two ? fmaf(__uint_as_float(o0[2 * e]), g0, __uint_as_float(o1[2 * e]) * g1)
                               : __uint_as_float(o0[2 * e]) * g0;
          const float v1 = two ? fmaf(__uint_as_float(o0[2 * e + 1]), g0,
                                      __uint_as_float(o1[2 * e + 1]) * g1)
                               : __uint_as_float(o0[2 * e + 1]) * g0;
          __nv_bfloat162 pp = __floats2bfloat162_rn(v0, v1);
          pend[cc][e] = *reinterpret_cast<uint32_t*>(&pp);
        }
      }
      tc_fence_before();
      mbar_arrive_cluster(leader_bar(kPOFree));
      if (qi < len) pend_dst = reinterpret_cast<uint4*>(out + wg * 64);
      if (wg == 0 && p.lse && qi < len) {
        pend_lse = p.lse + static_cast<int64_t>(head) * p.m_total + kstart + qi;
        pend_lse_v = (mm + log2f(lsum)) * kLn2;
      }
    }
    flush();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && leader) {
    // a wait gave up: let the loads (both CTAs' bytes land on these barriers)
    // and the MMAs already issued finish (bounded) before memory is released
    if (warp == 0 && lane == 0) {
      if (q_loads > 0) mbar_drain(bar(kPQFull), (q_loads - 1) & 1);
      for (int s = 0; s < kPKStages && s < k_loads; ++s)
        mbar_drain(bar(kPKFull + s), ((k_loads - 1 - s) / kPKStages) & 1);
      for (int s = 0; s < kPVStages && s < v_loads; ++s)
        mbar_drain(bar(kPVFull + s), ((v_loads - 1 - s) / kPVStages) & 1);
    }
    if (warp == 1 && lane == 0) {
      umma_commit_pair(leader_bar(kPDrain));
      mbar_drain(bar(kPDrain), 0);
    }
  }
  __syncthreads();
  cluster_sync_all();  // no commit, arrival or load can still target the other CTA
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host: work plan.  Items are enumerated in the kernel's rank order (query-tile
// level descending, prompts longest first, head pairs); an item at level t has
// t + 1 key tiles.  For k = 1..kMaxChunks chunks of the longest item, items
// longer than C = ceil(max / k) tiles are cut into ceil(n / C) chunks; the plan
// with the smallest modelled makespan under the kernel's boustrophedon deal
// wins (a split must gain at least 3 % to be taken).  Cost model, in times of
// one key tile of a head pair on one SM (measured): a unit costs its tiles
// plus 0.5 (Q load, epilogue), a chunk of a split item 3 more (partial store
// and merge).  The pair kernel runs a tile in 0.72 of that, but on two SMs.
// ---------------------------------------------------------------------------
struct AttnPlan {
  double span = 0.0;  // modelled makespan (0: not modelled)
  int grid = 0;
  int n_units = 0;
  int n_slots = 0;
  bool split = false;
  size_t workspace = 0;
};

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

static size_t split_workspace_bytes(int n_slots, int dh) {
  return align256(static_cast<size_t>(n_slots) * 2 * sizeof(int32_t)) +
         align256(static_cast<size_t>(n_slots) * 2 * 128 * sizeof(float)) +
         static_cast<size_t>(n_slots) * 2 * 128 * dh * sizeof(float);
}

static void item_lengths(const TcParams& p, int32_t* nkv) {
  int r = 0;
  for (int t = p.nt_sorted[0] - 1; t >= 0; --t)
    for (int k = 0; k < p.batch && p.nt_sorted[k] > t; ++k)
      for (int pr = 0; pr < p.pairs; ++pr) nkv[r++] = t + 1;
}

static double snake_makespan(const double* cost_sorted, int n, int g, double* load) {
  for (int i = 0; i < g; ++i) load[i] = 0.0;
  for (int i = 0; i < n; ++i) {
    const int k = i / g, r = i - k * g;
    load[(k & 1) ? g - 1 - r : r] += cost_sorted[i];
  }
  double mx = 0.0;
  for (int i = 0; i < g; ++i) mx = load[i] > mx ? load[i] : mx;
  return mx;
}

// Fills `tab` (when non-null and the plan splits) and returns the plan.
static AttnPlan make_plan(const TcParams& p, int dh, int n_sms, bool allow_split,
                          UnitTable<true>* tab, double kTile, double kChunkCost) {
  constexpr double kOverhead = 0.5;
  AttnPlan best;
  best.n_units = p.n_items;
  best.grid = p.n_items < n_sms ? p.n_items : n_sms;
  if (p.n_items > kMaxUnits || p.n_items == 0) return best;
  const int n = p.n_items;
  int32_t nkv[kMaxUnits];
  item_lengths(p, nkv);
  const int max_n = nkv[0];
  // unit lists for one candidate: (cost, item, chunk, chunks)
  struct U {
    double cost;
    int item, c, s;
  };
  static thread_local U units[kMaxUnits], sorted[kMaxUnits];
  static thread_local double costs[kMaxUnits], load[1024];
  const int g_cap = n_sms < 1024 ? n_sms : 1024;
  double base = 0.0;
  double best_span = 0.0;
  for (int k = 1; k <= (allow_split ? kMaxChunks : 1); ++k) {
    const int C = (max_n + k - 1) / k;
    if (k > 1 && C == (max_n + k - 2) / (k - 1)) continue;
    int nu = 0;
    bool fits = true;
    for (int i = 0; i < n && fits; ++i) {
      const int s = (nkv[i] + C - 1) / C;
      if (nu + s > kMaxUnits) {
        fits = false;
        break;
      }
      for (int c = 0; c < s; ++c) {
        const int lo = c * nkv[i] / s, hi = (c + 1) * nkv[i] / s;
        units[nu++] = {kTile * (hi - lo) + kOverhead + (s > 1 ? kChunkCost : 0.0), i, c, s};
      }
    }
    if (!fits) continue;
    // stable sort by cost, descending (insertion into runs: costs take few values)
    int m = 0;
    for (int i = 0; i < nu; ++i) {
      int j = m++;
      while (j > 0 && sorted[j - 1].cost < units[i].cost) {
        sorted[j] = sorted[j - 1];
        --j;
      }
      sorted[j] = units[i];
    }
    for (int i = 0; i < nu; ++i) costs[i] = sorted[i].cost;
    const int g = nu < g_cap ? nu : g_cap;
    const double span = snake_makespan(costs, nu, g, load);
    if (k == 1) {
      base = best_span = span;
      continue;
    }
    if (span < best_span && span < 0.97 * base) {
      best_span = span;
      best.n_units = nu;
      best.grid = g;
      best.split = true;
      if (tab) {
        int slot = 0;
        // slots: consecutive per split item, in item order
        static thread_local int32_t item_slot[kMaxUnits];
        for (int i = 0; i < n; ++i) item_slot[i] = -1;
        for (int i = 0; i < nu; ++i)
          if (units[i].s > 1 && units[i].c == 0) {
            item_slot[units[i].item] = slot;
            slot += units[i].s;
          }
        for (int i = 0; i < nu; ++i) {
          const U& e = sorted[i];
          const int sl = e.s > 1 ? item_slot[e.item] : 0;
          tab->unit[i] = make_int2(e.item, (sl << 8) | (e.c << 4) | e.s);
        }
        best.n_slots = slot;
      } else {
        int slot = 0;
        for (int i = 0; i < nu; ++i)
          if (units[i].s > 1 && units[i].c == 0) slot += units[i].s;
        best.n_slots = slot;
      }
    }
  }
  best.span = best_span;
  if (best.split) best.workspace = split_workspace_bytes(best.n_slots, dh);
  return best;
}

static tg_status fill_params(const PromptTable& pt, int hq, int hkv, TcParams* pp) {
  TcParams& p = *pp;
  memset(&p, 0, sizeof(p));
  p.batch = pt.batch;
  for (int b = 0; b <= pt.batch; ++b) p.kept_start[b] = pt.kept_start[b];
  // prompts by query-tile count, descending (stable)
  int nt[kMaxBatch];
  for (int b = 0; b < pt.batch; ++b) {
    nt[b] = (pt.kept_start[b + 1] - pt.kept_start[b] + kBM - 1) / kBM;
    p.order[b] = b;
  }
  for (int i = 1; i < pt.batch; ++i) {
    const int xb = p.order[i];
    int j = i - 1;
    while (j >= 0 && nt[p.order[j]] < nt[xb]) {
      p.order[j + 1] = p.order[j];
      --j;
    }
    p.order[j + 1] = xb;
  }
  int64_t tiles = 0;
  for (int i = 0; i < pt.batch; ++i) {
    p.nt_sorted[i] = nt[p.order[i]];
    tiles += p.nt_sorted[i];
  }
  p.m_total = pt.kept_start[pt.batch];
  p.hq = hq;
  p.group = hq / hkv;
  p.pairs_per_kvh = (p.group + 1) / 2;
  p.pairs = hkv * p.pairs_per_kvh;
  const int64_t n_items = tiles * p.pairs;
  if (n_items > 0x7FFFFFFF) return set_error(TG_ERR_UNSUPPORTED, "too many attention tiles");
  p.n_items = static_cast<int32_t>(n_items);
  p.n_units = p.n_items;
  return TG_OK;
}

template <int DH, bool kSplit>
tg_status launch_dh(const void* q, const void* k, const void* v, const TcParams& p,
                    const UnitTable<kSplit>& tab, int grid, int hkv, cudaStream_t st) {
  using Ly = Lay<DH>;
  CUtensorMap tq, tk, tv;
  const uint64_t M = static_cast<uint64_t>(p.m_total);
  if (!encode_tmap_2d_bf16(&tq, q, static_cast<uint64_t>(p.hq) * DH, M,
                           static_cast<uint64_t>(p.hq) * DH * 2, 64, kBM) ||
      !encode_tmap_2d_bf16(&tk, k, static_cast<uint64_t>(hkv) * DH, M,
                           static_cast<uint64_t>(hkv) * DH * 2, 64, kBN) ||
      !encode_tmap_2d_bf16(&tv, v, static_cast<uint64_t>(hkv) * DH, M,
                           static_cast<uint64_t>(hkv) * DH * 2, 64, kBN))
    return set_error(TG_ERR_CUDA, "cuTensorMapEncodeTiled failed for q/k/v");
  tg_status r = cuda_check(cudaFuncSetAttribute(attn_tc_kernel<DH, kSplit>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                static_cast<int>(Ly::kDynSmem)),
                           "attn smem attribute");
  if (r != TG_OK) return r;
  if (kSplit) {  // the counter reset runs just before: plain stream order
    attn_tc_kernel<DH, kSplit><<<grid, kThreads, Ly::kDynSmem, st>>>(tq, tk, tv, p, tab);
    return cuda_check(cudaGetLastError(), "attn_tc launch");
  }
  return cuda_check(launch_pdl(attn_tc_kernel<DH, kSplit>, dim3(grid), dim3(kThreads), Ly::kDynSmem,
                               st, tq, tk, tv, p, tab),
                    "attn_tc launch");
}

tg_status launch_pair(const void* q, const void* k, const void* v, const TcParams& p, int clusters,
                      int hkv, cudaStream_t st) {
  constexpr int DH = 128;
  CUtensorMap tq, tk, tv;
  const uint64_t M = static_cast<uint64_t>(p.m_total);
  if (!encode_tmap_2d_bf16(&tq, q, static_cast<uint64_t>(p.hq) * DH, M,
                           static_cast<uint64_t>(p.hq) * DH * 2, 64, kBM) ||
      !encode_tmap_2d_bf16(&tk, k, static_cast<uint64_t>(hkv) * DH, M,
                           static_cast<uint64_t>(hkv) * DH * 2, 64, 64) ||
      !encode_tmap_2d_bf16(&tv, v, static_cast<uint64_t>(hkv) * DH, M,
                           static_cast<uint64_t>(hkv) * DH * 2, 64, kBN))
    return set_error(TG_ERR_CUDA, "cuTensorMapEncodeTiled failed for q/k/v");
  tg_status r = cuda_check(cudaFuncSetAttribute(attn_pair_kernel,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                static_cast<int>(PairLay::kDynSmem)),
                           "attn pair smem attribute");
  if (r != TG_OK) return r;
  return cuda_check(launch_pdl(attn_pair_kernel, dim3(2 * clusters), dim3(kPairThreads),
                               PairLay::kDynSmem, st, tq, tk, tv, p),
                    "attn_pair launch");
}

// CTA pairs need an even group (both heads of every pair exist) and head_dim 128.
// They can pay off only for small batches, whose items cannot fill one SM
// each (a unit then runs on two SMs); the single-CTA kernel, two softmax
// warpgroups per SM, has the higher throughput per SM.  The modelled
// makespans of the two plans decide.
constexpr double kTilePair = 0.55;  // pair kernel's tile time, in single-CTA tile times
constexpr double kMergeCost = 3.0;
static bool pairs_possible(const TcParams& p, int hkv, int dh) {
  return dh == 128 && (p.hq / hkv) % 2 == 0 && num_sms() >= 2 && p.n_items <= num_sms();
}
static AttnPlan choose_plan(const TcParams& p, int hkv, int dh, bool allow_split,
                            UnitTable<true>* tab_single, bool* pairs) {
  AttnPlan plan = make_plan(p, dh, num_sms(), allow_split, tab_single, 1.0, kMergeCost);
  *pairs = false;
  if (pairs_possible(p, hkv, dh)) {
    // whole items only: with two SMs per unit, splitting does not pay for its merges
    const AttnPlan pp = make_plan(p, dh, num_sms() / 2, false, nullptr, kTilePair, kMergeCost);
    if (pp.span > 0.0 && pp.span < plan.span) {
      plan = pp;
      *pairs = true;
    }
  }
  return plan;
}

}  // namespace

int attn_tc_kernel_choice(const PromptTable& pt, int hq, int hkv, int dh, bool with_workspace) {
  TcParams p;
  if (fill_params(pt, hq, hkv, &p) != TG_OK || p.n_items == 0) return TG_ATTN_TC;
  bool pairs = false;
  const AttnPlan plan = choose_plan(p, hkv, dh, with_workspace, nullptr, &pairs);
  return pairs ? TG_ATTN_TC_PAIR : plan.split ? TG_ATTN_TC_SPLIT : TG_ATTN_TC;
}

size_t attn_tc_workspace_bytes(const PromptTable& pt, int hq, int hkv, int dh) {
  TcParams p;
  if (fill_params(pt, hq, hkv, &p) != TG_OK || p.n_items == 0) return 0;
  bool pairs = false;
  return choose_plan(p, hkv, dh, true, nullptr, &pairs).workspace;
}

tg_status launch_attn_tc(const void* q, const void* k, const void* v, const PromptTable& pt,
                         int max_len, int hq, int hkv, int dh, const float* logsig,
                         const float* gain, const float* temp, void* out, float* lse,
                         void* workspace, size_t workspace_bytes, cudaStream_t st) {
  (void)max_len;
  TcParams p;
  tg_status r = fill_params(pt, hq, hkv, &p);
  if (r != TG_OK) return r;
  if (p.n_items == 0) return TG_OK;
  p.logsig = logsig;
  p.gain = gain;
  p.temp = temp;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  static thread_local UnitTable<true> tab;  // split plans are single-CTA plans
  bool pairs = false;
  const AttnPlan plan = choose_plan(p, hkv, dh, workspace != nullptr, &tab, &pairs);
  if (plan.split && workspace_bytes < plan.workspace)
    return set_error(TG_ERR_WORKSPACE, "attention workspace: %zu bytes given, %zu needed",
                     workspace_bytes, plan.workspace);
  p.status = device_status_word();
  if (!p.status) return set_error(TG_ERR_CUDA, "device status word unavailable");
  if (!plan.split) {
    const UnitTable<false> none{0};
    if (pairs) return launch_pair(q, k, v, p, plan.grid, hkv, st);
    if (dh == 64) return launch_dh<64, false>(q, k, v, p, none, plan.grid, hkv, st);
    return launch_dh<128, false>(q, k, v, p, none, plan.grid, hkv, st);
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t cnt_bytes = align256(static_cast<size_t>(plan.n_slots) * 2 * sizeof(int32_t));
  const size_t lse_bytes = align256(static_cast<size_t>(plan.n_slots) * 2 * 128 * sizeof(float));
  p.part_cnt = reinterpret_cast<int32_t*>(ws);
  p.part_lse = reinterpret_cast<float*>(ws + cnt_bytes);
  p.part_o = reinterpret_cast<float4*>(ws + cnt_bytes + lse_bytes);
  p.n_units = plan.n_units;
  r = cuda_check(cudaMemsetAsync(p.part_cnt, 0, cnt_bytes, st), "attention workspace counters");
  if (r != TG_OK) return r;
  if (dh == 64) return launch_dh<64, true>(q, k, v, p, tab, plan.grid, hkv, st);
  return launch_dh<128, true>(q, k, v, p, tab, plan.grid, hkv, st);
}

}  // namespace tg
