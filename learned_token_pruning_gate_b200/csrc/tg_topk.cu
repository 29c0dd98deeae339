// Top-K over each prompt's document span with the question protected
// (TokenGate: "a top-K selector keeps the highest-scoring tokens"; "only the
// document part of the prompt is pruned, the question is never touched").
//
// One cluster of 8 CTAs per (budget, prompt), one launch; each CTA owns a
// contiguous eighth of the prompt.  Several budgets (a budget sweep served by
// one scoring pass) select from the same scores in the same launch.  The keys
// are either fp32 gate scores or caller-drawn uint32 keys (the random-K
// selector ablation): larger first, lower index on ties, in both cases.
//  1. Each CTA caches its slice of the scores in shared memory as
//     order-preserving 32-bit keys (padded by one word per 32 so both strided
//     and per-thread-contiguous walks are free of bank conflicts).
//  2. Up to three radix passes (11, 11, 10 bits) find the K-th largest key T;
//     when every key of a pass's boundary bin is kept, the low bits cannot
//     change the set and the search stops there (T then fixes only the high
//     bits; usually the last pass is skipped for continuous scores).
//     The first pass's histogram comes from the gate when it counted these
//     scores into the top-K workspace (tg_gate_score_hist): every CTA reads
//     the prompt's 2048 bins and picks the digit itself, with no exchange;
//     in a budget sweep every budget takes its first digit from that one
//     histogram.
//     Otherwise, and for the later passes, each CTA adds its non-zero bins
//     into every CTA's totals with remote shared-memory atomics, one cluster
//     barrier publishes them, and every CTA scans its own copy, so all of them
//     take the same digit without waiting on a leader.  No thread waits on a
//     distributed-shared-memory read.
//  3. Ordered compaction: thread t owns a contiguous run of keys; one packed
//     block scan of (count of keys > T or protected, count of keys == T) gives
//     every thread its output offset and its rank among the ties (CTA totals
//     are pushed to the higher-ranked CTAs), so ties go to the lower index and
//     the kept rows come out in ascending order.
// The only waits are hardware barriers.  The only global scratch is the
// optional top-K workspace, which the call leaves zeroed for the next gate.
#include <cooperative_groups.h>

#include "tg_internal.cuh"

namespace cg = cooperative_groups;

namespace tg {
namespace {

constexpr int kThreads = 1024;
constexpr int kBins = kHistBins;
constexpr int kMaxCluster = 8;

struct TopkParams {
  PromptTable pt;  // prompt offsets and document spans (budget-independent fields)
  int32_t k_keep[TG_MAX_BUDGETS][kMaxBatch];          // per budget: min(K, n_doc)
  int32_t kept_start[TG_MAX_BUDGETS][kMaxBatch + 1];  // per budget: cu_kept
  int32_t* kept_idx[TG_MAX_BUDGETS];
  int32_t* cu_kept[TG_MAX_BUDGETS];
  const float* z;      // scores (kKeys = false)
  const uint32_t* keys;  // caller keys (kKeys = true)
  uint32_t* status;
  uint32_t* hist;      // top-K workspace with the gate's first-pass histograms, or null
  int32_t n_budgets;   // clusters per prompt that read the same histogram
  int32_t cluster;     // CTAs per (budget, prompt)
};

__host__ __device__ __forceinline__ int padded(int i) { return i + (i >> 5); }

// Exclusive scan of one value per thread over the block (thread order); also
// returns the block total.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* s_warp,
                                                    uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = s_warp[lane];
    uint32_t wx = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, wx, o);
      if (lane >= o) wx += y;
    }
    s_warp[lane] = wx - w;
    if (lane == 31) s_warp[32] = wx;
  }
  __syncthreads();
  const uint32_t r = s_warp[warp] + x - v;
  if (total) *total = s_warp[32];
  __syncthreads();
  return r;
}

// Run by every thread of a CTA over one pass's totals tot[0, nb): the digit d
// whose bin holds the k_rem-th largest key, i.e. the keys of larger digits
// number fewer than k_rem and those of digits >= d at least k_rem.  Writes
// (d, keys above d, keys in d's bin) to s_sel, zeroes tot for a later pass and
// returns the totals' sum.  Thread t owns bins nb-1-t*bpt-j (descending digit
// order), so an exclusive scan counts the larger digits.
__device__ uint32_t select_digit(uint32_t* tot, uint32_t nb, uint32_t k_rem, uint32_t* s_scan,
                                 uint32_t* s_sel) {
  const int tid = threadIdx.x;
  const uint32_t bpt = nb / kThreads;  // 2 or 1
  uint32_t cnt[2] = {0, 0};
  for (uint32_t j = 0; j < bpt; ++j) {
    const uint32_t bin = nb - 1 - tid * bpt - j;
    cnt[j] = tot[bin];
    tot[bin] = 0;
  }
  const uint32_t mine = cnt[0] + cnt[1];
  uint32_t total = 0;
  uint32_t above = block_excl_scan(mine, s_scan, &total);
  if (above < k_rem && above + mine >= k_rem) {
    for (uint32_t j = 0; j < bpt; ++j) {
      if (above + cnt[j] >= k_rem) {
        s_sel[0] = nb - 1 - tid * bpt - j;
        s_sel[1] = above;
        s_sel[2] = cnt[j];
        break;
      }
      above += cnt[j];
    }
  }
  __syncthreads();
  return total;
}

template <bool kKeys>
__global__ void __launch_bounds__(kThreads, 1) topk_kernel(const __grid_constant__ TopkParams p) {
  extern __shared__ uint32_t s_keys[];  // padded layout
  __shared__ uint32_t s_hist[kBins];           // this CTA's histogram of the current pass
  __shared__ uint32_t s_total[2][kBins];       // cluster totals (every CTA holds a copy)
  __shared__ uint32_t s_scan[33];
  __shared__ uint32_t s_sel[3];                // digit, count above, count in the digit's bin
  __shared__ uint32_t s_cnt[kMaxCluster][2];   // lower-ranked CTAs' (sure, tie) counts

  cg::cluster_group cluster = cg::this_cluster();
  const int CL = p.cluster;
  const int r = static_cast<int>(cluster.block_rank());
  const int q = (blockIdx.x / CL) / p.pt.batch;  // budget
  const int b = (blockIdx.x / CL) - q * p.pt.batch;
  const int tid = threadIdx.x;

  const int32_t start = p.pt.start[b];
  const int32_t n = p.pt.start[b + 1] - start;
  const int32_t ds = p.pt.doc_begin[b], de = p.pt.doc_end[b];
  const int32_t kk = p.k_keep[q][b];
  const int32_t n_doc = de - ds;
  const int32_t chunk = (n + CL - 1) / CL;
  const int32_t lo = min(n, r * chunk);
  const int32_t len = min(n, lo + chunk) - lo;
  // mode 0: no document token kept; 1: whole document kept; 2: select
  const int mode = kk == 0 ? 0 : (kk >= n_doc ? 1 : 2);

  for (int i = tid; i < kBins; i += kThreads) {
    s_hist[i] = 0;
    s_total[0][i] = 0;
    s_total[1][i] = 0;
  }
  __syncthreads();
  // this CTA's totals are zero: the others may add into them once the barrier
  // completes (its wait comes after the scores are loaded)
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  grid_dep_wait();  // the scores (and the gate's histograms) are complete
  grid_dep_launch();

  // The gate's first-pass histogram of this prompt, when it counted these
  // scores (the tag names them); the same decision in every CTA of the cluster.
  uint32_t* hist_b = p.hist ? p.hist + static_cast<size_t>(b) * kHistStride : nullptr;
  bool from_gate = false;
  if (!kKeys && hist_b && mode == 2) {
    const uint32_t* tag = hist_b + kBins;
    const uint64_t zp = reinterpret_cast<uint64_t>(p.z);
    from_gate = tag[0] == kHistMagic &&
                tag[1] == static_cast<uint32_t>(p.pt.start[p.pt.batch]) &&
                tag[2] == static_cast<uint32_t>(zp) && tag[3] == static_cast<uint32_t>(zp >> 32);
    if (from_gate)
      for (int i = tid; i < kBins; i += kThreads) s_hist[i] = __ldcg(hist_b + i);
  }
  // keys into shared memory; the first-pass histogram on the way when it is
  // counted here
  for (int i = tid; i < len; i += kThreads) {
    const uint32_t key =
        kKeys ? __ldg(p.keys + start + lo + i) : order_key(__ldg(p.z + start + lo + i));
    s_keys[padded(i)] = key;
    const int32_t pos = lo + i;
    if (!from_gate && mode == 2 && pos >= ds && pos < de) atomicAdd(&s_hist[key >> 21], 1u);
  }
  __syncthreads();

  uint32_t T = 0, need = 0;
  uint32_t hmask = 0xFFFFFFFFu;  // key bits the threshold T fixes
  uint32_t prefix = 0, k_rem = static_cast<uint32_t>(kk);
  int pass = 0;
  bool done = mode != 2;
  if (from_gate) {
    const uint32_t total = select_digit(s_hist, kBins, k_rem, s_scan, s_sel);  // clears s_hist
    if (total == static_cast<uint32_t>(n_doc)) {
      prefix = s_sel[0] << 21;
      k_rem -= s_sel[1];
      pass = 1;
      if (s_sel[2] == k_rem) {  // the boundary bin is kept whole
        hmask = 0xFFFFFFFFu << 21;
        done = true;
      }
    } else {
      // not the histogram of these scores after all: count the first pass here
      for (int i = tid; i < len; i += kThreads) {
        const int32_t pos = lo + i;
        if (pos >= ds && pos < de) atomicAdd(&s_hist[s_keys[padded(i)] >> 21], 1u);
      }
      __syncthreads();
    }
  }
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");  // every CTA's totals are zero

#pragma unroll 1
  for (; !done && pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nbits = pass == 2 ? 10 : 11;
    const uint32_t nb = 1u << nbits;
    if (pass > 0) {
      const uint32_t high_mask = 0xFFFFFFFFu << (shift + nbits);
      for (int i = tid; i < len; i += kThreads) {
        const int32_t pos = lo + i;
        if (pos < ds || pos >= de) continue;
        const uint32_t key = s_keys[padded(i)];
        if ((key & high_mask) == prefix) atomicAdd(&s_hist[(key >> shift) & (nb - 1)], 1u);
      }
      __syncthreads();
    }
    // non-zero local bins into every CTA's totals (one-way), local bins cleared
    uint32_t* buf = s_total[pass & 1];
    for (int i = tid; i < static_cast<int>(nb); i += kThreads) {
      const uint32_t c = s_hist[i];
      if (c) {
        for (int rr = 0; rr < CL; ++rr) atomicAdd(cluster.map_shared_rank(buf, rr) + i, c);
        s_hist[i] = 0;
      }
    }
    cluster.sync();  // every CTA holds the cluster's totals of this pass
    select_digit(buf, nb, k_rem, s_scan, s_sel);  // clears buf for pass + 2
    prefix |= s_sel[0] << shift;
    k_rem -= s_sel[1];
    if (s_sel[2] == k_rem) {
      // every key of the boundary bin is kept: the remaining low bits cannot
      // change the set, so stop here (the same decision in every CTA)
      hmask = 0xFFFFFFFFu << shift;
      break;
    }
  }
  if (mode == 2) {
    T = prefix;
    need = k_rem;  // how many keys whose fixed bits equal T to keep, lowest indices first
  }

  // ---- ordered compaction -------------------------------------------------
  // thread t owns keys [t*per, t*per + per) of the slice
  const int32_t per = (len + kThreads - 1) / kThreads;
  const int32_t tlo = min(len, tid * per), thi = min(len, tlo + per);
  uint32_t gt = 0, eq = 0;
  for (int32_t i = tlo; i < thi; ++i) {
    const int32_t pos = lo + i;
    const bool doc = pos >= ds && pos < de;
    const uint32_t key = s_keys[padded(i)];
    gt += (!doc || mode == 1 || (mode == 2 && (key & hmask) > T)) ? 1u : 0u;
    eq += (doc && mode == 2 && (key & hmask) == T) ? 1u : 0u;
  }
  // packed (ties << 16 | sure) fits: at most 45056 keys per CTA
  uint32_t tot = 0;
  const uint32_t before = block_excl_scan(gt | (eq << 16), s_scan, &tot);
  if (tid > r && tid < CL) {  // push this CTA's totals to the higher-ranked CTAs
    uint32_t* c = cluster.map_shared_rank(&s_cnt[0][0], tid);
    c[2 * r] = tot & 0xFFFFu;
    c[2 * r + 1] = tot >> 16;
  }
  cluster.sync();  // counts of every lower-ranked CTA are visible; no remote access after this
  uint32_t pgt = 0, peq = 0;
  for (int rr = 0; rr < r; ++rr) {
    pgt += s_cnt[rr][0];
    peq += s_cnt[rr][1];
  }
  const uint32_t gt_before = before & 0xFFFFu, eq_before = before >> 16;
  const uint32_t need_here = need > peq ? need - peq : 0u;  // ties still to take in this CTA
  uint32_t out_pos = pgt + min(peq, need) + gt_before + min(need_here, eq_before);
  uint32_t tie_rank = eq_before;  // ties before this thread inside the CTA
  int32_t* out = p.kept_idx[q] + p.kept_start[q][b];
  const uint32_t m_b = static_cast<uint32_t>(p.kept_start[q][b + 1] - p.kept_start[q][b]);
  for (int32_t i = tlo; i < thi; ++i) {
    const int32_t pos = lo + i;
    const bool doc = pos >= ds && pos < de;
    const uint32_t key = s_keys[padded(i)];
    bool keep = !doc || mode == 1 || (mode == 2 && (key & hmask) > T);
    if (doc && mode == 2 && (key & hmask) == T) {
      keep = tie_rank < need_here;
      ++tie_rank;
    }
    if (keep) {
      if (out_pos < m_b) out[out_pos] = start + pos;
      else atomicOr(p.status, kDevTopkOverflow);
      ++out_pos;
    }
  }
  if (p.cu_kept[q] && r == 0 && tid == 0) {
    p.cu_kept[q][b + 1] = p.kept_start[q][b + 1];
    if (b == 0) p.cu_kept[q][0] = 0;
  }
  // Leave the workspace zeroed for the next gate: every CTA of this cluster read
  // it before the barriers above; the last of the prompt's budget clusters to
  // get here (a counter in the tag) clears the bins and the tag, so they are
  // never reused.
  if (hist_b && r == 0) {
    __shared__ uint32_t s_last;
    if (tid == 0)
      s_last = atomicAdd(hist_b + kBins + 4, 1u) == static_cast<uint32_t>(p.n_budgets - 1);
    __syncthreads();
    if (s_last) {
      for (int i = tid; i < kBins; i += kThreads) hist_b[i] = 0;
      if (tid < 8) hist_b[kBins + tid] = 0;
    }
  }
}

}  // namespace

tg_status launch_topk(const float* z, const uint32_t* keys, const PromptTable* tables,
                      int n_budgets, int max_len, int32_t* const* kept_idx,
                      int32_t* const* cu_kept, uint32_t* hist, cudaStream_t st) {
  static thread_local TopkParams p;  // ~11 KB: kept off the stack
  memset(&p, 0, sizeof(p));
  p.pt = tables[0];
  for (int q = 0; q < n_budgets; ++q) {
    for (int b = 0; b < tables[q].batch; ++b) p.k_keep[q][b] = tables[q].k_keep[b];
    for (int b = 0; b <= tables[q].batch; ++b) p.kept_start[q][b] = tables[q].kept_start[b];
    p.kept_idx[q] = kept_idx[q];
    p.cu_kept[q] = cu_kept ? cu_kept[q] : nullptr;
  }
  p.z = z;
  p.keys = keys;
  p.hist = keys ? nullptr : hist;
  p.n_budgets = n_budgets;
  p.status = device_status_word();
  if (!p.status) return set_error(TG_ERR_CUDA, "device status word unavailable");
  const int cl = kMaxCluster;  // latency-bound: spread every prompt over 8 SMs
  const int slice = (max_len + cl - 1) / cl;
  if (slice > 45056)  // 8 CTAs x 45056 keys: the largest slice whose keys fit in shared memory
    return set_error(TG_ERR_UNSUPPORTED, "prompt of %d tokens is too long for top-K", max_len);
  p.cluster = cl;
  const size_t dyn = static_cast<size_t>(padded(slice > 0 ? slice : 1) + 1) * sizeof(uint32_t);
  auto kernel = keys ? topk_kernel<true> : topk_kernel<false>;
  tg_status r = cuda_check(
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(dyn)),
      "topk smem attribute");
  if (r != TG_OK) return r;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(n_budgets * tables[0].batch * cl));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = dyn;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see grid_dep_wait
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cuda_check(cudaLaunchKernelEx(&cfg, kernel, p), "topk launch");
}

}  // namespace tg
