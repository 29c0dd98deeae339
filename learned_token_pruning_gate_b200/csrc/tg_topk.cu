// Top-K over each prompt's document span with the question protected
// (TokenGate: "a top-K selector keeps the highest-scoring tokens"; "only the
// document part of the prompt is pruned, the question is never touched").
//
// One thread-block cluster of 8 CTAs handles one prompt in a single launch:
//  1. each CTA loads a contiguous 1/8 slice of the prompt's scores and caches
//     them in shared memory as order-preserving 32-bit keys;
//  2. three radix passes (11, 11, 10 bits) find the K-th largest key T: each CTA
//     builds a shared-memory histogram of the candidate digits with
//     warp-aggregated atomics (__match_any_sync), the cluster barrier publishes
//     it, and every CTA sums the 8 histograms over distributed shared memory and
//     picks the same digit, so no CTA waits on a flag;
//  3. an ordered compaction writes the kept rows in ascending order: protected
//     tokens and document keys > T are kept, and of the keys == T the first
//     (K - count(> T)) in index order, which makes ties go to the lower index.
// The only waits are hardware cluster barriers; no global scratch is used.
#include <cooperative_groups.h>

#include "tg_internal.cuh"

namespace cg = cooperative_groups;

namespace tg {
namespace {

constexpr int kCluster = 8;
constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;

struct TopkParams {
  PromptTable pt;
  const float* z;
  int32_t* kept_idx;
  int32_t* cu_kept;
  uint32_t* status;
};

// Order-preserving key: larger score -> larger key; -0.0 maps to +0.0; NaN maps
// to 0, below every number (-inf maps to 0x007FFFFF).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0u;
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive scan of one value per thread over the block (thread order).
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* s_warp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = s_warp[lane];
    uint32_t wx = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, wx, o);
      if (lane >= o) wx += y;
    }
    s_warp[lane] = wx - w;  // exclusive prefix of warp totals
    if (lane == 31) s_warp[32] = wx;
  }
  __syncthreads();
  uint32_t r = s_warp[warp] + x - v;
  if (total) *total = s_warp[32];
  __syncthreads();
  return r;
}

__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads, 1)
    topk_kernel(const __grid_constant__ TopkParams p) {
  extern __shared__ uint32_t s_keys[];
  __shared__ uint32_t s_hist[2][kBins];
  __shared__ uint32_t s_scan[33];
  __shared__ uint32_t s_sel[2];
  __shared__ uint32_t s_wgt[kWarps], s_weq[kWarps], s_wkept[kWarps];
  __shared__ uint32_t s_cnt[2];  // this CTA's (kept-for-sure, tie) counts, read by peers

  cg::cluster_group cluster = cg::this_cluster();
  const int r = static_cast<int>(cluster.block_rank());
  const int b = blockIdx.x / kCluster;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const int32_t start = p.pt.start[b];
  const int32_t n = p.pt.start[b + 1] - start;
  const int32_t ds = p.pt.doc_begin[b], de = p.pt.doc_end[b];
  const int32_t kk = p.pt.k_keep[b];
  const int32_t n_doc = de - ds;
  const int32_t chunk = (n + kCluster - 1) / kCluster;
  const int32_t lo = min(n, r * chunk);
  const int32_t len = min(n, lo + chunk) - lo;

  // mode 0: no document token kept; 1: whole document kept; 2: select
  const int mode = kk == 0 ? 0 : (kk >= n_doc ? 1 : 2);

  for (int i = tid; i < len; i += kThreads) s_keys[i] = order_key(__ldg(p.z + start + lo + i));
  __syncthreads();

  uint32_t T = 0, need = 0;
  if (mode == 2) {
    uint32_t prefix = 0, k_rem = static_cast<uint32_t>(kk);
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const int nbits = pass == 2 ? 10 : 11;
      const uint32_t nb = 1u << nbits;
      const uint32_t high_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + nbits));
      uint32_t* hist = s_hist[pass & 1];
      for (int i = tid; i < kBins; i += kThreads) hist[i] = 0;
      __syncthreads();
      for (int base = 0; base < len; base += kThreads) {
        const int i = base + tid;
        const int32_t pos = lo + i;
        const bool valid = i < len && pos >= ds && pos < de;
        const uint32_t key = valid ? s_keys[i] : 0u;
        const bool match = valid && (key & high_mask) == prefix;
        const uint32_t digit = (key >> shift) & (nb - 1);
        const unsigned m = __ballot_sync(0xffffffffu, match);
        if (match) {
          const unsigned peers = __match_any_sync(m, digit);
          if (lane == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
        }
      }
      cluster.sync();  // every CTA's histogram for this pass is complete and visible

      // Thread t owns bins [nb-1 - t*bpt - (bpt-1), nb-1 - t*bpt]: thread order is
      // descending digit order, so an exclusive scan counts the larger digits.
      const uint32_t bpt = nb / kThreads;  // 2 or 1
      uint32_t cnt[2] = {0, 0};
      for (uint32_t j = 0; j < bpt; ++j) {
        const uint32_t bin = nb - 1 - tid * bpt - j;
        uint32_t c = 0;
#pragma unroll
        for (int rr = 0; rr < kCluster; ++rr) c += cluster.map_shared_rank(hist, rr)[bin];
        cnt[j] = c;
      }
      const uint32_t mine = cnt[0] + cnt[1];
      uint32_t above = block_excl_scan(mine, s_scan, nullptr);
      if (above < k_rem && above + mine >= k_rem) {
        for (uint32_t j = 0; j < bpt; ++j) {
          if (above + cnt[j] >= k_rem) {
            s_sel[0] = nb - 1 - tid * bpt - j;
            s_sel[1] = above;
            break;
          }
          above += cnt[j];
        }
      }
      __syncthreads();
      prefix |= s_sel[0] << shift;
      k_rem -= s_sel[1];
      __syncthreads();
    }
    T = prefix;
    need = k_rem;  // how many keys == T to keep, lowest indices first
  }

  // ---- ordered compaction -------------------------------------------------
  // Warp w walks the contiguous range [w*W, min(len, (w+1)*W)) 32 elements at a
  // time; lane order inside a step is index order, so ballots give ranks.
  const int32_t W = ((len + kWarps * 32 - 1) / (kWarps * 32)) * 32;
  const int32_t wlo = min(len, warp * W), whi = min(len, wlo + W);
  const unsigned lt_mask = (1u << lane) - 1u;
  uint32_t wgt = 0, weq = 0;
  for (int32_t base = wlo; base < whi; base += 32) {
    const int32_t i = base + lane;
    const bool valid = i < whi;
    const int32_t pos = lo + i;
    const bool doc = valid && pos >= ds && pos < de;
    const uint32_t key = valid ? s_keys[i] : 0u;
    const bool gt = valid && (!doc || mode == 1 || (mode == 2 && key > T));
    const bool eq = doc && mode == 2 && key == T;
    wgt += __popc(__ballot_sync(0xffffffffu, gt));
    weq += __popc(__ballot_sync(0xffffffffu, eq));
  }
  if (lane == 0) {
    s_wgt[warp] = wgt;
    s_weq[warp] = weq;
  }
  __syncthreads();
  if (warp == 0) {
    // CTA totals for the peers
    uint32_t g = s_wgt[lane], e = s_weq[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      g += __shfl_xor_sync(0xffffffffu, g, o);
      e += __shfl_xor_sync(0xffffffffu, e, o);
    }
    if (lane == 0) {
      s_cnt[0] = g;
      s_cnt[1] = e;
    }
  }
  cluster.sync();  // counts of every CTA are visible
  if (warp == 0) {
    uint32_t pgt = 0, peq = 0;
    if (lane < r) {
      const uint32_t* rc = cluster.map_shared_rank(s_cnt, lane);
      pgt = rc[0];
      peq = rc[1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      pgt += __shfl_xor_sync(0xffffffffu, pgt, o);
      peq += __shfl_xor_sync(0xffffffffu, peq, o);
    }
    // per-warp tie and kept prefixes inside this CTA
    const uint32_t e = s_weq[lane];
    uint32_t ex = e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, ex, o);
      if (lane >= o) ex += y;
    }
    const uint32_t eq_before = peq + ex - e;  // ties before this warp's range
    const uint32_t taken = need > eq_before ? min(need - eq_before, e) : 0u;
    const uint32_t kept_w = s_wgt[lane] + taken;
    uint32_t kx = kept_w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, kx, o);
      if (lane >= o) kx += y;
    }
    const uint32_t cta_kept_before = pgt + min(peq, need);
    s_wkept[lane] = cta_kept_before + kx - kept_w;
    s_weq[lane] = eq_before;
  }
  __syncthreads();

  uint32_t run_eq = s_weq[warp], run_kept = s_wkept[warp];
  int32_t* out = p.kept_idx + p.pt.kept_start[b];
  const uint32_t m_b = static_cast<uint32_t>(p.pt.kept_start[b + 1] - p.pt.kept_start[b]);
  for (int32_t base = wlo; base < whi; base += 32) {
    const int32_t i = base + lane;
    const bool valid = i < whi;
    const int32_t pos = lo + i;
    const bool doc = valid && pos >= ds && pos < de;
    const uint32_t key = valid ? s_keys[i] : 0u;
    const bool gt = valid && (!doc || mode == 1 || (mode == 2 && key > T));
    const bool eq = doc && mode == 2 && key == T;
    const unsigned eqb = __ballot_sync(0xffffffffu, eq);
    const bool keep = gt || (eq && run_eq + __popc(eqb & lt_mask) < need);
    const unsigned kb = __ballot_sync(0xffffffffu, keep);
    if (keep) {
      const uint32_t slot = run_kept + __popc(kb & lt_mask);
      if (slot < m_b) out[slot] = start + pos;
      else atomicOr(p.status, kDevTopkOverflow);
    }
    run_eq += __popc(eqb);
    run_kept += __popc(kb);
  }

  if (p.cu_kept && r == 0 && tid == 0) {
    p.cu_kept[b + 1] = p.pt.kept_start[b + 1];
    if (b == 0) p.cu_kept[0] = 0;
  }
  cluster.sync();  // peers may still be reading this CTA's shared memory
}

}  // namespace

tg_status launch_topk(const float* z, const PromptTable& pt, int max_len, int32_t* kept_idx,
                      int32_t* cu_kept, cudaStream_t st) {
  TopkParams p;
  p.pt = pt;
  p.z = z;
  p.kept_idx = kept_idx;
  p.cu_kept = cu_kept;
  p.status = device_status_word();
  if (!p.status) return set_error(TG_ERR_CUDA, "device status word unavailable");
  const int slice = (max_len + kCluster - 1) / kCluster;
  const size_t dyn = static_cast<size_t>(slice > 0 ? slice : 1) * sizeof(uint32_t);
  tg_status r = cuda_check(
      cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(dyn)),
      "topk smem attribute");
  if (r != TG_OK) return r;
  topk_kernel<<<pt.batch * kCluster, kThreads, dyn, st>>>(p);
  return cuda_check(cudaGetLastError(), "topk launch");
}

}  // namespace tg
