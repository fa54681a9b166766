// topk.cuh -- per-query top-k over indexer scores: radix select across a
// thread-block cluster, output in ascending index order.
//
// "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part V", CSA
// bullet: each query attends to only its k most relevant entries (1,024 in
// Pro, 512 in Flash).  The selected set is the k visible entries first in
// the order (score desc, index asc): ties go to the lower index; -0.0 ranks
// as +0.0; all visible entries when fewer than k.
//
// Design (one query row per cluster of CS CTAs, no global scratch, no spin
// waits):
//  1. each CTA loads its contiguous slice of the visible scores into shared
//     memory as order-preserving u32 keys (larger key = larger score);
//  2. four MSB-first 8-bit radix passes find the k-th largest key T: each CTA
//     histograms its slice (keys matching the prefix found so far), the
//     cluster barrier publishes the histograms, and every CTA sums all CS of
//     them through distributed shared memory in the same fixed order, so all
//     agree on the next digit without another exchange; a pass stops early
//     when the chosen bin holds exactly the keys still needed;
//  3. selection is then exact: keys above the threshold prefix are in; of
//     the keys equal to it, the lowest-index ones fill the rest.  Per-CTA
//     counts are exchanged once more and each CTA writes its selected indices
//     at fixed offsets, which yields the ascending-index output directly.
// Everything is integer work, so the result is bit-exact and independent of
// launch configuration.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace csa {

namespace cg = cooperative_groups;

constexpr int kTopkThreads = 512;
constexpr int kTopkSliceCap = 49152;  // keys per CTA held in shared memory
constexpr int kTopkMaxCluster = 8;

struct TopkShared {
  int hist[2][256];
  int scan[33];
  int digit_info[4];   // [0] chosen bin, [1] keys above it, [2] keys in it
  int cta_counts[2];   // this CTA's (greater, equal) counts, read by peers
};

template <int CS>
__device__ __forceinline__ void cluster_barrier() {
  if constexpr (CS > 1) {
    cg::this_cluster().sync();
  } else {
    __syncthreads();
  }
}

template <int CS>
__device__ __forceinline__ const TopkShared *peer(TopkShared *mine, int rank) {
  if constexpr (CS > 1) {
    return cg::this_cluster().map_shared_rank(mine, rank);
  } else {
    return mine;
  }
}

template <int CS>
__global__ void __launch_bounds__(kTopkThreads) k_topk(const float *__restrict__ scores,
                                                       const int32_t *__restrict__ lens,
                                                       const int32_t *__restrict__ q_pos, int Tq,
                                                       int nc_max, int k,
                                                       int32_t *__restrict__ idx_out) {
  extern __shared__ uint32_t keys[];  // [slice]
  __shared__ TopkShared sh;
  const int rank = (CS > 1) ? (int)cg::this_cluster().block_rank() : 0;
  const int r = blockIdx.x / CS;  // clusters tile the grid along x
  const int b = r / Tq, tq = r % Tq;
  const int tid = threadIdx.x;
  int32_t *orow = idx_out + (size_t)r * k;

  int t, v = 0;
  if (query_position(lens, q_pos, b, Tq, tq, t)) {
    v = (t + 1) / 4;
    if (v > nc_max) {
      if (tid == 0 && rank == 0) raise_dev_err(kDevErrCache);
      v = 0;
    }
  }

  // fewer visible entries than k: all of them, then -1 padding
  if (v <= k) {
    for (int j = rank * kTopkThreads + tid; j < k; j += CS * kTopkThreads) orow[j] = j < v ? j : -1;
    return;  // uniform across the cluster: no barrier was entered
  }

  const int per = (v + CS - 1) / CS;
  const int lo = min(v, rank * per), hi = min(v, lo + per);
  const int len = hi - lo;
  const float *srow = scores + (size_t)r * nc_max;
  for (int j = tid; j < len; j += kTopkThreads) keys[j] = order_key(__ldg(srow + lo + j));

  uint32_t pmask = 0u, pval = 0u;  // prefix of T found so far
  int need = k;                    // keys still needed among those matching the prefix
  bool all_eq = false;             // every key matching the prefix is selected
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    int *h = sh.hist[pass & 1];
    for (int j = tid; j < 256; j += kTopkThreads) h[j] = 0;
    __syncthreads();
    // warp-aggregated shared-memory histogram: scores crowd into few top
    // digits, so lanes with the same bin add once through their leader
    for (int j0 = 0; j0 < len; j0 += kTopkThreads) {
      const int j = j0 + tid;
      const uint32_t key = j < len ? keys[j] : 0u;
      const bool ok = j < len && (key & pmask) == pval;
      const unsigned act = __ballot_sync(0xffffffffu, ok);
      if (ok) {
        const uint32_t bin = (key >> shift) & 255u;
        const unsigned same = __match_any_sync(act, bin);
        if ((threadIdx.x & 31) == __ffs(same) - 1) atomicAdd(&h[bin], __popc(same));
      }
    }
    cluster_barrier<CS>();
    // bin totals over the cluster, in fixed rank order; thread j owns bin 255-j
    int cnt = 0;
    if (tid < 256) {
      const int bin = 255 - tid;
#pragma unroll
      for (int c = 0; c < CS; ++c) cnt += peer<CS>(&sh, c)->hist[pass & 1][bin];
    }
    int total;
    const int above = block_exclusive_scan(cnt, sh.scan, &total);  // keys in higher bins
    if (tid < 256 && above < need && above + cnt >= need) {
      sh.digit_info[0] = 255 - tid;
      sh.digit_info[1] = above;
      sh.digit_info[2] = cnt;
    }
    __syncthreads();
    const uint32_t bin = (uint32_t)sh.digit_info[0];
    need -= sh.digit_info[1];
    pmask |= 255u << shift;
    pval |= bin << shift;
    if (sh.digit_info[2] == need) {
      all_eq = true;
      break;
    }
  }

  // count this CTA's selected keys: greater than the prefix, and equal to it
  constexpr int NT = kTopkThreads;
  const int chunk = (len + NT - 1) / NT;
  const int c0 = min(len, tid * chunk), c1 = min(len, c0 + chunk);
  int n_gt = 0, n_eq = 0;
  for (int j = c0; j < c1; ++j) {
    const uint32_t km = keys[j] & pmask;
    n_gt += km > pval;
    n_eq += km == pval;
  }
  int cta_gt, cta_eq;
  const int gt_before = block_exclusive_scan(n_gt, sh.scan, &cta_gt);
  const int eq_before = block_exclusive_scan(n_eq, sh.scan, &cta_eq);
  if (tid == 0) {
    sh.cta_counts[0] = cta_gt;
    sh.cta_counts[1] = cta_eq;
  }
  cluster_barrier<CS>();
  // output offset of this CTA and the number of its equal keys to take
  int off = 0, eq_seen = 0, take_eq = 0;
#pragma unroll
  for (int c = 0; c < CS; ++c) {
    const TopkShared *p = peer<CS>(&sh, c);
    const int g = p->cta_counts[0], e = p->cta_counts[1];
    const int te = all_eq ? e : max(0, min(e, need - eq_seen));
    if (c < rank) off += g + te;
    if (c == rank) take_eq = te;
    eq_seen += e;
  }
  // per-thread: equal keys it takes, then its output position
  const int my_take = max(0, min(n_eq, take_eq - eq_before));
  int dummy;
  int pos = off + block_exclusive_scan(n_gt + my_take, sh.scan, &dummy);
  (void)gt_before;
  int eq_rank = eq_before;
  for (int j = c0; j < c1; ++j) {
    const uint32_t km = keys[j] & pmask;
    // (pos < k always holds: exactly k keys are selected; the guard keeps a
    // miscount from ever writing outside the row)
    if (km > pval) {
      if (pos < k) orow[pos] = lo + j;
      ++pos;
    } else if (km == pval) {
      if (eq_rank < take_eq) {
        if (pos < k) orow[pos] = lo + j;
        ++pos;
      }
      ++eq_rank;
    }
  }
  cluster_barrier<CS>();  // peers may still read this CTA's counts
}

}  // namespace csa
