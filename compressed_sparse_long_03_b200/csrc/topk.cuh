// topk.cuh -- per-query top-k over indexer scores, one query row per
// thread-block cluster, output in ascending index order.
//
// "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part V", CSA
// bullet: each query attends to only its k most relevant entries (1,024 in
// Pro, 512 in Flash).  The selected set is the k visible entries first in
// the order (score desc, index asc): ties go to the lower index; -0.0 ranks
// as +0.0; every visible entry when fewer than k.
//
// Design (cluster of CS CTAs per row; no spin waits):
//  A. each CTA loads a contiguous slice of the row's visible scores into
//     shared memory as order-preserving u32 keys and histograms them by their
//     12 leading bits (sign, exponent, 3 mantissa bits: monotone bins about
//     1/8 octave wide);
//  B. the cluster merges the histograms in two levels through distributed
//     shared memory -- 64 super-bins first, then the 64 bins of the super-bin
//     that holds the k-th largest key -- and finds that key's bin b* and the
//     count above it, which decide every key outside b*;
//  C. the keys inside b* ("candidates", a few hundred for real score
//     distributions) are ranked exactly: every CTA reads all candidates of
//     the cluster and, one warp per own candidate, counts the candidates
//     that beat it under (score desc, index asc).  When b* holds too many
//     keys for that (a degenerate distribution, e.g. all scores equal) an
//     MSB-first radix select over the remaining 20 key bits takes over,
//     ties resolved by index;
//  D. warp-contiguous 32-key groups: ballots give each selected key its slot,
//     per-warp and per-CTA counts (exchanged in the cluster) give the
//     offsets, and the indices come out in ascending order.
// All decisions are integer comparisons on the same keys in every CTA, so
// the result is bit-exact and independent of the launch configuration.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace csa {

namespace cg = cooperative_groups;

constexpr int kTopkThreads = 512;
constexpr int kTopkSliceCap = 40960;   // keys per CTA held in shared memory
constexpr int kTopkMaxCluster = 8;
constexpr int kTopkSuper = 64;         // super-bins of 64 score bins
constexpr int kTopkRankCap = 2048;     // candidates of a row ranked directly

struct TopkShared {
  int hist[kScoreBins];      // this CTA's score_bin histogram; later radix digits
  int super[kTopkSuper];     // this CTA's super-bin counts
  int scan[33];
  int info[4];               // [0] bin, [1] count above it, [2] count in it
  int ncand;                 // this CTA's candidates (keys in b*)
  int cta_counts[2];         // this CTA's (selected, tied) counts
  int peer_nc[16];           // candidates of each CTA of the cluster
  uint32_t all_key[kTopkRankCap];
  int all_idx[kTopkRankCap];
};

// Dynamic shared memory of one CTA for slices of up to `per` keys: the keys
// (plus alignment slack), the candidates (key and position) and two bit
// masks over the slice (keys above the threshold bin, chosen candidates).
__host__ __device__ constexpr size_t topk_dyn_bytes(int per) {
  return 4ull * ((size_t)per + 4 + 2 * (size_t)(per < kTopkRankCap ? per : kTopkRankCap) +
                 2 * (((size_t)per + 31) / 32));
}

template <int CS>
__device__ __forceinline__ void cluster_barrier() {
  if constexpr (CS > 1) {
    cg::this_cluster().sync();
  } else {
    __syncthreads();
  }
}

template <int CS, typename P>
__device__ __forceinline__ P *peer_ptr(P *mine, int rank) {
  if constexpr (CS > 1) {
    return cg::this_cluster().map_shared_rank(mine, rank);
  } else {
    return mine;
  }
}

// Descending search over n <= kTopkThreads buckets whose counts thread t
// supplies for bucket (n - 1 - t): the bucket holding the need-th largest
// key.  Writes sh.info = {bucket, count above it, count in it}.
__device__ __forceinline__ void find_bucket(TopkShared &sh, int n, int need, int cnt) {
  const int tid = threadIdx.x;
  int total;
  const int above = block_exclusive_scan(tid < n ? cnt : 0, sh.scan, &total);
  if (tid < n && above < need && above + cnt >= need) {
    sh.info[0] = n - 1 - tid;
    sh.info[1] = above;
    sh.info[2] = cnt;
  }
  __syncthreads();
}

// idx_out row r: the k selected visible entries, ascending.
template <int CS>
__global__ void __launch_bounds__(kTopkThreads) k_topk(const float *__restrict__ scores,
                                                       const int32_t *__restrict__ lens,
                                                       const int32_t *__restrict__ q_pos, int Tq,
                                                       int nc_max, int k,
                                                       int32_t *__restrict__ idx_out) {
  extern __shared__ uint32_t dyn[];
  __shared__ TopkShared sh;
  constexpr int NT = kTopkThreads;
  const int rank = (CS > 1) ? (int)cg::this_cluster().block_rank() : 0;
  const int r = blockIdx.x / CS;  // clusters tile the grid along x
  const int b = r / Tq, tq = r % Tq;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  int32_t *orow = idx_out + (size_t)r * k;
  pdl_wait();
  pdl_launch_dependents();

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
    for (int j = rank * NT + tid; j < k; j += CS * NT) orow[j] = j < v ? j : -1;
    return;  // uniform across the cluster: no barrier was entered
  }

  const int per = (v + CS - 1) / CS;  // the same in every CTA of the cluster
  const int lo = min(v, rank * per), hi = min(v, lo + per);
  const int len = hi - lo;
  const int ccap = per < kTopkRankCap ? per : kTopkRankCap;
  const int nwords = (per + 31) / 32;
  const float *srow = scores + (size_t)r * nc_max;
  // the slice start's misalignment to 16 B, mirrored in the key array so that
  // vector loads and vector stores line up
  const int head0 = (int)((16 - (reinterpret_cast<uintptr_t>(srow + lo) & 15)) & 15) / 4;
  uint32_t *keys = dyn + ((4 - head0) & 3);                     // [per], keys+head0 16 B aligned
  uint32_t *cand_key = dyn + per + 4;                           // [ccap]
  int *cand_pos = reinterpret_cast<int *>(dyn + per + 4 + ccap);  // [ccap]
  uint32_t *selbits = dyn + per + 4 + 2 * ccap;                 // [nwords] chosen candidates
  uint32_t *abovebits = selbits + nwords;                       // [nwords] keys above b*

  for (int j = tid; j < kScoreBins; j += NT) sh.hist[j] = 0;
  if (tid < kTopkSuper) sh.super[tid] = 0;
  if (tid == 0) sh.ncand = 0;
  __syncthreads();

  // ---- A: keys (16-byte vector loads, eight in flight per thread) and the
  // local histogram of their 12 leading bits
  auto take = [&](int j, float f) {
    const uint32_t key = order_key(f);
    keys[j] = key;
    atomicAdd(&sh.hist[score_bin(key)], 1);
  };
  {
    const float *src = srow + lo;
    const int head = min(head0, len);
    for (int j = tid; j < head; j += NT) take(j, __ldg(src + j));
    const int nvec = (len - head) / 4;
    const float4 *vsrc = reinterpret_cast<const float4 *>(src + head);
    uint4 *vkeys = reinterpret_cast<uint4 *>(keys + head);
    constexpr int UNR = 8;
    for (int u0 = 0; u0 < nvec; u0 += NT * UNR) {
      float4 f[UNR];
#pragma unroll
      for (int i = 0; i < UNR; ++i) {
        const int u = u0 + i * NT + tid;
        f[i] = u < nvec ? __ldg(vsrc + u) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int i = 0; i < UNR; ++i) {
        const int u = u0 + i * NT + tid;
        if (u < nvec) {
          const uint4 kv = make_uint4(order_key(f[i].x), order_key(f[i].y), order_key(f[i].z),
                                      order_key(f[i].w));
          vkeys[u] = kv;
          atomicAdd(&sh.hist[score_bin(kv.x)], 1);
          atomicAdd(&sh.hist[score_bin(kv.y)], 1);
          atomicAdd(&sh.hist[score_bin(kv.z)], 1);
          atomicAdd(&sh.hist[score_bin(kv.w)], 1);
        }
      }
    }
    for (int j = head + 4 * nvec + tid; j < len; j += NT) take(j, __ldg(src + j));
  }
  __syncthreads();
  {
    constexpr int BPT = kScoreBins / NT;  // bins per thread, one super-bin per 8 threads
    int sum = 0;
#pragma unroll
    for (int i = 0; i < BPT; ++i) sum += sh.hist[BPT * tid + i];
    atomicAdd(&sh.super[(BPT * tid) / (kScoreBins / kTopkSuper)], sum);
  }

  // ---- B: merge over the cluster: super-bins, then the bins of one
  cluster_barrier<CS>();
  {
    int c1 = 0;
    if (tid < kTopkSuper) {
#pragma unroll
      for (int c = 0; c < CS; ++c) c1 += peer_ptr<CS>(&sh, c)->super[kTopkSuper - 1 - tid];
    }
    find_bucket(sh, kTopkSuper, k, c1);
    const int sstar = sh.info[0], above_s = sh.info[1];
    __syncthreads();  // info is rewritten below
    constexpr int W = kScoreBins / kTopkSuper;
    int c2 = 0;
    if (tid < W) {
#pragma unroll
      for (int c = 0; c < CS; ++c) c2 += peer_ptr<CS>(&sh, c)->hist[W * sstar + W - 1 - tid];
    }
    find_bucket(sh, W, k - above_s, c2);
    if (tid == 0) {
      sh.info[0] += W * sstar;
      sh.info[1] += above_s;
    }
  }
  __syncthreads();
  const int bstar = sh.info[0];
  const int need = k - sh.info[1];  // keys to take from b*
  const int incand = sh.info[2];    // keys in b* over the whole row
  // keys of b*: mode 0 all selected, 1 selected where marked in selbits,
  // 2 by the radix threshold (pmask, pval) with ties by index
  const int mode = (incand == need) ? 0 : (incand <= kTopkRankCap ? 1 : 2);
  uint32_t pmask = 0u, pval = 0u;
  int need_eq = 0;
  bool all_eq = false;

  // warp w owns the contiguous chunk [w*cw, (w+1)*cw) of the slice, walked in
  // groups of 32 consecutive keys (group g = bit-mask word g)
  constexpr int NW = NT / 32;
  const int cw = ((len + NW - 1) / NW + 31) & ~31;
  const int w0 = min(len, wid * cw), w1 = min(len, w0 + cw);
  const unsigned lt = (1u << lane) - 1u;

  if (mode != 2) {
    // ---- C: one pass: keys above b* (and all of b* in mode 0) into
    // abovebits; in mode 1 the keys of b* into the candidate list
    for (int g = w0; g < w1; g += 32) {
      const int j = g + lane;
      const int bn = j < w1 ? score_bin(keys[j]) : -1;
      const unsigned ma = __ballot_sync(0xffffffffu, mode == 0 ? bn >= bstar : bn > bstar);
      const unsigned mc = __ballot_sync(0xffffffffu, mode == 1 && bn == bstar);
      if (lane == 0) {
        abovebits[g >> 5] = ma;
        selbits[g >> 5] = 0u;
      }
      if (mc) {
        int base = 0;
        if (lane == 0) base = atomicAdd(&sh.ncand, __popc(mc));
        base = __shfl_sync(0xffffffffu, base, 0);
        if ((mc >> lane) & 1u) {
          const int u = base + __popc(mc & lt);
          cand_key[u] = keys[j];
          cand_pos[u] = j;
        }
      }
    }
  }
  if (mode == 1) {
    // ---- C1: gather every candidate of the cluster, rank this CTA's own
    cluster_barrier<CS>();
    // every peer's candidate count in parallel, then all candidates at once
    if (tid < CS) sh.peer_nc[tid] = peer_ptr<CS>(&sh, tid)->ncand;
    __syncthreads();
    int coff[CS + 1];
    coff[0] = 0;
#pragma unroll
    for (int c = 0; c < CS; ++c) coff[c + 1] = coff[c] + sh.peer_nc[c];
    for (int m = tid; m < coff[CS]; m += NT) {
      int c = 0;
#pragma unroll
      for (int cc = 1; cc < CS; ++cc) c += m >= coff[cc];
      const int u = m - coff[c];
      sh.all_key[m] = peer_ptr<CS>(cand_key, c)[u];
      sh.all_idx[m] = min(v, c * per) + peer_ptr<CS>(cand_pos, c)[u];
    }
    __syncthreads();
    // one warp per own candidate, lanes over all candidates of the row
    for (int u = wid; u < sh.ncand; u += NT / 32) {
      const int pos = cand_pos[u];
      const uint32_t key = cand_key[u];
      const int gi = lo + pos;
      int beat = 0;
      for (int m = lane; m < incand; m += 32) {
        const uint32_t km = sh.all_key[m];
        beat += (km > key) || (km == key && sh.all_idx[m] < gi);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) beat += __shfl_xor_sync(0xffffffffu, beat, o);
      if (lane == 0 && beat < need) atomicOr(&selbits[pos >> 5], 1u << (pos & 31));
    }
    __syncthreads();
  } else if (mode == 2) {
    // ---- C2: radix select among the keys of b* (degenerate distributions)
    cluster_barrier<CS>();  // peers are done reading sh.hist
    need_eq = need;
    // the 12 leading bits are b*; digits of bits 19..12, 11..4, 3..0
    pmask = 0xFFF00000u;
    pval = (uint32_t)bstar << 20;
    const int shift0 = 12, npass = 3;
    for (int pass = 0; pass < npass; ++pass) {
      const int shift = shift0 - 8 * pass;
      const int sh_ = shift < 0 ? 0 : shift;
      const uint32_t dmask = shift < 0 ? 15u : 255u;  // the last fixed-bin digit has 4 bits
      int *h = sh.hist + 256 * (pass & 1);
      for (int j = tid; j < 256; j += NT) h[j] = 0;
      __syncthreads();
      for (int j0 = 0; j0 < len; j0 += NT) {
        const int j = j0 + tid;
        const uint32_t key = j < len ? keys[j] : 0u;
        const bool ok = j < len && (key & pmask) == pval;
        const unsigned act = __ballot_sync(0xffffffffu, ok);
        if (ok) {
          const uint32_t dg = (key >> sh_) & dmask;
          const unsigned same = __match_any_sync(act, dg);
          if (lane == __ffs(same) - 1) atomicAdd(&h[dg], __popc(same));
        }
      }
      cluster_barrier<CS>();
      int c2 = 0;
      if (tid < 256) {
        const int dg = 255 - tid;
#pragma unroll
        for (int c = 0; c < CS; ++c) c2 += peer_ptr<CS>(&sh, c)->hist[256 * (pass & 1) + dg];
      }
      int tot2;
      const int ab2 = block_exclusive_scan(c2, sh.scan, &tot2);
      if (tid < 256 && ab2 < need_eq && ab2 + c2 >= need_eq) {
        sh.info[0] = 255 - tid;
        sh.info[1] = ab2;
        sh.info[2] = c2;
      }
      __syncthreads();
      need_eq -= sh.info[1];
      pmask |= dmask << sh_;
      pval |= (uint32_t)sh.info[0] << sh_;
      const bool done = (sh.info[2] == need_eq);
      __syncthreads();  // info is read by every thread before the next pass rewrites it
      if (done) {
        all_eq = true;
        break;
      }
    }
  }

  // ---- D: count, exchange offsets, write in index order
  // classify (mode 2): 1 selected, 2 tied at the radix threshold, 0 not
  auto classify = [&](int j) -> int {
    const uint32_t key = keys[j];
    const int bn = score_bin(key);
    if (bn != bstar) return bn > bstar ? 1 : 0;
    const uint32_t km = key & pmask;
    if (km > pval) return 1;
    if (km == pval) return all_eq ? 1 : 2;
    return 0;
  };
  int n_sel = 0, n_eq = 0;  // warp totals (identical in every lane)
  if (mode != 2) {
    for (int g = w0; g < w1; g += 32) n_sel += __popc(abovebits[g >> 5] | selbits[g >> 5]);
  } else {
    for (int g = w0; g < w1; g += 32) {
      const int j = g + lane;
      const int cl = j < w1 ? classify(j) : 0;
      n_sel += __popc(__ballot_sync(0xffffffffu, cl == 1));
      n_eq += __popc(__ballot_sync(0xffffffffu, cl == 2));
    }
  }
  int cta_sel, cta_eq;
  const int sel_before = block_exclusive_scan(lane == 0 ? n_sel : 0, sh.scan, &cta_sel);
  const int eq_before = block_exclusive_scan(lane == 0 ? n_eq : 0, sh.scan, &cta_eq);
  if (tid == 0) {
    sh.cta_counts[0] = cta_sel;
    sh.cta_counts[1] = cta_eq;
  }
  cluster_barrier<CS>();
  int off = 0, eq_seen = 0, take_eq = 0;
#pragma unroll
  for (int c = 0; c < CS; ++c) {
    const TopkShared *p = peer_ptr<CS>(&sh, c);
    const int g = p->cta_counts[0], e = p->cta_counts[1];
    const int te = max(0, min(e, need_eq - eq_seen));
    if (c < rank) off += g + te;
    if (c == rank) take_eq = te;
    eq_seen += e;
  }
  // this warp's first output slot: selected keys of earlier warps, plus the
  // tied keys of earlier warps that are taken
  const int wsel = __shfl_sync(0xffffffffu, sel_before, 0);
  const int weq = __shfl_sync(0xffffffffu, eq_before, 0);
  int pos = off + wsel + max(0, min(weq, take_eq));
  int eq_rank = weq;
  for (int g = w0; g < w1; g += 32) {
    unsigned mall;
    if (mode != 2) {
      mall = abovebits[g >> 5] | selbits[g >> 5];
    } else {
      const int j = g + lane;
      const int cl = j < w1 ? classify(j) : 0;
      const unsigned ms = __ballot_sync(0xffffffffu, cl == 1);
      const unsigned me = __ballot_sync(0xffffffffu, cl == 2);
      // tied keys are taken in index order while eq_rank < take_eq
      const int te_here = max(0, min(__popc(me), take_eq - eq_rank));
      unsigned mt = me;  // keep the first te_here tied keys of this group
      for (int d = __popc(me) - te_here; d > 0; --d) mt &= ~(1u << (31 - __clz(mt)));
      mall = ms | mt;
      eq_rank += __popc(me);
    }
    if ((mall >> lane) & 1u) {
      const int p = pos + __popc(mall & lt);
      // (p < k always holds: exactly k keys are selected; the guard keeps a
      // miscount from ever writing outside the row)
      if (p < k) orow[p] = lo + g + lane;
    }
    pos += __popc(mall);
  }
  cluster_barrier<CS>();  // peers may still read this CTA's shared memory
}

}  // namespace csa
