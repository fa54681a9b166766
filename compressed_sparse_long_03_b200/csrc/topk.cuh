// topk.cuh -- per-query top-k over indexer scores, one query row per
// thread-block cluster, output in ascending index order.
//
// "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part V", CSA
// bullet: each query attends to only its k most relevant entries (1,024 in
// Pro, 512 in Flash).  The selected set is the k visible entries first in
// the order (score desc, index asc): ties go to the lower index; -0.0 ranks
// as +0.0; every visible entry when fewer than k.
//
// Design (cluster of CS CTAs per row; three cluster barriers; no spin waits):
//  A. each CTA loads a contiguous slice of the row's visible scores into
//     shared memory as order-preserving u32 keys and histograms them by their
//     12 leading bits (sign, exponent, 3 mantissa bits: monotone bins about
//     1/8 octave wide);                                         [barrier 1]
//  B. the cluster merges the histograms in two levels through distributed
//     shared memory -- 64 super-bins, then the 64 bins of the super-bin that
//     holds the k-th largest key -- giving that key's bin b* and the count
//     above it: every key outside b* is decided;
//  C. one pass over the slice marks the keys above b* in a bit mask (one
//     word per 32 keys) and collects the keys inside b* ("candidates", a few
//     hundred for real score distributions);                   [barrier 2]
//     every CTA then gathers all candidates of the cluster and resolves them
//     locally, identically: an 8-bit radix step on key bits 19..12 finds the
//     threshold sub-bin, and inside it candidates are ranked pairwise under
//     (score desc, index asc).  So every CTA knows how many keys each CTA of
//     the cluster selects;
//  D. the output offsets follow from those counts and from per-warp bit
//     counts, and each CTA writes its selected indices in ascending order
//     straight from the bit masks.                        [barrier 3: exit]
// When b* holds more candidates than fit (a degenerate distribution, e.g.
// all scores equal) an MSB-first radix select over the keys of b* with
// cluster-wide digit histograms takes over, ties resolved by index.
// All decisions are integer comparisons on the same keys in every CTA, so
// the result is bit-exact and independent of the launch configuration.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace csa {

namespace cg = cooperative_groups;

constexpr int kTopkThreads = 1024;
constexpr int kTopkSliceCap = 40960;   // keys per CTA held in shared memory
constexpr int kTopkMaxCluster = 8;     // portable; 16 where the device allows
constexpr int kTopkSuper = 64;         // super-bins of 64 score bins
constexpr int kTopkRankCap = 2048;     // candidates of a row resolved locally

struct TopkShared {
  int hist[kScoreBins];      // this CTA's score_bin histogram; later radix digits
  int super[kTopkSuper];     // this CTA's super-bin counts
  int scan[33];
  int info[4];               // [0] bin, [1] count above it, [2] count in it
  int ncand;                 // this CTA's candidates (keys in b*)
  int above;                 // this CTA's keys above b* (all of b* in mode 0)
  int cta_counts[2];         // legacy path: this CTA's (selected, tied) counts
  int peer_nc[16], peer_above[16], peer_sel[16];
  uint32_t all_key[kTopkRankCap];
  int all_idx[kTopkRankCap];
  unsigned char all_cta[kTopkRankCap];
};

// Dynamic shared memory of one CTA for slices of up to `per` keys: two bit
// masks over the slice (chosen candidates, keys above the threshold bin) and
// the largest bin of every 32-key group, then the keys (plus alignment
// slack), then the candidates (key and position).
__host__ __device__ constexpr size_t topk_mask_words(int per) { return ((size_t)per + 3 + 31) / 32; }
__host__ __device__ constexpr size_t topk_dyn_bytes(int per) {
  return 4ull * (((3 * topk_mask_words(per) + 3) & ~(size_t)3) + (size_t)per + 4 +
                 2 * (size_t)(per < kTopkRankCap ? per : kTopkRankCap));
}

template <int CS>
__device__ __forceinline__ void cluster_barrier() {
  if constexpr (CS > 1) {
    cg::this_cluster().sync();
  } else {
    __syncthreads();
  }
}

// The cluster barrier split in two: arrive once this CTA has finished
// reading its peers' shared memory, wait before leaving (so that no CTA
// exits while a peer may still read it).
template <int CS>
__device__ __forceinline__ void cluster_arrive_release() {
  if constexpr (CS > 1) asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
template <int CS>
__device__ __forceinline__ void cluster_wait_acquire() {
  if constexpr (CS > 1) asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int CS, typename P>
__device__ __forceinline__ P *peer_ptr(P *mine, int rank) {
  if constexpr (CS > 1) {
    return cg::this_cluster().map_shared_rank(mine, rank);
  } else {
    return mine;
  }
}

// Descending search over n <= blockDim buckets whose counts thread t
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

// idx_out row r: the k selected visible entries, ascending.  NT threads per
// CTA (1024 for long rows; 256 for short ones, so that several CTAs share an
// SM).
template <int CS, int NT = kTopkThreads>
__global__ void __launch_bounds__(NT) k_topk(const float *__restrict__ scores,
                                                       const int32_t *__restrict__ lens,
                                                       const int32_t *__restrict__ q_pos, int Tq,
                                                       int nc_max, int k,
                                                       int32_t *__restrict__ idx_out) {
  extern __shared__ uint32_t dyn[];
  __shared__ TopkShared sh;
  static_assert(NT >= 256 && kScoreBins % NT == 0, "256-bucket searches need 256 threads");
  constexpr int NW = NT / 32;
  const int rank = (CS > 1) ? (int)cg::this_cluster().block_rank() : 0;
  const int r = blockIdx.x / CS;  // clusters tile the grid along x
  const int b = r / Tq, tq = r % Tq;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  int32_t *orow = idx_out + (size_t)r * k;

  // layout for the largest slice (the same in every CTA of the cluster, so
  // peers find each other's candidates at the same offsets)
  const int per_max = (nc_max + CS - 1) / CS;
  const int nw_max = (int)topk_mask_words(per_max);
  const int ccap = per_max < kTopkRankCap ? per_max : kTopkRankCap;
  const int koff = (3 * nw_max + 3) & ~3;  // keys start 16-byte aligned
  uint32_t *selbits = dyn;                                         // chosen candidates
  uint32_t *abovebits = dyn + nw_max;                              // decided above b*
  uint32_t *gmaxbin = dyn + 2 * nw_max;                            // largest bin of a group
  uint32_t *cand_key = dyn + koff + per_max + 4;                   // [ccap]
  int *cand_pos = reinterpret_cast<int *>(cand_key + ccap);        // [ccap]

  // shared-memory set-up touches no global memory: before the wait
  for (int j = tid; j < kScoreBins; j += NT) sh.hist[j] = 0;
  if (tid < kTopkSuper) sh.super[tid] = 0;
  if (tid == 0) {
    sh.ncand = 0;
    sh.above = 0;
  }
  if (tid < 16) sh.peer_sel[tid] = 0;
  for (int j = tid; j < 3 * nw_max; j += NT) dyn[j] = 0u;  // both masks and group maxima
  __syncthreads();
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
  const float *srow = scores + (size_t)r * nc_max;
  // the slice start's misalignment to 16 B, mirrored in the key array so that
  // vector loads and vector stores line up.  Key j sits at position
  // P = j + p0 of the array; groups of 32 positions (one bit-mask word each)
  // never split a 16-byte vector.
  const int head0 = (int)((16 - (reinterpret_cast<uintptr_t>(srow + lo) & 15)) & 15) / 4;
  const int p0 = (4 - head0) & 3;
  const int ngroups = (p0 + len + 31) / 32;
  uint32_t *keys = dyn + koff + p0;  // [per], keys+head0 16 B aligned

  // ---- A: keys (16-byte vector loads, eight in flight per thread) and the
  // local histogram of their 12 leading bits
  {
    const float *src = srow + lo;
    const int head = min(head0, len);
    auto take = [&](int j, float f) {
      const uint32_t key = order_key(f);
      keys[j] = key;
      atomicAdd(&sh.hist[score_bin(key)], 1);
      atomicMax(&gmaxbin[(j + p0) >> 5], (uint32_t)score_bin(key));
    };
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
      // the lanes of a warp hold consecutive vectors; the 8 vectors of one
      // 32-position group form a run of lanes (cut at the warp's edges)
      const int r0 = (((head + p0) >> 2) + u0 + tid) & 7;  // this lane's place in its group
#pragma unroll
      for (int i = 0; i < UNR; ++i) {
        const int u = u0 + i * NT + tid;
        uint32_t gmax = 0;
        if (u < nvec) {
          const uint4 kv = make_uint4(order_key(f[i].x), order_key(f[i].y), order_key(f[i].z),
                                      order_key(f[i].w));
          vkeys[u] = kv;
          const int b0 = score_bin(kv.x), b1 = score_bin(kv.y), b2 = score_bin(kv.z),
                    b3 = score_bin(kv.w);
          atomicAdd(&sh.hist[b0], 1);
          atomicAdd(&sh.hist[b1], 1);
          atomicAdd(&sh.hist[b2], 1);
          atomicAdd(&sh.hist[b3], 1);
          gmax = (uint32_t)max(max(b0, b1), max(b2, b3));
        }
        // group maximum over the run (NT is a multiple of 8: r0 holds for every i)
        const int lo_l = max(0, lane - r0), hi_l = min(31, lane + 7 - r0);
        const unsigned seg = (hi_l == 31 ? 0xffffffffu : ((1u << (hi_l + 1)) - 1u)) & ~((1u << lo_l) - 1u);
        gmax = __reduce_max_sync(seg, gmax);
        if (lane == lo_l && u < nvec) atomicMax(&gmaxbin[(head + 4 * u + p0) >> 5], gmax);
      }
    }
    for (int j = head + 4 * nvec + tid; j < len; j += NT) take(j, __ldg(src + j));
  }
  __syncthreads();
  {
    constexpr int BPT = kScoreBins / NT;  // bins per thread
    int sum = 0;
#pragma unroll
    for (int i = 0; i < BPT; ++i) sum += sh.hist[BPT * tid + i];
    atomicAdd(&sh.super[(BPT * tid) / (kScoreBins / kTopkSuper)], sum);
  }

  // ---- B: merge over the cluster, in warp 0: the 64 super-bins summed over
  // the CTAs (two per lane, all loads in flight), the super-bin holding the
  // k-th largest key by a warp scan from the top, then its 64 bins likewise
  cluster_barrier<CS>();  // [1]
  static_assert(kTopkSuper == 64 && kScoreBins / kTopkSuper == 64, "two buckets per lane");
  if (wid == 0) {
    // descending: lane l holds buckets 63-2l (hi) and 62-2l (lo) of `arr`;
    // returns {bucket, count above it, count in it} for the need-th key
    auto pick = [&](const int *arr_mine, int need, int &bucket, int &above, int &cnt) {
      int ch = 0, cl = 0;
#pragma unroll
      for (int c = 0; c < CS; ++c) {
        const int *arr = peer_ptr<CS>(arr_mine, c);
        ch += arr[63 - 2 * lane];
        cl += arr[62 - 2 * lane];
      }
      int incl = ch + cl;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, incl >= need);
      const int f = __ffs(hit) - 1;  // hit != 0: the row holds more than k keys
      const int ex = __shfl_sync(0xffffffffu, incl - ch - cl, f);
      const int fch = __shfl_sync(0xffffffffu, ch, f), fcl = __shfl_sync(0xffffffffu, cl, f);
      if (ex + fch >= need) {
        bucket = 63 - 2 * f;
        above = ex;
        cnt = fch;
      } else {
        bucket = 62 - 2 * f;
        above = ex + fch;
        cnt = fcl;
      }
    };
    int sstar, above_s, cnt_s, bin, above_b, cnt_b;
    pick(sh.super, k, sstar, above_s, cnt_s);
    pick(sh.hist + 64 * sstar, k - above_s, bin, above_b, cnt_b);
    if (lane == 0) {
      sh.info[0] = 64 * sstar + bin;
      sh.info[1] = above_s + above_b;
      sh.info[2] = cnt_b;
    }
  }
  __syncthreads();
  const int bstar = sh.info[0];
  const int need = k - sh.info[1];  // keys to take from b*
  const int incand = sh.info[2];    // keys in b* over the whole row
  // keys of b*: mode 0 all selected; 1 resolved locally from the gathered
  // candidates; 2 the cluster-wide radix fallback
  const int mode = (incand == need) ? 0 : (incand <= kTopkRankCap ? 1 : 2);

  // warp w owns a contiguous run of 32-position groups [G0, G1); a group
  // whose largest bin is below b* holds nothing to select and is skipped
  const int gpw = (ngroups + NW - 1) / NW;
  const int G0 = min(ngroups, wid * gpw), G1 = min(ngroups, G0 + gpw);

  if (mode != 2) {
    // ---- C: decided keys into abovebits, candidates into the list
    int my_above = 0;
    for (int G = G0; G < G1; ++G) {
      if ((int)gmaxbin[G] < bstar) continue;  // warp-uniform
      const int j = 32 * G + lane - p0;
      const bool in = j >= 0 && j < len;
      const uint32_t key = in ? keys[j] : 0u;
      const int bn = in ? score_bin(key) : -1;
      const unsigned ma = __ballot_sync(0xffffffffu, mode == 0 ? bn >= bstar : bn > bstar);
      const unsigned mc = __ballot_sync(0xffffffffu, mode == 1 && bn == bstar);
      if (lane == 0) abovebits[G] = ma;
      my_above += __popc(ma);
      if (mc) {
        int base = 0;
        if (lane == 0) base = atomicAdd(&sh.ncand, __popc(mc));
        base = __shfl_sync(0xffffffffu, base, 0);
        if ((mc >> lane) & 1u) {
          const int u = base + __popc(mc & lt);
          cand_key[u] = key;
          cand_pos[u] = j;
        }
      }
    }
    if (lane == 0 && my_above) atomicAdd(&sh.above, my_above);
    cluster_barrier<CS>();  // [2]
    if (tid < CS) {
      const TopkShared *p = peer_ptr<CS>(&sh, tid);
      sh.peer_nc[tid] = p->ncand;
      sh.peer_above[tid] = p->above;
    }
    __syncthreads();
    if (mode == 1) {
      // ---- C1: gather all candidates of the cluster (all loads in flight)
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
        sh.all_cta[m] = (unsigned char)c;
      }
    }
    // no more reads of peers' shared memory by this CTA: [3] arrive
    cluster_arrive_release<CS>();
    if (mode == 1) {
      for (int j = tid; j < 256; j += NT) sh.hist[j] = 0;
      __syncthreads();
      // radix step on bits 19..12 of the candidates (all share bits 31..20)
      for (int m = tid; m < incand; m += NT) atomicAdd(&sh.hist[(sh.all_key[m] >> 12) & 255u], 1);
      __syncthreads();
      find_bucket(sh, 256, need, tid < 256 ? sh.hist[255 - tid] : 0);
      const uint32_t dstar = (uint32_t)sh.info[0];
      const int need2 = need - sh.info[1];  // to take from sub-bin d*
      const int nsub = sh.info[2];          // candidates in sub-bin d*
      // the members of d* in a short list (sh.hist as scratch)
      uint32_t *sub_key = reinterpret_cast<uint32_t *>(sh.hist);
      int *sub_idx = sh.hist + kTopkRankCap;
      if (tid == 0) sh.info[3] = 0;
      __syncthreads();
      for (int m = tid; m < incand; m += NT) {
        if (((sh.all_key[m] >> 12) & 255u) == dstar) {
          const int u = atomicAdd(&sh.info[3], 1);
          sub_key[u] = sh.all_key[m];
          sub_idx[u] = sh.all_idx[m];
        }
      }
      __syncthreads();
      // every candidate's fate: above d* in, below out, inside ranked
      // pairwise; own ones into selbits, and per-CTA counts
      for (int m = tid; m < incand; m += NT) {
        const uint32_t key = sh.all_key[m];
        const uint32_t d = (key >> 12) & 255u;
        bool sel = d > dstar;
        if (d == dstar) {
          const int gi = sh.all_idx[m];
          int beat = 0;
          for (int q = 0; q < nsub; ++q) {
            const uint32_t kq = sub_key[q];
            beat += (kq > key) || (kq == key && sub_idx[q] < gi);
          }
          sel = beat < need2;
        }
        if (sel) {
          const int c = sh.all_cta[m];
          atomicAdd(&sh.peer_sel[c], 1);
          if (c == rank) {
            const int P = sh.all_idx[m] - lo + p0;
            atomicOr(&selbits[P >> 5], 1u << (P & 31));
          }
        }
      }
      __syncthreads();
    }
    // ---- D: offsets from the counts, then the indices from the bit masks
    int off = 0;
#pragma unroll
    for (int c = 0; c < CS; ++c)
      if (c < rank) off += sh.peer_above[c] + sh.peer_sel[c];
    int n_sel = 0;  // this warp's selected keys
    for (int G = G0 + lane; G < G1; G += 32) n_sel += __popc(abovebits[G] | selbits[G]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n_sel += __shfl_xor_sync(0xffffffffu, n_sel, o);
    int cta_sel;
    const int before = block_exclusive_scan(lane == 0 ? n_sel : 0, sh.scan, &cta_sel);
    int pos = off + __shfl_sync(0xffffffffu, before, 0);
    for (int G = G0; G < G1; ++G) {
      const unsigned mall = abovebits[G] | selbits[G];
      if (mall == 0u) continue;  // warp-uniform
      if ((mall >> lane) & 1u) {
        const int p = pos + __popc(mall & lt);
        // (p < k always holds: exactly k keys are selected; the guard keeps a
        // miscount from ever writing outside the row)
        if (p < k) orow[p] = lo + 32 * G + lane - p0;
      }
      pos += __popc(mall);
    }
    cluster_wait_acquire<CS>();  // [3] wait: peers may still read this CTA's shared memory
    return;
  }

  // key-index chunks of 32 keys per warp for the fallback's passes
  const int cw = ((len + NW - 1) / NW + 31) & ~31;
  const int w0 = min(len, wid * cw), w1 = min(len, w0 + cw);
  // ---- fallback (mode 2): cluster-wide radix select among the keys of b*,
  // on bits 19..12, 11..4, 3..0, ties by index
  cluster_barrier<CS>();  // peers are done reading sh.hist
  int need_eq = need;
  uint32_t pmask = 0xFFF00000u, pval = (uint32_t)bstar << 20;
  bool all_eq = false;
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = 12 - 8 * pass;
    const int sh_ = shift < 0 ? 0 : shift;
    const uint32_t dmask = shift < 0 ? 15u : 255u;  // the last digit has 4 bits
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
#pragma unroll
      for (int c = 0; c < CS; ++c) c2 += peer_ptr<CS>(&sh, c)->hist[256 * (pass & 1) + 255 - tid];
    }
    find_bucket(sh, 256, need_eq, c2);
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
  // classify: 1 selected, 2 tied at the radix threshold, 0 not
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
  for (int g = w0; g < w1; g += 32) {
    const int j = g + lane;
    const int cl = j < w1 ? classify(j) : 0;
    n_sel += __popc(__ballot_sync(0xffffffffu, cl == 1));
    n_eq += __popc(__ballot_sync(0xffffffffu, cl == 2));
  }
  int cta_sel, cta_eq;
  const int sel_before = block_exclusive_scan(lane == 0 ? n_sel : 0, sh.scan, &cta_sel);
  const int eq_before = block_exclusive_scan(lane == 0 ? n_eq : 0, sh.scan, &cta_eq);
  if (tid == 0) {
    sh.cta_counts[0] = cta_sel;
    sh.cta_counts[1] = cta_eq;
  }
  cluster_barrier<CS>();
  if (tid < CS) {
    const TopkShared *p = peer_ptr<CS>(&sh, tid);
    sh.peer_above[tid] = p->cta_counts[0];
    sh.peer_nc[tid] = p->cta_counts[1];
  }
  __syncthreads();
  int off = 0, eq_seen = 0, take_eq = 0;
#pragma unroll
  for (int c = 0; c < CS; ++c) {
    const int g = sh.peer_above[c], e = sh.peer_nc[c];
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
    const int j = g + lane;
    const int cl = j < w1 ? classify(j) : 0;
    const unsigned ms = __ballot_sync(0xffffffffu, cl == 1);
    const unsigned me = __ballot_sync(0xffffffffu, cl == 2);
    // tied keys are taken in index order while eq_rank < take_eq
    const int te_here = max(0, min(__popc(me), take_eq - eq_rank));
    unsigned mt = me;  // keep the first te_here tied keys of this group
    for (int d = __popc(me) - te_here; d > 0; --d) mt &= ~(1u << (31 - __clz(mt)));
    const unsigned mall = ms | mt;
    eq_rank += __popc(me);
    if ((mall >> lane) & 1u) {
      const int p = pos + __popc(mall & lt);
      if (p < k) orow[p] = lo + j;
    }
    pos += __popc(mall);
  }
  cluster_barrier<CS>();  // peers may still read this CTA's shared memory
}

}  // namespace csa
