// attend_fma.cuh -- single-KV-head attention over selected (CSA) or all
// (HCA) compressed entries plus the sliding window, on the CUDA cores.
//
// "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part V":
//  - "The skeleton, and what's kept": one key-value head shared by every
//    query head; each cached entry is both the key and the value;
//  - CSA bullet: each query attends to its selected entries; HCA bullet:
//    queries attend to all compressed entries densely;
//  - first of the "three details": every layer also attends to the last 128
//    tokens, under the same softmax.
//
// One query row per cluster of CS CTAs.  The query's key list is
//   [selected entries (CSA: the k slots of idx; HCA: entries 0..v-1)]
//   ++ [window tokens max(0,t-W+1) .. t]
// and CTA `rank` takes a contiguous range of it.  Each CTA runs a base-2
// online softmax per head over its keys in tiles of 32 (warp lane = key), so
// every warp owns a few heads with their running (max, sum, output) in
// registers.  The partial (max, sum, output) of all CTAs are merged through
// distributed shared memory in fixed rank order: the result does not depend
// on timing.  This kernel serves fp32 inputs (and bf16 head sizes the
// tensor-core kernel does not take).
#pragma once

#include <cooperative_groups.h>

#include <type_traits>

#include "common.cuh"
#include "rope.cuh"

namespace csa {

namespace cg = cooperative_groups;

constexpr int kAttThreads = 256;
constexpr int kAttWarps = kAttThreads / 32;
constexpr int kAttTile = 32;
constexpr int kAttMaxHeadsPerWarp = 16;  // H <= 128

struct AttendArgs {
  const void *q;
  const void *kv_c;
  const void *kv_tok;
  const int32_t *idx;  // nullptr: every visible entry (HCA)
  const int32_t *lens;
  const int32_t *q_pos;
  void *out;
  const float *sink;  // [H] per-head sink logits (scaled-logit units), or nullptr
  int n_tok, k, Tq, H, nc_max, m, window;
  int R;             // query rows B * Tq
  float scale_log2;  // softmax scale * log2(e)
  // QK-norm and partial RoPE fused around the attention (third of the three
  // details): qk_flags kNrNorm normalises each query head (q_gamma [d] or
  // nullptr, q_eps), kNrRotate turns the query's last rope_r dims by its
  // position t and the output's back by -t; 0: the query is used as given
  int qk_flags, rope_r;
  const void *q_gamma;
  float q_eps;
  double rope_log2_base;
  // FP8 cache entries (tensor-core kernel, d = 128): the first 64 dims as
  // E4M3 codes [B][nc_max][64] with one UE8M0 scale byte per entry
  // [B][nc_max], the last 64 dims in bf16 [B][nc_max][64]; nullptr: kv_c
  const uint8_t *kv_fp8;
  const uint8_t *kv_sc;
  const void *kv_rope;
};

// Round a float to the storage type T (what a staged query holds).
template <typename T>
__device__ __forceinline__ float round_as(float v) {
  if constexpr (std::is_same<T, float>::value) {
    return v;
  } else {
    return __bfloat162float(__float2bfloat16_rn(v));
  }
}

// A head's sink logit in the kernels' base-2 units (-inf: no sink).  "Anatomy
// of a Frontier Model", second of the three details: a learned per-head logit
// whose exponential joins the softmax denominator (it carries no value).
__device__ __forceinline__ float sink_log2(const AttendArgs &a, int h) {
  return a.sink ? __ldg(a.sink + h) * 1.4426950408889634f : -INFINITY;
}

template <int CS>
__device__ __forceinline__ void att_cluster_sync() {
  if constexpr (CS > 1) {
    cg::this_cluster().sync();
  } else {
    __syncthreads();
  }
}

template <int CS, typename P>
__device__ __forceinline__ P *att_peer(P *mine, int rank) {
  if constexpr (CS > 1) {
    return cg::this_cluster().map_shared_rank(mine, rank);
  } else {
    return mine;
  }
}

template <typename T, int D, int CS>
__global__ void __launch_bounds__(kAttThreads) k_attend_fma(AttendArgs a) {
  extern __shared__ float smem[];
  __shared__ float2 rot_cs[64];  // (cos, sin) of the query position's RoPE angles
  const int H = a.H;
  float *qs = smem;                                   // [H][D]; later the partial outputs
  float *kt = qs + (size_t)H * D;                     // [kAttTile][D + 1]
  float *pm = kt + kAttTile * (D + 1);                // [H] partial max (base 2)
  float *pl = pm + H;                                 // [H] partial sum
  int *kvalid = reinterpret_cast<int *>(pl + H);      // [kAttTile]

  const int rank = (CS > 1) ? (int)cg::this_cluster().block_rank() : 0;
  const int r = blockIdx.x / CS;  // clusters tile the grid along x
  const int b = r / a.Tq, tq = r % a.Tq;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const T *q = static_cast<const T *>(a.q);
  const T *kv_c = static_cast<const T *>(a.kv_c);
  const T *kv_tok = static_cast<const T *>(a.kv_tok);
  T *out = static_cast<T *>(a.out) + (size_t)r * H * D;

  pdl_wait();  // launched with programmatic serialisation: inputs may still be in flight
  pdl_launch_dependents();
  int t;
  bool ok = query_position(a.lens, a.q_pos, b, a.Tq, tq, t);
  int v = 0, w0 = 0, nwin = 0;
  if (ok) {
    v = (t + 1) / a.m;
    w0 = max(0, t - a.window + 1);
    nwin = t - w0 + 1;
    if (v > a.nc_max) {
      if (tid == 0 && rank == 0) raise_dev_err(kDevErrCache);
      ok = false;
    } else if (nwin > a.n_tok) {
      if (tid == 0 && rank == 0) raise_dev_err(kDevErrRing);
      ok = false;
    }
  }
  if (!ok) {  // uniform over the cluster: zero this CTA's share of the heads
    for (int u = tid; u < H * D; u += kAttThreads)
      if ((u / D) % CS == rank) store_f(out + u, 0.f);
    return;
  }

  const int nsel = a.idx ? a.k : v;
  const int L = nsel + nwin;
  const int per = (L + CS - 1) / CS;
  const int lo = min(L, rank * per), hi = min(L, lo + per);

  constexpr int V = Vec16<T>::N;
  const T *qrow = q + (size_t)r * H * D;
  for (int u = tid; u < H * D / V; u += kAttThreads) {
    float f[V];
    load16(qrow + (size_t)u * V, f);
#pragma unroll
    for (int j = 0; j < V; ++j) qs[u * V + j] = f[j];
  }
  if (a.qk_flags) {
    // QK-norm and partial RoPE of the staged query heads, one warp per head,
    // D / 32 consecutive dims per lane; the result is rounded to T as a
    // normalised, rotated query stored in T would be
    constexpr int E = D / 32;
    if ((a.qk_flags & kNrRotate) && tid < a.rope_r / 2)
      rot_cs[tid] = rope_cos_sin(t, rope_turns(tid, a.rope_r, a.rope_log2_base));
    __syncthreads();
    const int d0 = D - a.rope_r;
    const T *gq = static_cast<const T *>(a.q_gamma);
    for (int h = wid; h < H; h += kAttWarps) {
      float x[E];
#pragma unroll
      for (int e = 0; e < E; ++e) x[e] = qs[(size_t)h * D + lane * E + e];
      if (a.qk_flags & kNrNorm) {
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) ss = fmaf(x[e], x[e], ss);
        ss = warp_sum(ss);
        const float inv = 1.f / sqrtf(ss / (float)D + a.q_eps);
#pragma unroll
        for (int e = 0; e < E; ++e) x[e] = x[e] * inv * (gq ? to_f(gq[lane * E + e]) : 1.f);
      }
      if (a.qk_flags & kNrRotate) {
#pragma unroll
        for (int e = 0; e < E; e += 2) {
          const int i = lane * E + e;
          if (i >= d0) rope_turn(x[e], x[e + 1], rot_cs[(i - d0) >> 1], false);
        }
      }
#pragma unroll
      for (int e = 0; e < E; ++e) qs[(size_t)h * D + lane * E + e] = round_as<T>(x[e]);
    }
  }

  constexpr int EPL = D / 32;  // output elements per lane
  float o[kAttMaxHeadsPerWarp][EPL];
  float mrun[kAttMaxHeadsPerWarp], lrun[kAttMaxHeadsPerWarp];
#pragma unroll
  for (int j = 0; j < kAttMaxHeadsPerWarp; ++j) {
    mrun[j] = -INFINITY;
    lrun[j] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[j][e] = 0.f;
  }

  for (int p0 = lo; p0 < hi; p0 += kAttTile) {
    __syncthreads();  // previous tile consumed (and qs staged on the first pass)
    // gather up to 32 key rows
    for (int u = tid; u < kAttTile * (D / V); u += kAttThreads) {
      const int jr = u / (D / V), col = (u % (D / V)) * V;
      const int p = p0 + jr;
      const T *row = nullptr;
      if (p < hi) {
        if (p < nsel) {
          const int i = a.idx ? __ldg(a.idx + (size_t)r * a.k + p) : p;
          if (i >= 0 && i < v) row = kv_c + ((size_t)b * a.nc_max + i) * D;
        } else {
          const int s = w0 + (p - nsel);
          row = kv_tok + ((size_t)b * a.n_tok + (s % a.n_tok)) * D;
        }
      }
      if (col == 0) kvalid[jr] = row != nullptr;
      float f[V];
      if (row) {
        load16(row + col, f);
      } else {
#pragma unroll
        for (int j = 0; j < V; ++j) f[j] = 0.f;  // weight 0 must not meet stale NaNs
      }
#pragma unroll
      for (int j = 0; j < V; ++j) kt[jr * (D + 1) + col + j] = f[j];
    }
    __syncthreads();
    const bool valid = kvalid[lane] != 0;
#pragma unroll
    for (int j = 0; j < kAttMaxHeadsPerWarp; ++j) {
      const int h = wid + kAttWarps * j;
      if (h >= H) break;
      const float *qh = qs + (size_t)h * D;
      float dot = 0.f;
#pragma unroll 8
      for (int e = 0; e < D; ++e) dot = fmaf(qh[e], kt[lane * (D + 1) + e], dot);
      const float lg = valid ? dot * a.scale_log2 : -INFINITY;
      const float mnew = fmaxf(mrun[j], warp_max(lg));
      if (mnew == -INFINITY) continue;  // nothing valid yet for this head
      const float p = exp2f(lg - mnew);
      const float alpha = exp2f(mrun[j] - mnew);
      lrun[j] = lrun[j] * alpha + warp_sum(p);
      mrun[j] = mnew;
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[j][e] *= alpha;
#pragma unroll 8
      for (int jr = 0; jr < kAttTile; ++jr) {
        const float pj = __shfl_sync(0xffffffffu, p, jr);
#pragma unroll
        for (int e = 0; e < EPL; ++e) o[j][e] = fmaf(pj, kt[jr * (D + 1) + lane + 32 * e], o[j][e]);
      }
    }
  }

  // publish this CTA's partial (max, sum, output) per head
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kAttMaxHeadsPerWarp; ++j) {
    const int h = wid + kAttWarps * j;
    if (h >= H) break;
    if (lane == 0) {
      pm[h] = mrun[j];
      pl[h] = lrun[j];
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) qs[(size_t)h * D + lane + 32 * e] = o[j][e];
  }
  att_cluster_sync<CS>();
  // merge: this CTA finalises heads h with h % CS == rank, ranks in order
  const int nmine = (H - rank + CS - 1) / CS;
  for (int u = tid; u < nmine * D; u += kAttThreads) {
    const int h = rank + CS * (u / D), e = u % D;
    const float sk = sink_log2(a, h);
    float M = sk;
#pragma unroll
    for (int c = 0; c < CS; ++c) M = fmaxf(M, att_peer<CS>(pm, c)[h]);
    float Ls = sk == -INFINITY ? 0.f : exp2f(sk - M), Os = 0.f;
#pragma unroll
    for (int c = 0; c < CS; ++c) {
      const float mc = att_peer<CS>(pm, c)[h];
      if (mc == -INFINITY) continue;
      const float wgt = exp2f(mc - M);
      Ls = fmaf(att_peer<CS>(pl, c)[h], wgt, Ls);
      Os = fmaf(att_peer<CS>(qs, c)[(size_t)h * D + e], wgt, Os);
    }
    float val = Os / Ls;
    if (a.qk_flags & kNrRotate) {
      // turn the output back by the query's position: the pair partner of
      // dim e is dim e ^ 1, held by lane ^ 1 (D * nmine is a multiple of 64,
      // so every lane of the warp is in this iteration)
      const float other = __shfl_xor_sync(0xffffffffu, val, 1);
      const int d0 = D - a.rope_r;
      if (e >= d0) {
        float u0 = (e & 1) ? other : val, u1 = (e & 1) ? val : other;
        rope_turn(u0, u1, rot_cs[(e - d0) >> 1], true);
        val = (e & 1) ? u1 : u0;
      }
    }
    store_f(out + (size_t)h * D + e, val);
  }
  att_cluster_sync<CS>();  // peers may still be reading this CTA's partials
}

}  // namespace csa
