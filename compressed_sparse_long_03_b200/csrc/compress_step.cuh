// compress_step.cuh -- the decode-time compressors: one new entry per
// sequence, from the token ring the decode step keeps, when the newest token
// completes a block.
//
// "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part V", "The
// attention: compress, then select" and the first of its three details: a
// compressed entry is formed only once its block is complete; until then the
// block's tokens are reached through the sliding window.  So at decode the
// caches grow by one entry whenever lens[b] reaches a multiple of the stride:
// CSA entry i = lens/4 - 1 pools blocks i-1 and i (tokens 4i-4 .. 4i+3), HCA
// entry i = lens/m - 1 pools tokens m*i .. m*i+m-1 -- the same pooling as the
// full compressors (compress.cuh), restricted to that entry.  The tokens come
// from the ring (token s at row s % n_tok), so the ring is the compressor's
// whole state: no partial-block accumulator is kept.
//
// One CTA per sequence, one thread per channel (CUDA cores: one entry per
// sequence is d x d x 8 (CSA) or d x d x m (HCA) multiply-adds).  The
// weights pass through shared memory in blocks of 32 input channels (one
// load round trip per block, not one per input channel).
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace csa {

namespace cg = cooperative_groups;
constexpr int kStepWRows = 32;

template <typename T, int D>
__global__ void __launch_bounds__(D) k_csa_compress_step(const T *__restrict__ tok, int n_tok,
                                                         const int32_t *__restrict__ lens,
                                                         const T *__restrict__ Wa,
                                                         const T *__restrict__ Wb,
                                                         const T *__restrict__ bias8,
                                                         T *__restrict__ cache, int nc_max) {
  __shared__ float xs[8][D];
  __shared__ float sWa[kStepWRows][D], sWb[kStepWRows][D];
  const int b = blockIdx.x, c = threadIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  const int n = __ldg(lens + b);
  if (n <= 0 || (n & 3)) return;  // no block completes with this token
  const int i = n / 4 - 1;
  if (i >= nc_max) {
    if (c == 0) raise_dev_err(kDevErrCache);
    return;
  }
  if (min(8, n) > n_tok) {  // the ring must hold both blocks
    if (c == 0) raise_dev_err(kDevErrRing);
    return;
  }
  const long s0 = 4L * (i - 1);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const long s = s0 + j;
    xs[j][c] = s >= 0 ? to_f(tok[((size_t)b * n_tok + (size_t)(s % n_tok)) * D + c]) : 0.f;
  }
  __syncthreads();
  float z[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) z[j] = to_f(bias8[j * D + c]);
  static_assert(D % kStepWRows == 0, "whole weight blocks");
  for (int e0 = 0; e0 < D; e0 += kStepWRows) {
    // all loads of the block in flight before the first store
    float wa_r[kStepWRows], wb_r[kStepWRows];
#pragma unroll
    for (int ee = 0; ee < kStepWRows; ++ee) {
      wa_r[ee] = to_f(Wa[(size_t)(e0 + ee) * D + c]);
      wb_r[ee] = to_f(Wb[(size_t)(e0 + ee) * D + c]);
    }
#pragma unroll
    for (int ee = 0; ee < kStepWRows; ++ee) {
      sWa[ee][c] = wa_r[ee];
      sWb[ee][c] = wb_r[ee];
    }
    __syncthreads();
    for (int ee = 0; ee < kStepWRows; ++ee) {
      const float wa = sWa[ee][c], wb = sWb[ee][c];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        z[j] = fmaf(xs[j][e0 + ee], wa, z[j]);
        z[j + 4] = fmaf(xs[j + 4][e0 + ee], wb, z[j + 4]);
      }
    }
    __syncthreads();
  }
  const int j0 = i == 0 ? 4 : 0;  // entry 0 has no previous block
  float mx = -INFINITY;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j >= j0) mx = fmaxf(mx, z[j]);
  float den = 0.f, num = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < j0) continue;
    const float p = expf(z[j] - mx);
    den += p;
    num = fmaf(p, xs[j][c], num);
  }
  store_f(cache + ((size_t)b * nc_max + i) * D + c, num / den);
}

constexpr int kStepChunk = 32;
constexpr int kStepCluster = 8;  // CTAs sharing one HCA entry

// HCA: a cluster of kStepCluster CTAs per sequence; CTA `rank` folds the
// entry's tokens [rank*per, rank*per + per) into a per-channel (max, sum,
// pooled sum) and CTA 0 merges the eight partials through distributed shared
// memory, in rank order.
template <typename T, int D>
__global__ void __launch_bounds__(D) k_hca_compress_step(const T *__restrict__ tok, int n_tok,
                                                         const int32_t *__restrict__ lens, int m,
                                                         const T *__restrict__ W,
                                                         const T *__restrict__ bias,
                                                         T *__restrict__ cache, int nc_max) {
  __shared__ float xs[kStepChunk][D];
  __shared__ float sW[kStepWRows][D];
  __shared__ float part[3][D];  // this CTA's (max, sum, pooled sum) per channel
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int b = blockIdx.x / kStepCluster, c = threadIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  const int n = __ldg(lens + b);
  // uniform over the cluster: every CTA of the sequence takes the same exits
  if (n <= 0 || n % m) return;  // no block completes with this token
  const int i = n / m - 1;
  if (i >= nc_max || m > n_tok) {
    if (c == 0 && rank == 0) raise_dev_err(i >= nc_max ? kDevErrCache : kDevErrRing);
    return;
  }
  const int per = (m + kStepCluster - 1) / kStepCluster;
  const int t0 = min(m, rank * per), t1 = min(m, t0 + per);
  const long first = (long)m * i;
  float run_max = -INFINITY, den = 0.f, num = 0.f;
  for (int j0 = t0; j0 < t1; j0 += kStepChunk) {
    const int len = min(kStepChunk, t1 - j0);
    __syncthreads();
    {
      float xr[kStepChunk];
#pragma unroll
      for (int u = 0; u < kStepChunk; ++u)
        xr[u] = u < len ? to_f(tok[((size_t)b * n_tok + (size_t)((first + j0 + u) % n_tok)) * D + c]) : 0.f;
#pragma unroll
      for (int u = 0; u < kStepChunk; ++u) xs[u][c] = xr[u];
    }
    __syncthreads();
    float z[kStepChunk];
#pragma unroll
    for (int u = 0; u < kStepChunk; ++u) z[u] = 0.f;
    static_assert(D % kStepWRows == 0, "whole weight blocks");
    for (int e0 = 0; e0 < D; e0 += kStepWRows) {
      float wr[kStepWRows];
#pragma unroll
      for (int ee = 0; ee < kStepWRows; ++ee) wr[ee] = to_f(W[(size_t)(e0 + ee) * D + c]);
      __syncthreads();
#pragma unroll
      for (int ee = 0; ee < kStepWRows; ++ee) sW[ee][c] = wr[ee];
      __syncthreads();
      for (int ee = 0; ee < kStepWRows; ++ee) {
        const float we = sW[ee][c];
#pragma unroll
        for (int u = 0; u < kStepChunk; ++u)
          if (u < len) z[u] = fmaf(xs[u][e0 + ee], we, z[u]);
      }
    }
    float cmax = -INFINITY;
#pragma unroll
    for (int u = 0; u < kStepChunk; ++u) {
      if (u < len) {
        z[u] += to_f(bias[(size_t)(j0 + u) * D + c]);
        cmax = fmaxf(cmax, z[u]);
      }
    }
    const float nmax = fmaxf(run_max, cmax);
    const float alpha = expf(run_max - nmax);  // 0 on the first chunk
    den *= alpha;
    num *= alpha;
#pragma unroll
    for (int u = 0; u < kStepChunk; ++u) {
      if (u < len) {
        const float p = expf(z[u] - nmax);
        den += p;
        num = fmaf(p, xs[u][c], num);
      }
    }
    run_max = nmax;
  }
  part[0][c] = run_max;
  part[1][c] = den;
  part[2][c] = num;
  cluster.sync();
  if (rank == 0) {
    float M = -INFINITY;
#pragma unroll
    for (int r = 0; r < kStepCluster; ++r) M = fmaxf(M, cluster.map_shared_rank(&part[0][0], r)[c]);
    float Ds = 0.f, Ns = 0.f;
#pragma unroll
    for (int r = 0; r < kStepCluster; ++r) {
      const float mr = cluster.map_shared_rank(&part[0][0], r)[c];
      if (mr == -INFINITY) continue;  // a CTA without tokens
      const float w = expf(mr - M);
      Ds = fmaf(cluster.map_shared_rank(&part[1][0], r)[c], w, Ds);
      Ns = fmaf(cluster.map_shared_rank(&part[2][0], r)[c], w, Ns);
    }
    store_f(cache + ((size_t)b * nc_max + i) * D + c, Ns / Ds);
  }
  cluster.sync();  // CTA 0 has read every peer's partials
}

}  // namespace csa
