// index_score_fma.cuh -- lightning-indexer scores on the CUDA cores (fp32).
//
// "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part V", CSA
// bullet: a small indexer of HI heads x dI dims ranks the compressed blocks;
// "The Exchange Rates of a Million Tokens", section 3: ReLU-gated dot
// products.  I[t,i] = sum_h w[t,h] * max(0, qI[t,h,:] . kI[i,:]) for visible
// i < floor((t+1)/4); -inf for the rest of the row.
//
// This kernel serves fp32 inputs, whose scores must match an fp64 reference
// to ~1e-5 and so stay off the reduced-precision tensor-core formats.  One
// CTA scores 128 entries of one query row: the query's HI x dI block and the
// 128 keys are staged in shared memory as fp32, each thread owns one entry.
#pragma once

#include "common.cuh"

namespace csa {

constexpr int kIdxFmaTile = 128;

template <typename T, int DI>
__global__ void __launch_bounds__(kIdxFmaTile) k_index_score_fma(
    const T *__restrict__ qI, const T *__restrict__ w, const T *__restrict__ kI,
    const int32_t *__restrict__ lens, const int32_t *__restrict__ q_pos, int Tq, int HI,
    int nc_max, float *__restrict__ scores) {
  extern __shared__ float smem[];
  float *qs = smem;                        // [HI][DI]
  float *ws = qs + (size_t)HI * DI;        // [HI]
  float *ks = ws + ((HI + 3) & ~3);        // [kIdxFmaTile][DI + 1]
  const int r = blockIdx.y;                // query row b*Tq + tq
  const int b = r / Tq, tq = r % Tq;
  const int i0 = blockIdx.x * kIdxFmaTile;
  const int tid = threadIdx.x;
  float *srow = scores + (size_t)r * nc_max;

  int t;
  int vis = 0;
  if (query_position(lens, q_pos, b, Tq, tq, t)) {
    vis = (t + 1) / 4;
    if (vis > nc_max) {
      if (tid == 0 && blockIdx.x == 0) raise_dev_err(kDevErrCache);
      vis = 0;
    }
  }
  const int nvis = min(kIdxFmaTile, vis - i0);  // visible entries of this tile
  if (nvis <= 0) {
    if (i0 + tid < nc_max) srow[i0 + tid] = -INFINITY;
    return;
  }

  // stage the query block and the key tile
  constexpr int V = Vec16<T>::N;
  const T *qrow = qI + (size_t)r * HI * DI;
  for (int u = tid; u < HI * DI / V; u += kIdxFmaTile) {
    float f[V];
    load16(qrow + (size_t)u * V, f);
#pragma unroll
    for (int j = 0; j < V; ++j) qs[u * V + j] = f[j];
  }
  for (int h = tid; h < HI; h += kIdxFmaTile) ws[h] = to_f(w[(size_t)r * HI + h]);
  const T *ktile = kI + ((size_t)b * nc_max + i0) * DI;
  for (int u = tid; u < nvis * (DI / V); u += kIdxFmaTile) {
    const int row = u / (DI / V), col = (u % (DI / V)) * V;
    float f[V];
    load16(ktile + (size_t)row * DI + col, f);
#pragma unroll
    for (int j = 0; j < V; ++j) ks[row * (DI + 1) + col + j] = f[j];
  }
  __syncthreads();

  const int i = i0 + tid;
  if (tid < nvis) {
    float kr[DI];
#pragma unroll
    for (int e = 0; e < DI; ++e) kr[e] = ks[tid * (DI + 1) + e];
    float acc = 0.f;
    for (int h = 0; h < HI; ++h) {
      const float *qh = qs + h * DI;
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < DI; ++e) dot = fmaf(qh[e], kr[e], dot);
      acc = fmaf(ws[h], fmaxf(dot, 0.f), acc);
    }
    srow[i] = acc;
  } else if (i < nc_max) {
    srow[i] = -INFINITY;
  }
}

}  // namespace csa
