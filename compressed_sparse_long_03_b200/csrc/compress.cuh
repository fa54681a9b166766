// compress.cuh -- CSA (stride 4, 8-token overlapping windows) and HCA
// (stride m, no overlap) softmax-weighted per-channel compressors.
//
// "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part V",
// "The attention: compress, then select": CSA pools every 4 tokens into one
// entry with learned per-channel softmax weights and position biases over 8
// tokens (own block + the previous one); HCA pools every 128 tokens, no
// overlap.  "The Exchange Rates of a Million Tokens", section 3: the two
// overlapping series share one joint softmax.
//
// These CUDA-core kernels serve fp32 and d = 32 (bf16 with d in {64, 128}
// runs on the tensor cores, compress_tc.cuh); the pooling itself is per
// channel.
#pragma once

#include "common.cuh"

namespace csa {

// ---------------------------------------------------------------------------
// CSA: one CTA = kCsaEntries consecutive entries of one sequence, one thread
// per channel c.  Entry i pools tokens s = 4(i-1)+j, j = 0..7; slots j < 4
// use W_a, slots j >= 4 use W_b; logits z = x_s . W[:,c] + bias8[j][c]; tokens
// outside [0, lens[b]) are masked.
// ---------------------------------------------------------------------------
constexpr int kCsaEntries = 8;

template <typename T, int D>
__global__ void __launch_bounds__(D) k_csa_compress(const T *__restrict__ x,
                                                    const int32_t *__restrict__ lens, int n_max,
                                                    const T *__restrict__ Wa,
                                                    const T *__restrict__ Wb,
                                                    const T *__restrict__ bias8,
                                                    T *__restrict__ out, int nc_max) {
  constexpr int E = kCsaEntries;
  constexpr int NTOK = 4 * (E + 1);  // blocks i0-1 .. i0+E-1
  __shared__ float xs[NTOK][D];

  const int b = blockIdx.y;
  const int i0 = blockIdx.x * E;
  const int c = threadIdx.x;
  int n = __ldg(lens + b);
  if (n < 0 || n > n_max) {
    if (c == 0 && blockIdx.x == 0) raise_dev_err(kDevErrLen);
    n = 0;  // treat as empty: every row of this sequence is zero
  }
  const int nc = (n + 3) / 4;
  const long s0 = 4L * (i0 - 1);  // token of xs[0]

  // stage the tokens (fp32) in shared memory, zero outside the sequence
#pragma unroll
  for (int u = 0; u < NTOK; ++u) {
    const long s = s0 + u;
    float v = 0.f;
    if (s >= 0 && s < n) v = to_f(x[((size_t)b * n_max + s) * D + c]);
    xs[u][c] = v;
  }
  __syncthreads();

  // za[u]: token xs[u] as a previous-block member (series a),
  // zb[u]: token xs[u+4] as an own-block member (series b)
  float za[4 * E], zb[4 * E];
#pragma unroll
  for (int u = 0; u < 4 * E; ++u) za[u] = zb[u] = 0.f;
  // this thread's weight column, 16 inputs at a time with all loads in
  // flight (one round trip per block instead of one per input)
  for (int e0 = 0; e0 < D; e0 += 16) {
    float wa[16], wb[16];
#pragma unroll
    for (int ee = 0; ee < 16; ++ee) {
      wa[ee] = to_f(Wa[(size_t)(e0 + ee) * D + c]);
      wb[ee] = to_f(Wb[(size_t)(e0 + ee) * D + c]);
    }
#pragma unroll
    for (int ee = 0; ee < 16; ++ee) {
#pragma unroll
      for (int u = 0; u < 4 * E; ++u) {
        za[u] = fmaf(xs[u][e0 + ee], wa[ee], za[u]);
        zb[u] = fmaf(xs[u + 4][e0 + ee], wb[ee], zb[u]);
      }
    }
  }
  float bias[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) bias[j] = to_f(bias8[j * D + c]);

#pragma unroll
  for (int q = 0; q < E; ++q) {
    const int i = i0 + q;
    if (i >= nc_max) break;
    float res = 0.f;
    if (i < nc) {
      float z[8];
      bool ok[8];
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const long s = 4L * (i - 1) + j;
        ok[j] = (s >= 0 && s < n);
        z[j] = (j < 4 ? za[4 * q + j] : zb[4 * q + j - 4]) + bias[j];
        if (ok[j]) mx = fmaxf(mx, z[j]);
      }
      float den = 0.f, num = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (!ok[j]) continue;
        const float p = expf(z[j] - mx);
        den += p;
        num = fmaf(p, xs[4 * q + j][c], num);
      }
      res = num / den;
    }
    store_f(out + ((size_t)b * nc_max + i) * D + c, res);
  }
}

// ---------------------------------------------------------------------------
// HCA: one CTA = one entry (block of m tokens) of one sequence, one thread per
// channel; tokens streamed through shared memory in chunks of 32 with an
// online (running max) softmax.
// ---------------------------------------------------------------------------
constexpr int kHcaChunk = 32;

template <typename T, int D>
__global__ void __launch_bounds__(D) k_hca_compress(const T *__restrict__ x,
                                                    const int32_t *__restrict__ lens, int n_max,
                                                    int m, const T *__restrict__ W,
                                                    const T *__restrict__ bias,
                                                    T *__restrict__ out, int nc_max) {
  __shared__ float xs[kHcaChunk][D];
  const int b = blockIdx.y;
  const int i = blockIdx.x;
  const int c = threadIdx.x;
  int n = __ldg(lens + b);
  if (n < 0 || n > n_max) {
    if (c == 0 && i == 0) raise_dev_err(kDevErrLen);
    n = 0;
  }
  const long first = (long)m * i;
  long cnt = (long)n - first;
  if (cnt > m) cnt = m;
  float res = 0.f;
  if (cnt > 0) {
    float run_max = -INFINITY, den = 0.f, num = 0.f;
    for (long j0 = 0; j0 < cnt; j0 += kHcaChunk) {
      const int len = (int)((cnt - j0) < kHcaChunk ? (cnt - j0) : kHcaChunk);
      __syncthreads();
#pragma unroll
      for (int u = 0; u < kHcaChunk; ++u)
        xs[u][c] = (u < len) ? to_f(x[((size_t)b * n_max + first + j0 + u) * D + c]) : 0.f;
      __syncthreads();
      float z[kHcaChunk];
#pragma unroll
      for (int u = 0; u < kHcaChunk; ++u) z[u] = 0.f;
      for (int e0 = 0; e0 < D; e0 += 16) {
        float we[16];
#pragma unroll
        for (int ee = 0; ee < 16; ++ee) we[ee] = to_f(W[(size_t)(e0 + ee) * D + c]);
#pragma unroll
        for (int ee = 0; ee < 16; ++ee) {
#pragma unroll
          for (int u = 0; u < kHcaChunk; ++u) z[u] = fmaf(xs[u][e0 + ee], we[ee], z[u]);
        }
      }
      float cmax = -INFINITY;
#pragma unroll
      for (int u = 0; u < kHcaChunk; ++u) {
        if (u < len) {
          z[u] += to_f(bias[(size_t)(j0 + u) * D + c]);
          cmax = fmaxf(cmax, z[u]);
        }
      }
      const float new_max = fmaxf(run_max, cmax);
      const float alpha = expf(run_max - new_max);  // 0 on the first chunk
      den *= alpha;
      num *= alpha;
#pragma unroll
      for (int u = 0; u < kHcaChunk; ++u) {
        if (u < len) {
          const float p = expf(z[u] - new_max);
          den += p;
          num = fmaf(p, xs[u][c], num);
        }
      }
      run_max = new_max;
    }
    res = num / den;
  }
  if (i < nc_max) store_f(out + ((size_t)b * nc_max + i) * D + c, res);
}

}  // namespace csa
