// common.cuh -- small device helpers shared by the CSA/HCA kernels.
//
// The library is built as one translation unit (csa_api.cu includes every
// kernel header), so the device error word below has a single definition.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace csa {

// ---------------------------------------------------------------------------
// device error word: kernels record the first invalid length / position they
// meet (first writer wins); csa_check_device_error() reads and clears it.
// ---------------------------------------------------------------------------
enum DevErr : int {
  kDevErrNone = 0,
  kDevErrPos = 1,    // a query position outside [0, lens[b])
  kDevErrLen = 2,    // lens[b] < 0 or > n_max
  kDevErrCache = 3,  // visible entries exceed the cache rows
  kDevErrRing = 4,   // a query's window does not fit the token ring
  kDevErrTimeout = 5,  // a tensor-core pipeline wait passed its time limit
};

__device__ int g_dev_err;

__device__ __forceinline__ void raise_dev_err(int code) { atomicCAS(&g_dev_err, 0, code); }

// ---------------------------------------------------------------------------
// programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while its predecessor in the stream is finishing.
// It waits for the predecessor's completion (and memory) before touching
// global memory, and lets its own dependents launch once all its CTAs run.
// Both are no-ops for a kernel launched without the attribute.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// element conversion
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void store_f(float *p, float v) { *p = v; }
__device__ __forceinline__ void store_f(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

// Elements per 16-byte vector.
template <typename T>
struct Vec16 {
  static constexpr int N = 16 / sizeof(T);
};

// Load 16 bytes (4 floats or 8 bf16) at p (16-byte aligned) as floats.
__device__ __forceinline__ void load16(const float *p, float *f) {
  float4 v = __ldg(reinterpret_cast<const float4 *>(p));
  f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
__device__ __forceinline__ void load16(const __nv_bfloat16 *p, float *f) {
  uint4 v = __ldg(reinterpret_cast<const uint4 *>(p));
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// ---------------------------------------------------------------------------
// query position and visibility
// ---------------------------------------------------------------------------
// Position of query (b, tq): q_pos[b][tq], or lens[b] - Tq + tq when q_pos is
// NULL.  Returns false (and records the error) when outside [0, lens[b]).
__device__ __forceinline__ bool query_position(const int32_t *lens, const int32_t *q_pos, int b,
                                               int Tq, int tq, int &t) {
  const int n = __ldg(lens + b);
  t = q_pos ? __ldg(q_pos + (size_t)b * Tq + tq) : n - Tq + tq;
  if (t < 0 || t >= n) {
    raise_dev_err(kDevErrPos);
    return false;
  }
  return true;
}

// ---------------------------------------------------------------------------
// order-preserving 32-bit key of an fp32 score: larger score -> larger key;
// -0.0 is folded onto +0.0 so that the two tie.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Histogram bin of a score for the top-k threshold search: the 12 leading
// bits of its order key (sign, exponent, 3 mantissa bits), so bins are
// monotone in the score and about 1/8 octave wide.
constexpr int kScoreBins = 4096;
__device__ __forceinline__ int score_bin(uint32_t key) { return (int)(key >> 20); }

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Exclusive block-wide prefix sum of one int per thread (blockDim.x a
// multiple of 32, at most 1024).  `scratch` holds >= 33 ints.  Returns the
// exclusive prefix; *total receives the block sum.  Contains __syncthreads.
__device__ __forceinline__ int block_exclusive_scan(int v, int *scratch, int *total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int s = lane < nw ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < nw) scratch[lane] = s;  // inclusive warp totals
    if (lane == 31) scratch[32] = s;
  }
  __syncthreads();
  const int base = wid > 0 ? scratch[wid - 1] : 0;
  const int res = base + x - v;
  *total = scratch[32];
  __syncthreads();
  return res;
}

}  // namespace csa
