// fp8.cuh -- FP8 cache entries: the quantiser, and the E4M3 widening the
// attention's gather uses.
//
// "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part V", "The
// KV cache, recomputed": an entry keeps its 64 RoPE dims in BF16 and the
// rest in FP8 with one-byte UE8M0 scales (448 numbers, 7 scales: one per 64).
// Format read as E4M3 codes with, per 64-element block, the power-of-two
// scale 2^X, X = floor(log2 amax) - 8 (8 is the exponent of E4M3's largest
// finite value, 448), clamped to [-127, 127] and stored as X + 127 (-127 for
// an all-zero block); each element is x / 2^X rounded to the nearest E4M3
// value, ties to even, saturating at 448.  Planes: codes [rows][d - r],
// scales [rows][(d - r) / 64], the last r dims [rows][r] unchanged.
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace csa {

constexpr int kF8Threads = 256;

// One warp per entry: the blocks of 64 FP8 elements (two per lane: amax by a
// warp reduction, the scale from the exponent, the hardware round-to-nearest-
// even, saturating conversion), then the copy of the rotated dims.
template <typename T>
__global__ void __launch_bounds__(kF8Threads) k_quantize_fp8_entries(const T *__restrict__ x, long rows, int d,
                                                                     int r, uint8_t *__restrict__ fp8,
                                                                     uint8_t *__restrict__ sc,
                                                                     T *__restrict__ rope) {
  const int lane = threadIdx.x & 31;
  const long nw = (long)gridDim.x * (kF8Threads / 32);
  const int q = d - r;
  pdl_wait();
  pdl_launch_dependents();
  for (long row = (long)blockIdx.x * (kF8Threads / 32) + (threadIdx.x >> 5); row < rows; row += nw) {
    const T *xr = x + (size_t)row * d;
    for (int blk = 0; blk < q / 64; ++blk) {
      const float v0 = to_f(xr[blk * 64 + 2 * lane]), v1 = to_f(xr[blk * 64 + 2 * lane + 1]);
      const float amax = warp_max(fmaxf(fabsf(v0), fabsf(v1)));
      int X = amax > 0.f ? ilogbf(amax) - 8 : -127;
      X = max(-127, min(127, X));
      const __nv_fp8_storage_t c0 = __nv_cvt_float_to_fp8(ldexpf(v0, -X), __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8_storage_t c1 = __nv_cvt_float_to_fp8(ldexpf(v1, -X), __NV_SATFINITE, __NV_E4M3);
      *reinterpret_cast<uint16_t *>(fp8 + (size_t)row * q + blk * 64 + 2 * lane) =
          (uint16_t)((uint32_t)c0 | ((uint32_t)c1 << 8));
      if (lane == 0) sc[(size_t)row * (q / 64) + blk] = (uint8_t)(X + 127);
    }
    for (int e = lane; e < r; e += 32) rope[(size_t)row * r + e] = xr[q + e];
  }
}

// 2^X as a float for X in [-127, 127] (2^-127 is subnormal).
__device__ __forceinline__ float f8_pow2(int X) {
  return X >= -126 ? __uint_as_float((uint32_t)(X + 127) << 23) : __uint_as_float(0x00400000u);
}

// Eight E4M3 codes (the bytes of lo, hi in order) times 2^X as eight bf16
// values packed in four words (element 2i in the low half of word i).  Each
// code widens exactly to fp16, the product by a power of two is exact in
// fp32 and, having at most 4 significant bits, in bf16.
__device__ __forceinline__ void f8_widen8(uint32_t lo, uint32_t hi, float s, uint32_t *w) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t word = i < 2 ? lo : hi;
    const int sh = (i & 1) * 16;
    const __half_raw h0 = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)((word >> sh) & 0xFF), __NV_E4M3);
    const __half_raw h1 = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)((word >> (sh + 8)) & 0xFF), __NV_E4M3);
    const float f0 = __half2float(__half(h0)) * s, f1 = __half2float(__half(h1)) * s;
    __nv_bfloat162 pr = __floats2bfloat162_rn(f0, f1);
    w[i] = *reinterpret_cast<uint32_t *>(&pr);
  }
}

}  // namespace csa
