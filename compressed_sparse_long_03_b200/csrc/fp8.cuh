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

#include <type_traits>

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

// The same with eight consecutive elements per lane, for d in {64, 128,
// 256}: a row spans d / 8 lanes (several rows per warp), a 64-element block
// is an aligned group of 8 lanes (its amax by three shuffles), a lane's 8
// codes are one 8-byte store and its rotated dims are copied as they are.
template <typename T>
__global__ void __launch_bounds__(kF8Threads) k_quantize_fp8_entries_v8(const T *__restrict__ x, long rows, int d,
                                                                        int r, uint8_t *__restrict__ fp8,
                                                                        uint8_t *__restrict__ sc,
                                                                        T *__restrict__ rope) {
  constexpr int NV = 8 * (int)sizeof(T) / 16;  // 16-byte vectors per lane
  const int lane = threadIdx.x & 31, lpr = d >> 3, rpw = 32 / lpr;
  const int sub = lane / lpr, l = lane % lpr, q = d - r;
  const long nw = (long)gridDim.x * (kF8Threads / 32);
  const long w = (long)blockIdx.x * (kF8Threads / 32) + (threadIdx.x >> 5);
  const bool is_q = l * 8 < q;  // this lane's dims are FP8 dims (q is a multiple of 64)
  pdl_wait();
  pdl_launch_dependents();
  for (long row0 = w * rpw; row0 < rows; row0 += nw * rpw) {  // uniform over the warp
    const long row = row0 + sub;
    const bool ok = row < rows;
    uint4 raw[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i)
      raw[i] = ok ? *reinterpret_cast<const uint4 *>(x + (size_t)row * d + l * 8 + i * (16 / sizeof(T)))
                  : make_uint4(0, 0, 0, 0);
    float v[8];
    if constexpr (std::is_same<T, float>::value) {
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        v[4 * i] = __uint_as_float(raw[i].x);
        v[4 * i + 1] = __uint_as_float(raw[i].y);
        v[4 * i + 2] = __uint_as_float(raw[i].z);
        v[4 * i + 3] = __uint_as_float(raw[i].w);
      }
    } else {
      const uint32_t ww[4] = {raw[0].x, raw[0].y, raw[0].z, raw[0].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(ww[i] << 16);
        v[2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u);
      }
    }
    float am = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) am = fmaxf(am, fabsf(v[k]));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
    if (!ok) continue;
    if (is_q) {
      int X = am > 0.f ? ilogbf(am) - 8 : -127;
      X = max(-127, min(127, X));
      uint32_t c[2] = {0u, 0u};
#pragma unroll
      for (int k = 0; k < 8; ++k)
        c[k >> 2] |= (uint32_t)__nv_cvt_float_to_fp8(ldexpf(v[k], -X), __NV_SATFINITE, __NV_E4M3) << (8 * (k & 3));
      *reinterpret_cast<uint2 *>(fp8 + (size_t)row * q + l * 8) = make_uint2(c[0], c[1]);
      if ((l & 7) == 0) sc[(size_t)row * (q / 64) + (l >> 3)] = (uint8_t)(X + 127);
    } else {
#pragma unroll
      for (int i = 0; i < NV; ++i)
        *reinterpret_cast<uint4 *>(rope + (size_t)row * r + (l * 8 - q) + i * (16 / sizeof(T))) = raw[i];
    }
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
