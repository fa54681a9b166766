// rope.cuh -- QK-norm and partial RoPE.
//
// "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part V", "The
// attention: compress, then select", third detail: queries and compressed
// entries are RMS-normalised per head and RoPE turns only the last dims of
// each vector; because the cached entry is also the value, the attention
// output carries absolute position and is turned back by its own query's
// position.  Per head of d dims:
//   y = x / sqrt(mean(x^2) + eps) * gamma            (normalisation)
//   (y[i], y[i+1]) turned by the angle p * base^(-2j/r) for the adjacent
//   pairs i = d - r + 2j of the last r dims          (rotation; -p: inverse)
//
// Angles: a position can reach 2^31 and the first pair turns at one radian
// per position, so the angle is reduced in fp64 as a fraction of a full turn
// (p * f_j, f_j = base^(-2j/r) / 2pi, computed once per thread in fp64)
// before the fp32 sine and cosine of that fraction.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace csa {

enum NormRopeFlags : int { kNrNorm = 1, kNrRotate = 2, kNrInverse = 4 };

struct NormRopeArgs {
  const void *x;
  void *y;  // may be x
  long rows;  // R * G head vectors (< 2^31: positions use 32-bit division)
  int G;      // heads sharing one position
  // position of row group r: pos[r]; else lens[r / Tq] - Tq + r % Tq (the
  // decode rule of the attention); else stride * (r % Tq) + offset
  const int32_t *pos;
  const int32_t *lens;
  int Tq, stride, offset;
  const void *gamma;  // [d] or nullptr (ones)
  float eps;
  int r;      // rotated dims (even, <= d)
  int flags;  // NormRopeFlags
  double log2_base;
};

// Turns per unit of position of rotated pair j: base^(-2j/r) / (2 pi).
__device__ __forceinline__ double rope_turns(int j, int r, double log2_base) {
  return exp2(-2.0 * j / r * log2_base) * 0.15915494309189535;
}

__device__ __forceinline__ long nr_position(const NormRopeArgs &a, uint32_t g) {
  if (a.pos) return __ldg(a.pos + g);
  const uint32_t tq = (uint32_t)a.Tq, b = g / tq, r = g - b * tq;
  if (a.lens) return (long)__ldg(a.lens + b) - a.Tq + (long)r;
  return (long)a.stride * r + a.offset;
}

// (cos, sin) of the angle 2 pi * p * f (p may be negative).
__device__ __forceinline__ float2 rope_cos_sin(long p, double f) {
  double t = (double)p * f;
  t -= floor(t);  // a fraction of a turn in [0, 1)
  float s, c;
  sincospif(2.f * (float)t, &s, &c);
  return make_float2(c, s);
}

// Turns per position in 64-bit fixed point (f < 1: the fraction f * 2^64).
__device__ __forceinline__ uint64_t rope_turns_fixed(double f) {
  return (uint64_t)__double2ll_rn(f * 18446744073709551616.0);
}

// (cos, sin) of the angle 2 pi * p * F / 2^64 for a result stored in T.  The
// product p * F taken modulo 2^64 is the angle's fraction of a turn (integer
// arithmetic: exact for any p, negative p included); its top 32 bits, read
// as a signed number, are that fraction in [-1/2, 1/2).  bf16: the hardware
// sine / cosine of the reduced angle (absolute error a few 1e-7, far below
// the bf16 spacing of 2^-8 relative); fp32: the accurate sincospif.
template <typename T>
__device__ __forceinline__ float2 rope_cos_sin_fixed(long p, uint64_t F) {
  const int32_t hi = (int32_t)(((uint64_t)p * F) >> 32);
  float s, c;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    __sincosf((float)hi * 1.4629180792671596e-09f, &s, &c);  // 2 pi / 2^32
  } else {
    sincospif((float)hi * 4.6566128730773926e-10f, &s, &c);  // 2^-31
  }
  return make_float2(c, s);
}

// Turn the pair (u, v) by the angle whose (cos, sin) is cs; backwards when
// `back` (the inverse rotation).
__device__ __forceinline__ void rope_turn(float &u, float &v, float2 cs, bool back) {
  const float a = u, b = v, s = back ? -cs.y : cs.y;
  u = a * cs.x - b * s;
  v = a * s + b * cs.x;
}

template <typename T, int E>
struct NrVec;
template <>
struct NrVec<float, 2> {
  static __device__ __forceinline__ void ld(const void *p, float *f) {
    const float2 v = *reinterpret_cast<const float2 *>(p);
    f[0] = v.x; f[1] = v.y;
  }
  static __device__ __forceinline__ void st(void *p, const float *f) {
    *reinterpret_cast<float2 *>(p) = make_float2(f[0], f[1]);
  }
};
template <>
struct NrVec<float, 4> {
  static __device__ __forceinline__ void ld(const void *p, float *f) {
    const float4 v = *reinterpret_cast<const float4 *>(p);
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
  }
  static __device__ __forceinline__ void st(void *p, const float *f) {
    *reinterpret_cast<float4 *>(p) = make_float4(f[0], f[1], f[2], f[3]);
  }
};
template <>
struct NrVec<__nv_bfloat16, 2> {
  static __device__ __forceinline__ void ld(const void *p, float *f) {
    const uint32_t w = *reinterpret_cast<const uint32_t *>(p);
    f[0] = __uint_as_float(w << 16);
    f[1] = __uint_as_float(w & 0xFFFF0000u);
  }
  static __device__ __forceinline__ void st(void *p, const float *f) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f[0], f[1]);
    *reinterpret_cast<__nv_bfloat162 *>(p) = h;
  }
};
template <>
struct NrVec<__nv_bfloat16, 4> {
  static __device__ __forceinline__ void ld(const void *p, float *f) {
    const uint2 w = *reinterpret_cast<const uint2 *>(p);
    f[0] = __uint_as_float(w.x << 16);
    f[1] = __uint_as_float(w.x & 0xFFFF0000u);
    f[2] = __uint_as_float(w.y << 16);
    f[3] = __uint_as_float(w.y & 0xFFFF0000u);
  }
  static __device__ __forceinline__ void st(void *p, const float *f) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(f[0], f[1]), hi = __floats2bfloat162_rn(f[2], f[3]);
    uint2 w;
    w.x = *reinterpret_cast<uint32_t *>(&lo);
    w.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(p) = w;
  }
};

constexpr int kNrThreads = 256;
constexpr int kNrUnroll = 4;  // head vectors a warp has in flight

// One warp per head vector, E = D / 32 consecutive dims per lane (a rotated
// pair never straddles two lanes: d - r and 2j are even).  Each warp loads
// kNrUnroll vectors before it works on them, for enough loads in flight to
// stream large caches at HBM speed.  A row's angles are spread over the
// whole warp (lane l computes pairs l and l + 32) and handed to the lanes
// that own the pairs' dims by shuffles.
template <typename T, int D>
__global__ void __launch_bounds__(kNrThreads) k_norm_rope(NormRopeArgs a) {
  constexpr int E = D / 32;
  static_assert(E == 2 || E == 4, "d of 64 or 128");
  using V = NrVec<T, E>;
  const int lane = threadIdx.x & 31;
  const long nwarps = (long)gridDim.x * (kNrThreads / 32);
  const long w0 = (long)blockIdx.x * (kNrThreads / 32) + (threadIdx.x >> 5);
  const T *x = static_cast<const T *>(a.x);
  T *y = static_cast<T *>(a.y);
  pdl_wait();
  pdl_launch_dependents();
  float g[E];
#pragma unroll
  for (int k = 0; k < E; ++k)
    g[k] = a.gamma ? to_f(static_cast<const T *>(a.gamma)[lane * E + k]) : 1.f;
  const int d0 = D - a.r;  // first rotated dim
  const int npairs = a.r >> 1;
  // turns per position of the pairs this lane computes angles for
  const uint64_t F0 = lane < npairs ? rope_turns_fixed(rope_turns(lane, a.r, a.log2_base)) : 0;
  const uint64_t F1 = lane + 32 < npairs ? rope_turns_fixed(rope_turns(lane + 32, a.r, a.log2_base)) : 0;
  for (long base = w0; base < a.rows; base += nwarps * kNrUnroll) {
    float v[kNrUnroll][E];
#pragma unroll
    for (int u = 0; u < kNrUnroll; ++u) {
      const long row = base + u * nwarps;
      if (row < a.rows) V::ld(x + (size_t)row * D + lane * E, v[u]);
    }
#pragma unroll
    for (int u = 0; u < kNrUnroll; ++u) {
      const long row = base + u * nwarps;
      if (row >= a.rows) break;  // uniform over the warp
      if (a.flags & kNrNorm) {
        float ss = 0.f;
#pragma unroll
        for (int k = 0; k < E; ++k) ss = fmaf(v[u][k], v[u][k], ss);
        ss = warp_sum(ss);
        float inv;
        if constexpr (std::is_same<T, __nv_bfloat16>::value) {
          inv = rsqrtf(ss / (float)D + a.eps);  // within 2 ulp: far below the bf16 spacing
        } else {
          inv = 1.f / sqrtf(ss / (float)D + a.eps);
        }
#pragma unroll
        for (int k = 0; k < E; ++k) v[u][k] = v[u][k] * inv * g[k];
      }
      if (a.flags & kNrRotate) {  // uniform over the warp: every lane takes the shuffles
        long p = nr_position(a, a.G == 1 ? (uint32_t)row : (uint32_t)row / (uint32_t)a.G);
        if (a.flags & kNrInverse) p = -p;
        const float2 cs0 = rope_cos_sin_fixed<T>(p, F0);
        const float2 cs1 = npairs > 32 ? rope_cos_sin_fixed<T>(p, F1) : cs0;
#pragma unroll
        for (int k = 0; k < E; k += 2) {
          const int i = lane * E + k;
          const int j = (i - d0) >> 1;  // this lane's pair (negative: not rotated)
          float2 c;
          c.x = __shfl_sync(0xffffffffu, cs0.x, j & 31);
          c.y = __shfl_sync(0xffffffffu, cs0.y, j & 31);
          if (npairs > 32) {
            const float cx = __shfl_sync(0xffffffffu, cs1.x, j & 31);
            const float cy = __shfl_sync(0xffffffffu, cs1.y, j & 31);
            if (j >= 32) c = make_float2(cx, cy);
          }
          if (i >= d0) rope_turn(v[u][k], v[u][k + 1], c, false);
        }
      }
      V::st(y + (size_t)row * D + lane * E, v[u]);
    }
  }
}

}  // namespace csa
