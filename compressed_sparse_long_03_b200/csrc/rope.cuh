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
// before the fp32 sin/cos of that fraction.
#pragma once

#include "common.cuh"

namespace csa {

enum NormRopeFlags : int { kNrNorm = 1, kNrRotate = 2, kNrInverse = 4 };

struct NormRopeArgs {
  const void *x;
  void *y;  // may be x
  long rows;  // R * G head vectors
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

__device__ __forceinline__ long nr_position(const NormRopeArgs &a, long g) {
  if (a.pos) return __ldg(a.pos + g);
  if (a.lens) return (long)__ldg(a.lens + g / a.Tq) - a.Tq + g % a.Tq;
  return (long)a.stride * (g % a.Tq) + a.offset;
}

// (cos, sin) of the angle 2 pi * p * f (p may be negative).
__device__ __forceinline__ float2 rope_cos_sin(long p, double f) {
  double t = (double)p * f;
  t -= floor(t);  // a fraction of a turn in [0, 1)
  float s, c;
  sincospif(2.f * (float)t, &s, &c);
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
// stream large caches at HBM speed.
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
  double f[E / 2];         // turns per position of this lane's pairs
#pragma unroll
  for (int k = 0; k < E; k += 2) {
    const int i = lane * E + k;
    f[k / 2] = i >= d0 ? rope_turns((i - d0) >> 1, a.r, a.log2_base) : 0.0;
  }
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
        const float inv = 1.f / sqrtf(ss / (float)D + a.eps);
#pragma unroll
        for (int k = 0; k < E; ++k) v[u][k] = v[u][k] * inv * g[k];
      }
      if ((a.flags & kNrRotate) && lane * E + E > d0) {
        long p = nr_position(a, row / a.G);
        if (a.flags & kNrInverse) p = -p;
#pragma unroll
        for (int k = 0; k < E; k += 2) {
          const int i = lane * E + k;
          if (i >= d0) rope_turn(v[u][k], v[u][k + 1], rope_cos_sin(p, f[k / 2]), false);
        }
      }
      V::st(y + (size_t)row * D + lane * E, v[u]);
    }
  }
}

}  // namespace csa
