// attend_tc.cuh -- single-KV-head attention over selected (CSA) or all (HCA)
// compressed entries plus the sliding window, on the tcgen05 tensor cores.
// bf16 inputs, head dim 128, up to 128 query heads.
//
// "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part V":
// "The skeleton, and what's kept" (one key-value head shared by all query
// heads; the cached entry is both key and value), CSA and HCA bullets (the
// selected / all entries), first of the "three details" (every layer also
// attends to the last 128 tokens under the same softmax).
//
// One query row per cluster of CS CTAs; CTA `rank` takes a contiguous range
// of the row's key list ([selected entries] ++ [window tokens]) in tiles of
// up to 256 keys.  Per tile:
//   gather  cp.async 16-byte chunks of the key rows into shared memory in the
//           128-byte-swizzled layout (invalid slots are zero-filled);
//   S = Q K^T   tcgen05.mma, M = 128 (heads, zero-padded), N = tile keys,
//           K = 128; A = Q (K-major), B = the key tile (K-major);
//   softmax thread h owns TMEM lane h = head h: base-2 online softmax over
//           its row of S; P (bf16) written back in the swizzled K-major layout;
//   O = P V  tcgen05.mma, M = 128, N = 128 (head dim), K = tile keys;
//           A = P, B = the SAME key tile read MN-major (the entry is the value);
//   accumulate  O is read back per lane and folded into registers with the
//           running rescale.
// Each CTA pushes its partial (max, sum, output) of every head into the
// shared memory of the CTA that finalises that head (distributed shared
// memory stores); after one cluster barrier each CTA merges its heads in
// fixed rank order from local memory.
#pragma once

#include <cooperative_groups.h>

#include "attend_fma.cuh"
#include "common.cuh"
#include "fp8.cuh"
#include "sm100.cuh"

namespace csa {

constexpr int kAtThreads = 256;  // two threads per TMEM lane (head): column halves
constexpr int kAtMaxTile = 192;                      // keys per tile
constexpr uint32_t kAtQAtom = 128 * 128;             // 128 rows x 128 B
constexpr uint32_t kAtKHalf = kAtMaxTile * 128;      // one 64-wide d slice of the key tile
constexpr uint32_t kAtPAtom = 128 * 128;             // 128 heads x 64 keys x 2 B
constexpr uint32_t kAtPart = 128 * 128 * 4;          // partial outputs pushed by the cluster
constexpr uint32_t kAtF8Rows = kAtMaxTile * 64 + kAtMaxTile * 4;  // raw codes + scale words of a tile
// Dynamic shared memory: Q, the key tile (two, double-buffered, for one-CTA
// rows), P, for clusters the partials pushed by the peers, and with FP8
// entries the tiles' raw codes and scale words.
__host__ __device__ constexpr size_t at_smem_bytes(int cs, bool fp8 = false) {
  return 1024 + 2 * kAtQAtom + (cs == 1 ? 2 : 1) * 2 * kAtKHalf + (kAtMaxTile / 64) * kAtPAtom +
         (cs == 1 ? 0 : kAtPart) + (fp8 ? (cs == 1 ? 2 : 1) * kAtF8Rows : 0);
}

__device__ __forceinline__ void at_cp_async4(uint32_t dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

template <int CS>
__global__ void __launch_bounds__(kAtThreads, 1) k_attend_tc(AttendArgs a) {
  using namespace sm100;
  constexpr int D = 128;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_holder;
  __shared__ uint64_t bar_s, bar_o;
  constexpr int NKB = CS == 1 ? 2 : 1;  // key-tile buffers
  __shared__ int kvalid[NKB][kAtMaxTile / 32];  // validity bits, one word per 32 keys
  __shared__ const __nv_bfloat16 *rowp[NKB][kAtMaxTile];
  __shared__ int rowe[NKB][kAtMaxTile];  // FP8 entries: the entry's row in the cache planes, else -1
  __shared__ float pm[136], pl[136];   // pushed partial max / sum [hl * CS + c]
  __shared__ float xmax[2][128];       // per-half row max (then sum) of the partner
  __shared__ float mw[136], minv[128];  // merge weights [hl * CS + c], 1 / sum
  __shared__ int abort_flag;
  __shared__ float2 rot_cs[64];  // (cos, sin) of the query position's RoPE angles
  __shared__ float sgam[128];    // the query's RMSNorm gain (QK-norm)

  uint8_t *base = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = base;
  uint8_t *sK = sQ + 2 * kAtQAtom;       // NKB x [2 d-halves][kAtMaxTile rows][128 B]
  uint8_t *sP = sK + NKB * 2 * kAtKHalf;
  // partials of the heads this CTA finalises, written by every CTA of the
  // cluster: [head slot hl][source rank c][128] (slot hl = head h / CS)
  float *part = reinterpret_cast<float *>(sP + (kAtMaxTile / 64) * kAtPAtom);
  // FP8 entries: raw codes [NKB][tile rows][64 B], then scale words [NKB][tile rows]
  uint8_t *sF8 = reinterpret_cast<uint8_t *>(part) + (CS == 1 ? 0 : kAtPart);
  uint32_t *sF8s = reinterpret_cast<uint32_t *>(sF8 + NKB * kAtMaxTile * 64);
  const bool f8 = a.kv_fp8 != nullptr;
  const __nv_bfloat16 *kv_rp = static_cast<const __nv_bfloat16 *>(a.kv_rope);

  const int rank = (CS > 1) ? (int)cg::this_cluster().block_rank() : 0;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int H = a.H;
  const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(a.q);
  const __nv_bfloat16 *kv_c = static_cast<const __nv_bfloat16 *>(a.kv_c);
  const __nv_bfloat16 *kv_tok = static_cast<const __nv_bfloat16 *>(a.kv_tok);

  // set-up that touches no global memory runs before the wait on the
  // previous kernel: barriers and the TMEM allocation
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_holder), 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar_s), 1);
    mbar_init(smem_u32(&bar_o), 1);
    fence_barrier_init();
  }
  pdl_wait();
  pdl_launch_dependents();
  uint32_t ns = 0, no = 0;  // mbarrier phases, carried from row to row
  bool cta_alive = true;
  // one query row per cluster; with one CTA per row (CS == 1) the CTAs are
  // persistent and take rows blockIdx.x, blockIdx.x + gridDim.x, ...
  for (int r = blockIdx.x / CS; r < a.R && cta_alive; r += (CS == 1 ? (int)gridDim.x : a.R)) {
  const int b = r / a.Tq, tq = r % a.Tq;
  __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(a.out) + (size_t)r * H * D;
  // Q rows (heads) in the swizzled K-major layout; heads >= H are zero rows
  const __nv_bfloat16 *qrow = q + (size_t)r * H * D;
  for (int u = tid; u < 128 * 16; u += kAtThreads) {
    const int h = u >> 4, c = u & 15;
    const uint32_t dst = smem_u32(sQ) + (c >> 3) * kAtQAtom + h * 128 + (((c & 7) ^ (h & 7)) << 4);
    cp_async16(dst, h < H ? qrow + (size_t)h * D + c * 8 : qrow, h < H ? 16u : 0u);
  }
  cp_async_commit();  // Q in a group of its own: the QK-norm prologue waits for Q alone
  if ((a.qk_flags & kNrNorm) && tid < D)
    sgam[tid] = a.q_gamma ? __bfloat162float(static_cast<const __nv_bfloat16 *>(a.q_gamma)[tid]) : 1.f;
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
  if (!ok) {  // uniform over the cluster
    for (int u = tid; u < H * D; u += kAtThreads)
      if ((u / D) % CS == rank) out[u] = __float2bfloat16_rn(0.f);
    cp_async_wait_all();
    __syncthreads();  // Q's buffer is free for the next row
    continue;
  }

  const int nsel = a.idx ? a.k : v;
  const int L = nsel + nwin;
  const int per = (L + CS - 1) / CS;
  const int lo = min(L, rank * per), hi = min(L, lo + per);
  if ((a.qk_flags & kNrRotate) && tid < a.rope_r / 2)
    rot_cs[tid] = rope_cos_sin(t, rope_turns(tid, a.rope_r, a.rope_log2_base));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tS = tmem_holder, tO = tmem_holder + 256;
  // warp w reads TMEM lanes 32*(w%4).. (its quadrant: heads hq..hq+31) and
  // works on one half of the columns (w/4): the key chunks [c0, c1) of S and
  // the output columns [64*half, 64*half+64) of O
  const int quad = warp & 3, half = warp >> 2;
  const int hrow = quad * 32 + (tid & 31);  // this thread's head (TMEM lane)
  const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
  const bool live = quad * 32 < H;  // quadrants of padded heads (>= H) skip the math
  volatile int *abort = &abort_flag;

  float o[D / 2];
#pragma unroll
  for (int e = 0; e < D / 2; ++e) o[e] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;  // l_run: this half's share of the sum
  bool alive = true;

  // row pointers (one coalesced index read) and validity words of the tile
  // at p0 into buffer kb
  auto stage_ptrs = [&](int p0, int kb) {
    const int nt = min(kAtMaxTile, hi - p0), nc = (nt + 31) >> 5;
    for (int j = tid; j < nc * 32; j += kAtThreads) {
      const int p = p0 + j;
      const __nv_bfloat16 *row = nullptr;
      int e = -1;
      if (j < nt) {
        if (p < nsel) {
          const int i = a.idx ? __ldg(a.idx + (size_t)r * a.k + p) : p;
          if (i >= 0 && i < v) {
            if (f8) {
              e = b * a.nc_max + i;
              row = kv_rp + (size_t)e * (D / 2);
            } else {
              row = kv_c + ((size_t)b * a.nc_max + i) * D;
            }
          }
        } else {
          const int s = w0 + (p - nsel);
          row = kv_tok + ((size_t)b * a.n_tok + (s % a.n_tok)) * D;
        }
      }
      rowp[kb][j] = row;
      rowe[kb][j] = e;
      // a warp covers 32 consecutive keys: one validity word per 32
      const unsigned vm = __ballot_sync(0xffffffffu, row != nullptr);
      if ((tid & 31) == 0) kvalid[kb][j >> 5] = (int)vm;
    }
  };
  // the tile's rows into key buffer kb: 16 chunks of 16 B each (one
  // cp.async group)
  auto gather = [&](int p0, int kb) {
    const int nt = min(kAtMaxTile, hi - p0), nc = (nt + 31) >> 5;
    const uint32_t k0 = smem_u32(sK) + kb * 2 * kAtKHalf;
    for (int u = tid; u < nc * 32 * 16; u += kAtThreads) {
      const int j = u >> 4, c = u & 15;
      const __nv_bfloat16 *row = rowp[kb][j];
      const uint32_t dst = k0 + (c >> 3) * kAtKHalf + j * 128 + (((c & 7) ^ (j & 7)) << 4);
      const int e = f8 ? rowe[kb][j] : -1;
      if (e < 0) {
        cp_async16(dst, row ? row + c * 8 : kv_tok, row ? 16u : 0u);
      } else if (c >= 8) {  // the bf16 (rotated) half of an FP8 entry, straight into the tile
        cp_async16(dst, row + (c - 8) * 8, 16u);
      } else if (c < 4) {   // its 64 codes, raw, widened once the tile has landed
        cp_async16(smem_u32(sF8) + (kb * kAtMaxTile + j) * 64 + c * 16, a.kv_fp8 + (size_t)e * 64 + c * 16, 16u);
      } else if (c == 4) {  // the aligned word holding its scale byte
        at_cp_async4(smem_u32(sF8s + kb * kAtMaxTile + j), a.kv_sc + (e & ~3));
      }
    }
    cp_async_commit();
  };
  if constexpr (NKB == 2) {
    if (lo < hi) {
      stage_ptrs(lo, 0);
      __syncthreads();
      gather(lo, 0);
    }
  }

  int kb = 0;
  for (int p0 = lo; p0 < hi && alive; p0 += kAtMaxTile, kb ^= NKB - 1) {
    const int ntile = min(kAtMaxTile, hi - p0);
    const int nchunk = (ntile + 31) >> 5;  // 32-key chunks; MMA N = 32 * nchunk
    const int pn = p0 + kAtMaxTile;
    if constexpr (NKB == 1) {
      stage_ptrs(p0, 0);
      __syncthreads();
      gather(p0, 0);
    } else if (pn < hi) {
      stage_ptrs(pn, kb ^ 1);  // while this tile's rows are in flight
    }
    if (a.qk_flags && p0 == lo) {
      // QK-norm and partial RoPE of the staged query rows, in place, while
      // the first key tile is still in flight: this thread's 64 columns of
      // head hrow are the 8 swizzled 16-byte chunks of row hrow in Q atom
      // `half`; the row's sum of squares is completed through the partner
      cp_async_wait_group<1>();  // Q's group (the older one) has landed
      __syncthreads();
      const uint32_t qa = smem_u32(sQ) + half * kAtQAtom + hrow * 128;
      float ss = 0.f;
      if (hrow < H) {
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t w0_, w1_, w2_, w3_;
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(w0_), "=r"(w1_), "=r"(w2_), "=r"(w3_)
                       : "r"(qa + ((cc ^ (hrow & 7)) << 4)));
          const uint32_t w[4] = {w0_, w1_, w2_, w3_};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = __uint_as_float(w[e] << 16), x1 = __uint_as_float(w[e] & 0xFFFF0000u);
            ss = fmaf(x0, x0, fmaf(x1, x1, ss));
          }
        }
      }
      xmax[half][hrow] = ss;
      __syncthreads();
      ss += xmax[half ^ 1][hrow];
      const bool nrm = (a.qk_flags & kNrNorm) != 0;
      const float inv = nrm ? 1.f / sqrtf(ss / (float)D + a.q_eps) : 1.f;
      const int d0 = D - a.rope_r;
      if (hrow < H) {
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          const uint32_t addr = qa + ((cc ^ (hrow & 7)) << 4);
          uint32_t w0_, w1_, w2_, w3_;
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(w0_), "=r"(w1_), "=r"(w2_), "=r"(w3_)
                       : "r"(addr));
          uint32_t w[4] = {w0_, w1_, w2_, w3_};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int col = half * (D / 2) + cc * 8 + 2 * e;
            float x0 = __uint_as_float(w[e] << 16) * inv, x1 = __uint_as_float(w[e] & 0xFFFF0000u) * inv;
            if (nrm) {
              x0 *= sgam[col];
              x1 *= sgam[col + 1];
            }
            if ((a.qk_flags & kNrRotate) && col >= d0) rope_turn(x0, x1, rot_cs[(col - d0) >> 1], false);
            __nv_bfloat162 pr = __floats2bfloat162_rn(x0, x1);
            w[e] = *reinterpret_cast<uint32_t *>(&pr);
          }
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                       "r"(w[3])
                       : "memory");
        }
      }
      // made visible to the tensor core by the fence and barrier below
    }
    cp_async_wait_group<0>();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if constexpr (NKB == 2) {
      if (pn < hi) gather(pn, kb ^ 1);  // the next tile's rows during this tile's math
    }
    const uint32_t sKb = smem_u32(sK) + kb * 2 * kAtKHalf;
    if (f8) {
      // widen the FP8 entries' codes into the tile's first 64 dims: 8 codes
      // (16 B of bf16, one swizzled chunk) per thread and step
      for (int u = tid; u < nchunk * 32 * 8; u += kAtThreads) {
        const int j = u >> 3, c = u & 7;
        const int e = rowe[kb][j];
        if (e < 0) continue;
        const uint32_t sw = sF8s[kb * kAtMaxTile + j];
        const int X = (int)((sw >> (8 * (e & 3))) & 0xFFu) - 127;
        const uint2 raw = *reinterpret_cast<const uint2 *>(sF8 + (kb * kAtMaxTile + j) * 64 + c * 8);
        uint32_t w[4];
        f8_widen8(raw.x, raw.y, f8_pow2(X), w);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sKb + j * 128 + ((c ^ (j & 7)) << 4)),
                     "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                     : "memory");
      }
      fence_proxy_async_smem();
      __syncthreads();
    }
    // ---- S = Q K^T
    if (tid == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 32 * nchunk);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * kAtQAtom + (k & 3) * 32;
        const uint32_t koff = (k >> 2) * kAtKHalf + (k & 3) * 32;
        umma_bf16(tS, sdesc_kmajor_sw128(smem_u32(sQ) + off), sdesc_kmajor_sw128(sKb + koff), idesc, k > 0);
      }
      umma_commit(smem_u32(&bar_s));
    }
    alive = mbar_wait(smem_u32(&bar_s), ns & 1, abort);
    alive = __syncthreads_and(alive);
    ++ns;
    if (!alive) break;
    tc_fence_after();
    // ---- softmax over this head's row, the two column halves in parallel:
    // this thread's chunks are read from TMEM once (one wait), the row max
    // is combined with the partner thread through shared memory
    const int cs0 = (nchunk + 1) >> 1;
    const int c0 = half ? cs0 : 0, c1 = half ? nchunk : cs0;
    uint32_t sv[kAtMaxTile / 64][32];
    float mt = -INFINITY;
    if (live) {
#pragma unroll
      for (int i = 0; i < kAtMaxTile / 64; ++i) {
        if (c0 + i < c1) {
          tmem_ld16(tS + lane_off + 32 * (c0 + i), sv[i]);
          tmem_ld16(tS + lane_off + 32 * (c0 + i) + 16, sv[i] + 16);
        }
      }
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < kAtMaxTile / 64; ++i) {
        if (c0 + i < c1) {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) asm volatile("" : "+r"(sv[i][jj]));
          const uint32_t vm = (uint32_t)kvalid[kb][c0 + i];
#pragma unroll
          for (int jj = 0; jj < 32; ++jj)
            if ((vm >> jj) & 1u) mt = fmaxf(mt, __uint_as_float(sv[i][jj]) * a.scale_log2);
        }
      }
    }
    xmax[half][hrow] = mt;
    __syncthreads();
    mt = fmaxf(mt, xmax[half ^ 1][hrow]);
    const float m_new = fmaxf(m_run, mt);
    const float alpha = (m_new == -INFINITY) ? 1.f : ex2(m_run - m_new);
    float lsum = 0.f;
    if (live) {
#pragma unroll
      for (int i = 0; i < kAtMaxTile / 64; ++i) {
        if (c0 + i < c1) {
          const int c = c0 + i;
          const uint32_t vm = (uint32_t)kvalid[kb][c];
#pragma unroll
          for (int g = 0; g < 4; ++g) {  // 8 keys -> one 16-byte chunk of P
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j0 = 8 * g + 2 * e;
              const float p0v = ((vm >> j0) & 1u) ? ex2(__uint_as_float(sv[i][j0]) * a.scale_log2 - m_new) : 0.f;
              const float p1v =
                  ((vm >> (j0 + 1)) & 1u) ? ex2(__uint_as_float(sv[i][j0 + 1]) * a.scale_log2 - m_new) : 0.f;
              lsum += p0v + p1v;
              __nv_bfloat162 pr = __floats2bfloat162_rn(p0v, p1v);
              pk[e] = *reinterpret_cast<uint32_t *>(&pr);
            }
            const int kg = 4 * c + g;  // 8-key group index 0..23
            const uint32_t dst =
                smem_u32(sP) + (kg >> 3) * kAtPAtom + hrow * 128 + (((kg & 7) ^ (hrow & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(pk[0]), "r"(pk[1]),
                         "r"(pk[2]), "r"(pk[3])
                         : "memory");
          }
        }
      }
    }
    if (m_new != -INFINITY) {
      l_run = l_run * alpha + lsum;
      m_run = m_new;
    }
    tc_fence_before();
    fence_proxy_async_smem();
    __syncthreads();
    tc_fence_after();
    // ---- O = P V (the key tile read MN-major as the value operand)
    if (tid == 0) {
      const uint32_t idesc = idesc_bf16_f32_bmn(128, D);
      for (int k = 0; k < 2 * nchunk; ++k) {  // 16 keys per MMA
        const uint32_t poff = (k >> 2) * kAtPAtom + (k & 3) * 32;
        umma_bf16(tO, sdesc_kmajor_sw128(smem_u32(sP) + poff),
                  sdesc_mnmajor_sw128(sKb + k * 2048, kAtKHalf), idesc, k > 0);
      }
      umma_commit(smem_u32(&bar_o));
    }
    alive = mbar_wait(smem_u32(&bar_o), no & 1, abort);
    alive = __syncthreads_and(alive);
    ++no;
    if (!alive) break;
    tc_fence_after();
    const float scl = (m_new == -INFINITY) ? 1.f : alpha;
    if (live) {
      uint32_t ov[D / 2];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld16(tO + lane_off + half * (D / 2) + 16 * c, ov + 16 * c);
      tmem_wait_ld_regs<D / 2>(ov);
#pragma unroll
      for (int e = 0; e < D / 2; ++e) o[e] = fmaf(o[e], scl, __uint_as_float(ov[e]));
    }
    tc_fence_before();
    __syncthreads();  // every lane done with S, P and O before they are rewritten
  }
  cp_async_wait_group<0>();  // a tile still in flight after a timeout lands before exit

  xmax[half][hrow] = l_run;
  __syncthreads();
  if constexpr (CS == 1) {
    // one CTA holds the whole row: normalise (with the sink when given) and
    // store this half's 64 output columns
    if (hrow < H) {
      const float lt = l_run + xmax[half ^ 1][hrow];
      const float sk = sink_log2(a, hrow);
      float f = 1.f / lt;
      if (sk != -INFINITY) {
        const float M = fmaxf(m_run, sk), so = ex2(m_run - M);
        f = so / (lt * so + ex2(sk - M));
      }
      uint4 *dst = reinterpret_cast<uint4 *>(out + (size_t)hrow * D + half * (D / 2));
#pragma unroll
      for (int j = 0; j < D / 16; ++j) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float x0 = o[8 * j + 2 * e] * f, x1 = o[8 * j + 2 * e + 1] * f;
          const int col = half * (D / 2) + 8 * j + 2 * e;
          if ((a.qk_flags & kNrRotate) && col >= D - a.rope_r)  // back by the query's position
            rope_turn(x0, x1, rot_cs[(col - (D - a.rope_r)) >> 1], true);
          __nv_bfloat162 pr = __floats2bfloat162_rn(x0, x1);
          w4[e] = *reinterpret_cast<uint32_t *>(&pr);
        }
        dst[j] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
    }
  } else {
  // ---- push this CTA's partial (max, sum, output) of head h into the CTA
  // that finalises h (rank h % CS), one cluster barrier, merge locally; the
  // two halves of a row push their output columns, half 0 the max and the
  // sum of both halves
  if (hrow < H) {
    const int own = hrow % CS, slot = (hrow / CS) * CS + rank;
    float4 *dst = reinterpret_cast<float4 *>(att_peer<CS>(part, own) + (size_t)slot * D + half * (D / 2));
#pragma unroll
    for (int j = 0; j < D / 8; ++j) dst[j] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
    if (half == 0) {
      att_peer<CS>(pm, own)[slot] = m_run;
      att_peer<CS>(pl, own)[slot] = l_run + xmax[1][hrow];
    }
  }
  att_cluster_sync<CS>();
  // merge weights of this CTA's heads (h = rank + CS * hl), ranks in order
  const int nmine = (H - rank + CS - 1) / CS;
  if (tid < nmine) {
    const float sk = sink_log2(a, rank + CS * tid);
    float M = sk;
#pragma unroll
    for (int c = 0; c < CS; ++c) M = fmaxf(M, pm[tid * CS + c]);
    float Ls = sk == -INFINITY ? 0.f : ex2(sk - M);
#pragma unroll
    for (int c = 0; c < CS; ++c) {
      const float mc = pm[tid * CS + c];
      const float wgt = (mc == -INFINITY) ? 0.f : ex2(mc - M);
      Ls = fmaf(pl[tid * CS + c], wgt, Ls);
      mw[tid * CS + c] = wgt;
    }
    minv[tid] = 1.f / Ls;
  }
  __syncthreads();
  for (int u = tid; u < nmine * (D / 4); u += kAtThreads) {
    const int hl = u / (D / 4), j = u % (D / 4);
    const int h = rank + CS * hl;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int c = 0; c < CS; ++c) {
      const float wgt = mw[hl * CS + c];
      if (wgt == 0.f) continue;
      const float4 p = reinterpret_cast<const float4 *>(part + (size_t)(hl * CS + c) * D)[j];
      acc.x = fmaf(p.x, wgt, acc.x);
      acc.y = fmaf(p.y, wgt, acc.y);
      acc.z = fmaf(p.z, wgt, acc.z);
      acc.w = fmaf(p.w, wgt, acc.w);
    }
    const float il = minv[hl];
    acc.x *= il;
    acc.y *= il;
    acc.z *= il;
    acc.w *= il;
    if (a.qk_flags & kNrRotate) {  // back by the query's position
      const int d0 = D - a.rope_r;
      if (4 * j >= d0) rope_turn(acc.x, acc.y, rot_cs[(4 * j - d0) >> 1], true);
      if (4 * j + 2 >= d0) rope_turn(acc.z, acc.w, rot_cs[(4 * j + 2 - d0) >> 1], true);
    }
    __nv_bfloat162 lo2 = __floats2bfloat162_rn(acc.x, acc.y);
    __nv_bfloat162 hi2 = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t *>(&lo2);
    pk.y = *reinterpret_cast<uint32_t *>(&hi2);
    *reinterpret_cast<uint2 *>(out + (size_t)h * D + 4 * j) = pk;
  }
  }  // clusters
  if (!alive) cta_alive = false;  // a wait gave up: no further rows
  tc_fence_before();
  __syncthreads();  // every thread is done with this row's Q, tiles, P and TMEM reads
  tc_fence_after();
  }  // rows
  if (tid == 0 && abort_flag) raise_dev_err(kDevErrTimeout);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_holder, 512);
  }
}

}  // namespace csa
