// mxfp4.cuh -- MXFP4 indexer keys: the quantiser, and the indexer scores
// over an MXFP4 key cache on the tcgen05 tensor cores.
//
// "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part V", "The KV
// cache, recomputed": the indexer key is 128 numbers in FP4 plus one byte of
// scale per 32 (68 bytes instead of 256 in bf16); CSA bullet: the lightning
// indexer runs in FP4.  Format (the OCP microscaling layout): per block of 32
// elements a power-of-two scale 2^X stored as the byte X + 127; per element
// an E2M1 code (sign bit 3; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), two per
// byte, element 2j in the low nibble.  Codes [rows][dI/2], scales
// [rows][dI/32].
//
// The scores over such a cache are exactly the bf16 indexer's scores over the
// dequantised keys (every dequantised value is a bf16 number).  The decode
// scan is HBM-bound, so the kernel streams the 68-byte keys and widens them
// on chip: TMA brings 128-key code tiles (8 KB) into shared memory, two sets
// of four converter warps (alternate tiles) expand each code byte through a
// 256-entry table (two bf16 values per byte) and apply the block's scale
// with one exact bf16x2 multiply, writing the 128-byte-swizzled bf16 tile
// that the MMA reads;
// producer, MMA issuer and epilogue are those of the bf16 kernel
// (index_score_tc.cuh).  All waits are time-bounded.
#pragma once

#include "common.cuh"
#include "index_score_tc.cuh"
#include "sm100.cuh"

namespace csa {

// ---------------------------------------------------------------------------
// quantiser: one thread per 32-element block
// ---------------------------------------------------------------------------
// floor(log2(a)) of a finite a > 0 (normal or subnormal float)
__device__ __forceinline__ int floor_log2f(float a) {
  const uint32_t u = __float_as_uint(a);
  const int e = (int)((u >> 23) & 0xFF);
  if (e) return e - 127;
  return (31 - __clz(u & 0x7FFFFF)) - 149;  // subnormal: m * 2^-149
}

// nearest E2M1 magnitude code of y >= 0 (exact comparisons), ties to the
// even code, saturating at 6
__device__ __forceinline__ uint32_t e2m1_code(float y) {
  uint32_t c = 0;
  c += (y > 0.25f);
  c += (y >= 0.75f);  // midpoint -> code 2 (even)
  c += (y > 1.25f);
  c += (y >= 1.75f);  // -> 4
  c += (y > 2.5f);
  c += (y >= 3.5f);   // -> 6
  c += (y > 5.0f);
  return c;
}

template <typename T>
__global__ void __launch_bounds__(256) k_quantize_mxfp4(const T *__restrict__ k, long blocks,
                                                        uint8_t *__restrict__ codes,
                                                        uint8_t *__restrict__ scales) {
  pdl_wait();
  pdl_launch_dependents();
  const long g = (long)blockIdx.x * blockDim.x + threadIdx.x;  // block of 32 elements
  if (g >= blocks) return;
  float x[32];
#pragma unroll
  for (int e = 0; e < 32; e += Vec16<T>::N) load16(k + g * 32 + e, x + e);
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(x[e]));
  int X = -127;
  if (amax > 0.f) X = max(-127, min(127, floor_log2f(amax) - 2));
  // 2^-X exactly (X in [-127, 127]; 2^127 is a normal float)
  const float inv = (-X >= -126) ? __uint_as_float((uint32_t)(127 - X) << 23) : __uint_as_float(0x00400000u);
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float v = x[8 * q + e];
      uint32_t c = e2m1_code(fabsf(v) * inv);
      if (__float_as_uint(v) >> 31) c |= 8u;
      word |= c << (4 * e);
    }
    w[q] = word;
  }
  *reinterpret_cast<uint4 *>(codes + g * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  scales[g] = (uint8_t)(X + 127);
}

// ---------------------------------------------------------------------------
// indexer scores over MXFP4 keys
// ---------------------------------------------------------------------------
constexpr int kF4Threads = 448;  // producer, MMA, 4 epilogue warps, 2 x 4 converter warps

// bf16 pair of the two codes of byte b at scale 2^0 (low nibble in the low half)
__host__ __device__ inline uint32_t e2m1_bf16(uint32_t c) {
  // magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 as bf16: exponent (c >> 1) - 1 + 127
  // and mantissa bit c & 1 for c >= 2; 0.5 for c == 1; 0 for c == 0
  const uint32_t m = c & 7;
  const uint32_t mag = m >= 2 ? ((((m >> 1) + 126u) << 7) | ((m & 1u) << 6)) : (m ? 0x3F00u : 0u);
  return ((c & 8) ? 0x8000u : 0u) | mag;
}
__host__ __device__ inline uint32_t e2m1_pair_bf16(uint32_t b) {
  return e2m1_bf16(b & 15) | (e2m1_bf16(b >> 4) << 16);
}

template <int N, int DI>
__global__ void __launch_bounds__(kF4Threads, 1)
    k_index_score_fp4(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmQ,
                      IndexTcArgs a, const uint8_t *__restrict__ scales) {
  using namespace sm100;
  constexpr int KATOMS = DI / 64;
  constexpr uint32_t A_ATOM = kTcRows * 128;
  constexpr uint32_t A_STAGE = A_ATOM * KATOMS;       // bf16 key tile
  constexpr uint32_t C_STAGE = kTcRows * (DI / 2);    // code tile
  constexpr uint32_t B_ATOM = N * 128;
  constexpr uint32_t B_SLOT = B_ATOM * KATOMS;
  constexpr uint32_t TMEM_COLS = (2 * N <= 32) ? 32 : (2 * N <= 64) ? 64 : (2 * N <= 128) ? 128 : 256;
  constexpr uint32_t IDESC = idesc_bf16_f32(kTcRows, N);
  constexpr int SA = 3;  // bf16 tile stages
  constexpr int SC = 6;  // code tile stages

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_holder;
  __shared__ int abort_flag;
  __shared__ int range[3];
  __shared__ int scan[33];
  __shared__ uint32_t lut[256];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t *base = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = base;                         // SA bf16 tiles
  uint8_t *sB = sA + SA * A_STAGE;            // 2 query blocks
  uint8_t *sC = sB + 2 * B_SLOT;              // SC code tiles
  uint64_t *bars = reinterpret_cast<uint64_t *>(sC + SC * C_STAGE);
  const uint32_t c_full = smem_u32(bars), c_empty = c_full + 8 * SC;
  const uint32_t a_full = c_empty + 8 * SC, a_empty = a_full + 8 * SA;
  const uint32_t q_full = a_empty + 8 * SA, q_empty = q_full + 16;
  const uint32_t t_full = q_empty + 16, t_empty = t_full + 16, drain = t_empty + 16;
  volatile int *abort = &abort_flag;

  for (int i = tid; i < 256; i += kF4Threads) lut[i] = e2m1_pair_bf16((uint32_t)i);
  if (tid == 0) {
    abort_flag = 0;
    range[2] = 0;
    for (int s = 0; s < SC; ++s) {
      mbar_init(c_full + 8 * s, 1);
      mbar_init(c_empty + 8 * s, 4);  // converter warps
    }
    for (int s = 0; s < SA; ++s) {
      mbar_init(a_full + 8 * s, 4);   // converter warps
      mbar_init(a_empty + 8 * s, 1);  // MMA commit
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full + 8 * i, 1);
      mbar_init(q_empty + 8 * i, 1);
      mbar_init(t_full + 8 * i, 1);
      mbar_init(t_empty + 8 * i, 4);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmC);
    tma_prefetch_desc(&tmQ);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();
  pdl_launch_dependents();

  // this CTA's contiguous share of the visible tiles (one row per unit)
  {
    const int per = (a.U + kF4Threads - 1) / kF4Threads;
    const int rb = min(a.U, tid * per), re = min(a.U, rb + per);
    int mine = 0;
    for (int r = rb; r < re; ++r) mine += tc_unit_tiles(a, r);
    int total;
    const int before = block_exclusive_scan(mine, scan, &total);
    const long lo = (long)total * blockIdx.x / gridDim.x;
    const long hi = (long)total * (blockIdx.x + 1) / gridDim.x;
    if (lo < hi && before <= lo && lo < before + mine) {
      long acc = before;
      for (int r = rb; r < re; ++r) {
        const int t = tc_unit_tiles(a, r);
        if (lo < acc + t) {
          range[0] = r;
          range[1] = (int)(lo - acc);
          range[2] = (int)(hi - lo);
          break;
        }
        acc += t;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_holder;

  TileWalk wk;
  wk.r = range[0];
  wk.j = range[1];
  wk.left = range[2];
  wk.tiles = wk.left > 0 ? tc_unit_tiles(a, wk.r) : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && wk.left > 0) {
      const uint64_t pol = make_evict_first();
      int cur_r = -1;
      uint32_t nq = 0, nt = 0;
      bool ok = true;
      for (; wk.left > 0 && ok; wk.advance(a)) {
        if (wk.r != cur_r) {
          const uint32_t slot = nq & 1;
          if (!(ok = mbar_wait(q_empty + 8 * slot, ((nq >> 1) & 1) ^ 1, abort))) break;
          mbar_arrive_expect_tx(q_full + 8 * slot, B_SLOT);
#pragma unroll
          for (int ka = 0; ka < KATOMS; ++ka)
            tma_load_2d(smem_u32(sB + slot * B_SLOT + ka * B_ATOM), &tmQ, 64 * ka, wk.r * a.HI,
                        q_full + 8 * slot);
          ++nq;
          cur_r = wk.r;
        }
        const uint32_t s = nt % SC;
        if (!(ok = mbar_wait(c_empty + 8 * s, ((nt / SC) & 1) ^ 1, abort))) break;
        mbar_arrive_expect_tx(c_full + 8 * s, C_STAGE);
        tma_load_2d_hint(smem_u32(sC + s * C_STAGE), &tmC, 0, (wk.r / a.Tq) * a.nc_max + wk.j * kTcRows,
                         c_full + 8 * s, pol);
        ++nt;
      }
      if (!ok) {
        volatile int no_abort = 0;
        for (uint32_t n = (nt > (uint32_t)SC ? nt - SC : 0); n < nt; ++n)
          mbar_wait(c_full + 8 * (n % SC), (n / SC) & 1, &no_abort);
        for (uint32_t n = (nq > 2 ? nq - 2 : 0); n < nq; ++n)
          mbar_wait(q_full + 8 * (n & 1), (n >> 1) & 1, &no_abort);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0 && wk.left > 0) {
      int cur_r = -1;
      uint32_t nq = 0, nt = 0, slot = 0;
      bool ok = true;
      for (; wk.left > 0 && ok; wk.advance(a)) {
        if (wk.r != cur_r) {
          if (cur_r >= 0) umma_commit(q_empty + 8 * slot);
          slot = nq & 1;
          if (!(ok = mbar_wait(q_full + 8 * slot, (nq >> 1) & 1, abort))) break;
          ++nq;
          cur_r = wk.r;
        }
        const uint32_t s = nt % SA, acc = nt & 1;
        if (!(ok = mbar_wait(a_full + 8 * s, (nt / SA) & 1, abort))) break;
        if (!(ok = mbar_wait(t_empty + 8 * acc, ((nt >> 1) & 1) ^ 1, abort))) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * N;
        const uint32_t a0 = smem_u32(sA + s * A_STAGE), b0 = smem_u32(sB + slot * B_SLOT);
#pragma unroll
        for (int k = 0; k < DI / 16; ++k) {
          const uint32_t off = (k >> 2) * A_ATOM + (k & 3) * 32;
          const uint32_t boff = (k >> 2) * B_ATOM + (k & 3) * 32;
          umma_bf16(d, sdesc_kmajor_sw128(a0 + off), sdesc_kmajor_sw128(b0 + boff), IDESC, k > 0);
        }
        umma_commit(a_empty + 8 * s);
        umma_commit(t_full + 8 * acc);
        ++nt;
      }
      umma_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    float wv[N];
    int cur_r = -1, vis = 0;
    uint32_t nt = 0;
    for (; wk.left > 0; wk.advance(a)) {
      if (wk.r != cur_r) {
        cur_r = wk.r;
        vis = tc_row_visible(a, cur_r);
#pragma unroll
        for (int h = 0; h < N; ++h)
          wv[h] = h < a.HI ? __bfloat162float(a.w[(size_t)cur_r * a.HI + h]) : 0.f;
      }
      const uint32_t acc = nt & 1;
      const bool ok = mbar_wait(t_full + 8 * acc, (nt >> 1) & 1, abort);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t d[N];
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + acc * N;
#pragma unroll
      for (int c = 0; c < N / 16; ++c) tmem_ld16(taddr + 16 * c, d + 16 * c);
      tmem_wait_ld_regs<N>(d);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(t_empty + 8 * acc);
      float sc = 0.f;
#pragma unroll
      for (int h = 0; h < N; ++h) sc = fmaf(wv[h], fmaxf(__uint_as_float(d[h]), 0.f), sc);
      const int i = wk.j * kTcRows + row;
      if (i < a.nc_max) a.scores[(size_t)cur_r * a.nc_max + i] = i < vis ? sc : -INFINITY;
      ++nt;
    }
    if (a.fill_invisible) {
      const int et = tid - 64;
      for (int r = blockIdx.x; r < a.R; r += gridDim.x) {
        const int from = tc_row_tiles(a, r) * kTcRows;
        for (int i = from + et; i < a.nc_max; i += 128) a.scores[(size_t)r * a.nc_max + i] = -INFINITY;
      }
    }
  } else {
    // ------------------------------------------------------------ converters
    // thread t widens key row t of the tile: its DI/2 code bytes (16-byte
    // chunks read in a rotated order against bank conflicts) and DI/32
    // scale bytes into 2*DI bytes of the swizzled bf16 tile
    const int t = (tid - 192) & 127;      // the tile row
    const uint32_t set = (tid - 192) >> 7;  // this set widens tiles nt % 2 == set
    // the row's scale bytes (DI / 32 of them), loaded kPre own tiles ahead by
    // a second cursor into a register ring (a load per tile would put a DRAM
    // round trip in front of every tile)
    constexpr int kPre = 8;
    auto scale_word = [&](const TileWalk &w) -> uint32_t {
      if (w.left <= 0 || w.j * kTcRows + t >= a.nc_max) return 0u;
      const long key = (long)(w.r / a.Tq) * a.nc_max + (long)w.j * kTcRows + t;
      if constexpr (DI == 128) return __ldg(reinterpret_cast<const uint32_t *>(scales) + key);
      else return __ldg(reinterpret_cast<const uint16_t *>(scales) + key);
    };
    TileWalk ahead = wk;
    if (set && ahead.left > 0) ahead.advance(a);  // this set's first tile
    auto skip_other = [&](TileWalk &w) {          // to this set's next tile
      for (int i = 0; i < 2 && w.left > 0; ++i) w.advance(a);
    };
    uint32_t ring[kPre];
#pragma unroll
    for (int i = 0; i < kPre; ++i) {
      ring[i] = scale_word(ahead);
      skip_other(ahead);
    }
    uint32_t nt = 0;
    bool alive = true;
    for (; wk.left > 0 && alive; wk.advance(a), ++nt) {
      if ((nt & 1) != set) continue;  // the other set's tile
      const uint32_t sc = nt % SC, sa = nt % SA;
      const uint32_t sbytes = ring[0];
#pragma unroll
      for (int i = 0; i < kPre - 1; ++i) ring[i] = ring[i + 1];
      ring[kPre - 1] = scale_word(ahead);
      skip_other(ahead);
      bool ok = mbar_wait(c_full + 8 * sc, (nt / SC) & 1, abort);
      ok = ok && mbar_wait(a_empty + 8 * sa, ((nt / SA) & 1) ^ 1, abort);
      if (!__all_sync(0xffffffffu, ok)) {
        alive = false;
        break;
      }
      constexpr int NCH = DI / 32;  // 16-byte code chunks per row, 32 elements each
      // chunk (q + t) % NCH is read and widened in step q: neighbouring rows
      // start on different banks
      uint4 cw[NCH];
      const uint8_t *crow = sC + sc * C_STAGE + t * (DI / 2);
#pragma unroll
      for (int q = 0; q < NCH; ++q) cw[q] = *reinterpret_cast<const uint4 *>(crow + 16 * ((q + t) & (NCH - 1)));
      __syncwarp();
      if (lane == 0) mbar_arrive(c_empty + 8 * sc);
      uint8_t *arow = sA + sa * A_STAGE + t * 128;
#pragma unroll
      for (int q = 0; q < NCH; ++q) {
        const int cq = (q + t) & (NCH - 1);
        const uint32_t X = (sbytes >> (8 * cq)) & 0xFF;  // scale byte: 2^(X - 127)
        // 2^(X-127) as bf16 (X = 0: the subnormal 2^-127)
        const uint32_t sb = X ? (X << 7) : 0x0040u;
        __nv_bfloat162 s2;
        *reinterpret_cast<uint32_t *>(&s2) = sb | (sb << 16);
        const uint32_t wds[4] = {cw[q].x, cw[q].y, cw[q].z, cw[q].w};
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {  // 8 elements: one 16-byte chunk of the tile
          uint32_t o[4];
#pragma unroll
          for (int by = 0; by < 4; ++by) {
            uint32_t p = lut[(wds[hh] >> (8 * by)) & 0xFF];
            __nv_bfloat162 v = __hmul2(*reinterpret_cast<__nv_bfloat162 *>(&p), s2);
            o[by] = *reinterpret_cast<uint32_t *>(&v);
          }
          const int cc = 4 * cq + hh;  // 16-byte chunk of the bf16 row (0..DI/8-1)
          *reinterpret_cast<uint4 *>(arow + (cc >> 3) * A_ATOM + (((cc & 7) ^ (t & 7)) << 4)) =
              make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
      fence_proxy_async_smem();  // the tile, visible to the tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(a_full + 8 * sa);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  if (tid == 0 && abort_flag) raise_dev_err(kDevErrTimeout);
}

}  // namespace csa
