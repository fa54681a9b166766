// index_score_tc.cuh -- lightning-indexer scores on the 5th-generation tensor
// cores (tcgen05 + TMEM), bf16 inputs, fp32 accumulation.
//
// "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part V", CSA
// bullet: a lightning indexer of 64 heads x 128 dims ranks every compressed
// entry for each query; "The Exchange Rates of a Million Tokens", section 3:
// ReLU-gated dot products.
//     I[t,i] = sum_h w[t,h] * max(0, qI[t,h,:] . kI[i,:])
//
// At decode this is a stream over the whole indexer-key cache (256 B per
// entry) with 64 FLOP per byte: HBM-bound, but past what the CUDA cores can
// multiply at HBM speed, so the contraction runs on the tensor cores:
//   D[128 entries x N heads] = K_tile[128 x dI] . Q[N x dI]^T   (TMEM, fp32)
// and the epilogue reduces each entry's row of D to one score.
//
// Structure: one persistent CTA per SM, 6 warps.
//   warp 0  TMA producer: key tiles (128 x dI bf16, 128-byte swizzle) into an
//           S-stage ring; the query's indexer block into a 2-slot ring
//   warp 1  MMA issuer (one thread): dI/16 tcgen05.mma per tile into one of
//           two TMEM accumulators; commits release the key stage and signal
//           the accumulator
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//           lanes 32*(w%4)..), score = sum_h w_h*max(d_h,0) in fp32, in a
//           fixed head order, coalesced store of 128 scores
// Work: the visible 128-entry tiles of all query units, in order, cut into
// one contiguous range per CTA (so a CTA loads each query block once); every
// role walks the same range.  A unit is one query row at decode; with
// several query rows per sequence (prefill) it is G consecutive rows of one
// sequence, whose G x HI query vectors form one B operand (N = G HI <= 256):
// each key tile is then read once for G rows, and the epilogue produces G
// scores per entry, each masked by its own row's visibility.  Tiles past a
// unit's visible entries are never loaded.  All waits are time-bounded
// (sm100.cuh).
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace csa {

constexpr int kTcRows = 128;      // entries per tile = MMA M
constexpr int kTcThreads = 192;   // producer, MMA, 4 epilogue warps

struct IndexTcArgs {
  const __nv_bfloat16 *w;  // [R][HI]
  const int32_t *lens;
  const int32_t *q_pos;
  float *scores;           // [R][nc_max]
  int Tq, HI, nc_max, R;
  int G, gpb, U;           // rows per unit, units per sequence, units
  int stages;              // depth of the key-tile ring
  int fill_invisible;      // also write -inf past each row's visible entries
};

// visible entries of query row r (0 for an invalid row; the error is raised)
__device__ __forceinline__ int tc_row_visible(const IndexTcArgs &a, int r) {
  int t;
  if (!query_position(a.lens, a.q_pos, r / a.Tq, a.Tq, r % a.Tq, t)) return 0;
  int v = (t + 1) / 4;
  if (v > a.nc_max) {
    raise_dev_err(kDevErrCache);
    v = 0;
  }
  return v;
}

__device__ __forceinline__ int tc_row_tiles(const IndexTcArgs &a, int r) {
  return (tc_row_visible(a, r) + kTcRows - 1) / kTcRows;
}

// first query row and row count of unit u
__device__ __forceinline__ int tc_unit_row0(const IndexTcArgs &a, int u) {
  return (u / a.gpb) * a.Tq + (u % a.gpb) * a.G;
}
__device__ __forceinline__ int tc_unit_rows(const IndexTcArgs &a, int u) {
  return min(a.G, a.Tq - (u % a.gpb) * a.G);
}
// tiles of unit u: the most any of its rows sees
__device__ __forceinline__ int tc_unit_tiles(const IndexTcArgs &a, int u) {
  const int r0 = tc_unit_row0(a, u), n = tc_unit_rows(a, u);
  int t = 0;
  for (int i = 0; i < n; ++i) t = max(t, tc_row_tiles(a, r0 + i));
  return t;
}

// Cursor over a contiguous range of the unit-major list of visible tiles.
struct TileWalk {
  int r, j, tiles, left;  // r: the unit
  __device__ void advance(const IndexTcArgs &a) {
    if (--left <= 0) return;
    if (++j < tiles) return;
    j = 0;
    do {
      ++r;
      tiles = tc_unit_tiles(a, r);
    } while (tiles == 0 && r + 1 < a.U);
  }
};

template <int N1, int G, int DI>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_index_score_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                     IndexTcArgs a) {
  constexpr int N = N1 * G;  // MMA N: G rows' query vectors (N1 heads each)
  using namespace sm100;
  constexpr int KATOMS = DI / 64;                       // 128-byte K slices
  constexpr uint32_t A_ATOM = kTcRows * 128;            // bytes per K slice of a key tile
  constexpr uint32_t A_STAGE = A_ATOM * KATOMS;
  constexpr uint32_t B_ATOM = N * 128;
  constexpr uint32_t B_SLOT = B_ATOM * KATOMS;
  constexpr uint32_t TMEM_COLS = (2 * N <= 32) ? 32 : (2 * N <= 64) ? 64 : (2 * N <= 128) ? 128 : 256;
  constexpr uint32_t IDESC = idesc_bf16_f32(kTcRows, N);

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_holder;
  __shared__ int abort_flag;
  __shared__ int range[3];  // first row, first tile, tile count
  __shared__ int scan[33];
  __shared__ float sw[2][G > 1 ? N : 1];  // grouped units: the G rows' head weights

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = a.stages;
  uint8_t *base = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = base;
  uint8_t *sB = sA + (size_t)S * A_STAGE;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sB + 2 * B_SLOT);
  const uint32_t b_full = smem_u32(bars), b_empty = b_full + 8 * S;
  const uint32_t q_full = b_empty + 8 * S, q_empty = q_full + 16;
  const uint32_t t_full = q_empty + 16, t_empty = t_full + 16, drain = t_empty + 16;
  volatile int *abort = &abort_flag;

  if (tid == 0) {
    abort_flag = 0;
    range[2] = 0;
    for (int s = 0; s < S; ++s) {
      mbar_init(b_full + 8 * s, 1);
      mbar_init(b_empty + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full + 8 * i, 1);
      mbar_init(q_empty + 8 * i, 1);
      mbar_init(t_full + 8 * i, 1);
      mbar_init(t_empty + 8 * i, 4);  // one arrive per epilogue warp
    }
    mbar_init(drain, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmQ);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();  // inputs may come from the previous kernel in the stream
  pdl_launch_dependents();

  // this CTA's contiguous share of the visible tiles
  {
    const int per = (a.U + kTcThreads - 1) / kTcThreads;
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
            tma_load_2d(smem_u32(sB + slot * B_SLOT + ka * B_ATOM), &tmQ, 64 * ka,
                        tc_unit_row0(a, wk.r) * a.HI, q_full + 8 * slot);
          ++nq;
          cur_r = wk.r;
        }
        const uint32_t s = nt % S;
        if (!(ok = mbar_wait(b_empty + 8 * s, ((nt / S) & 1) ^ 1, abort))) break;
        mbar_arrive_expect_tx(b_full + 8 * s, A_STAGE);
        const int y = (wk.r / a.gpb) * a.nc_max + wk.j * kTcRows;
#pragma unroll
        for (int ka = 0; ka < KATOMS; ++ka)
          tma_load_2d_hint(smem_u32(sA + s * A_STAGE + ka * A_ATOM), &tmK, 64 * ka, y, b_full + 8 * s,
                           pol);
        ++nt;
      }
      if (!ok) {
        // drain: wait (bounded) for the copies this thread put in flight
        volatile int no_abort = 0;
        for (uint32_t n = (nt > (uint32_t)S ? nt - S : 0); n < nt; ++n)
          mbar_wait(b_full + 8 * (n % S), (n / S) & 1, &no_abort);
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
          if (cur_r >= 0) umma_commit(q_empty + 8 * slot);  // previous query block free when done
          slot = nq & 1;
          if (!(ok = mbar_wait(q_full + 8 * slot, (nq >> 1) & 1, abort))) break;
          ++nq;
          cur_r = wk.r;
        }
        const uint32_t s = nt % S, acc = nt & 1;
        if (!(ok = mbar_wait(b_full + 8 * s, (nt / S) & 1, abort))) break;
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
        umma_commit(b_empty + 8 * s);   // key stage free once these MMAs finish
        umma_commit(t_full + 8 * acc);  // accumulator ready for the epilogue
        ++nt;
      }
      // every issued MMA complete before TMEM can be released
      umma_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
    const int row = quad * 32 + lane;
    float wv[G == 1 ? N1 : 1];
    int vis[G];
    int cur_u = -1, r0 = 0, nrows = 1, upar = 0;
    uint32_t nt = 0;
    for (; wk.left > 0; wk.advance(a)) {
      if (wk.r != cur_u) {
        cur_u = wk.r;
        r0 = tc_unit_row0(a, cur_u);
        nrows = tc_unit_rows(a, cur_u);
#pragma unroll
        for (int g = 0; g < G; ++g) vis[g] = g < nrows ? tc_row_visible(a, r0 + g) : 0;
        if constexpr (G == 1) {
#pragma unroll
          for (int h = 0; h < N1; ++h)
            wv[h] = h < a.HI ? __bfloat162float(a.w[(size_t)r0 * a.HI + h]) : 0.f;
        } else {
          // the unit's head weights into shared memory (the 4 epilogue warps;
          // two buffers, so the previous unit's may still be read)
          upar ^= 1;
          for (int u = tid - 64; u < N; u += 128) {
            const int g = u / N1, h = u % N1;
            sw[upar][u] = (g < nrows && h < a.HI) ? __bfloat162float(a.w[(size_t)(r0 + g) * a.HI + h]) : 0.f;
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");
        }
      }
      const uint32_t acc = nt & 1;
      // every lane waits; the warp leaves together if any lane timed out, so
      // the .sync.aligned TMEM loads below never see a divergent warp
      const bool ok = mbar_wait(t_full + 8 * acc, (nt >> 1) & 1, abort);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + acc * N;
      const int i = wk.j * kTcRows + row;
      if constexpr (G == 1) {
        uint32_t d[N1];
#pragma unroll
        for (int c = 0; c < N1 / 16; ++c) tmem_ld16(taddr + 16 * c, d + 16 * c);
        tmem_wait_ld_regs<N1>(d);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(t_empty + 8 * acc);
        float sc = 0.f;
#pragma unroll
        for (int h = 0; h < N1; ++h) sc = fmaf(wv[h], fmaxf(__uint_as_float(d[h]), 0.f), sc);
        if (i < a.nc_max) a.scores[(size_t)r0 * a.nc_max + i] = i < vis[0] ? sc : -INFINITY;
      } else {
        const float *wu = sw[upar];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          uint32_t d[N1];
#pragma unroll
          for (int c = 0; c < N1 / 16; ++c) tmem_ld16(taddr + g * N1 + 16 * c, d + 16 * c);
          tmem_wait_ld_regs<N1>(d);
          float sc = 0.f;
#pragma unroll
          for (int h = 0; h < N1; ++h) sc = fmaf(wu[g * N1 + h], fmaxf(__uint_as_float(d[h]), 0.f), sc);
          if (g < nrows && i < a.nc_max) {
            if (i < vis[g]) a.scores[(size_t)(r0 + g) * a.nc_max + i] = sc;
            else if (a.fill_invisible) a.scores[(size_t)(r0 + g) * a.nc_max + i] = -INFINITY;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(t_empty + 8 * acc);
      }
      ++nt;
    }
    // -inf past each row's visible tiles (rows split over the CTAs)
    if (a.fill_invisible) {
      const int et = tid - 64;
      for (int r = blockIdx.x; r < a.R; r += gridDim.x) {
        const int from = tc_row_tiles(a, r) * kTcRows;
        for (int i = from + et; i < a.nc_max; i += 128) a.scores[(size_t)r * a.nc_max + i] = -INFINITY;
      }
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
