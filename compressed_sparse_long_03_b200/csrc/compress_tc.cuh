// compress_tc.cuh -- the CSA and HCA compressors on the tcgen05 tensor cores
// (bf16 tokens and parameters, fp32 logits and pooling, d in {64, 128}).
//
// "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part V",
// "The attention: compress, then select": every 4 tokens (CSA) or 128 tokens
// (HCA) become one entry, a learned softmax-weighted pooling computed per
// channel with learned position biases; a CSA entry pools its own block and
// the previous one.  "The Exchange Rates of a Million Tokens", section 3: the
// two overlapping series share one joint softmax.
//     z_s[c] = (x_s . W)[c] + bias[slot(s)][c],   C_i[c] = sum_s softmax_s(z[c]) x_s[c]
// (CSA: W = W_a for the previous block, W_b for the own block.)
//
// The logit contraction is d x d per token per series -- 137 GFLOP for the
// 32 x 131,072-token HCA workload -- which the CUDA cores cannot do at HBM
// speed; on the tensor cores the kernel streams the tokens at HBM speed.
// The contraction is computed transposed, Z^T = W^T X^T (M = 128 channel
// lanes, N = the tile's tokens, K = d), so that TMEM lane c holds channel c
// for every token of the tile and one epilogue thread owns one channel: the
// per-channel softmax over an entry's tokens is a per-thread loop, and the
// token values x_s[c] come from the same shared-memory tile the MMA read.
//
// Structure: one persistent CTA per SM, 10 warps.
//   warp 0  TMA producer: token tiles (rows x d bf16, 128-byte swizzle) into
//           an S-stage ring; a stage is freed by the epilogue (it reads x)
//   warp 1  MMA issuer: D/16 tcgen05.mma per series into TMEM
//   warps 2-9  epilogue, two warps per TMEM lane quadrant: thread (c, half)
//           owns channel c (TMEM lane c) for one half of the tile's tokens:
//           logits from TMEM, bias, masked softmax per entry (base 2),
//           pooled sum, bf16 store (coalesced over channels); an entry that
//           spans both halves merges the halves' (max, sum, pooled sum)
//           through shared memory
// W^T is staged once per CTA (K-major, swizzled; lanes >= d are zero); the
// HCA bias for strides up to 128, times log2(e), sits in TMEM next to the
// accumulators (lane c, one column per position), so the epilogue reads it
// with the logits.
// Work units (round-robin over CTAs):
//   CSA  32 entries = 128 own tokens, plus a 16-token halo before them (the
//        previous block of the first entry), N = 144; series a and b
//   HCA  m in {32, 64}: one 128-token tile of 128/m entries;
//        m a multiple of 128: one entry of m/128 tiles (online softmax)
// All waits are time-bounded (sm100.cuh).
#pragma once

#include <type_traits>

#include "common.cuh"
#include "sm100.cuh"

namespace csa {

constexpr int kCtThreads = 320;  // producer, MMA, 8 epilogue warps
constexpr int kCtEpi = 8;        // epilogue warps
constexpr int kCtHalo = 16;

struct CompressTcArgs {
  const __nv_bfloat16 *Wa;    // [d][d], [in][out] (HCA: W)
  const __nv_bfloat16 *Wb;    // [d][d] (CSA only)
  const __nv_bfloat16 *bias;  // CSA [8][d]; HCA [m][d]
  const int32_t *lens;
  __nv_bfloat16 *out;  // [B][nc_max][d]
  int n_max, nc_max, m;
  int units, per_seq;  // work units, units per sequence
  int stages;
};

// HCA compressors on the tensor cores need every 32-token chunk inside one
// entry and tiles that do not straddle entries.
__host__ __device__ constexpr bool hca_tc_stride_ok(int m) {
  return m == 32 || m == 64 || (m >= 128 && m % 128 == 0);
}

template <bool CSA, int D>
__global__ void __launch_bounds__(kCtThreads, 1)
    k_compress_tc(const __grid_constant__ CUtensorMap tmX, CompressTcArgs a) {
  using namespace sm100;
  constexpr int NSER = CSA ? 2 : 1;
  constexpr int NTOK = CSA ? 128 + kCtHalo : 128;  // rows of a token tile (MMA N)
  constexpr int KATOMS = D / 64;
  constexpr uint32_t A_ATOM = 128 * 128;            // 128 lanes x 128 B
  constexpr uint32_t A_SER = A_ATOM * KATOMS;
  constexpr uint32_t X_ATOM = NTOK * 128;
  constexpr uint32_t X_STAGE = X_ATOM * KATOMS;
  constexpr int NB = CSA ? 1 : 2;                       // TMEM accumulator buffers
  constexpr uint32_t SER_COL = CSA ? 256 : 0;           // column offset of series b
  constexpr uint32_t BUF_COL = CSA ? 0 : 128;           // column offset of buffer 1
  constexpr uint32_t TMEM_COLS = 512;
  constexpr uint32_t BIAS_COL = 256;                    // HCA: bias columns (m <= 128)
  constexpr uint32_t IDESC = idesc_bf16_f32(128, NTOK);
  constexpr float kLog2e = 1.4426950408889634f;

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_holder;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = a.stages;
  uint8_t *base = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = base;                   // NSER x [KATOMS][128 lanes][128 B]
  uint8_t *sX = sA + NSER * A_SER;      // S x [KATOMS][NTOK rows][128 B]
  uint64_t *bars = reinterpret_cast<uint64_t *>(sX + (size_t)S * X_STAGE);
  const uint32_t x_full = smem_u32(bars), x_empty = x_full + 8 * S;
  const uint32_t t_full = x_empty + 8 * S, t_empty = t_full + 8 * NB, drain = t_empty + 8 * NB;
  volatile int *abort = &abort_flag;
  const int tiles_per_unit = (!CSA && a.m > 128) ? a.m / 128 : 1;

  if (tid == 0) {
    abort_flag = 0;
    for (int s = 0; s < S; ++s) {
      mbar_init(x_full + 8 * s, 1);
      mbar_init(x_empty + 8 * s, kCtEpi);  // one arrive per epilogue warp
    }
    for (int i = 0; i < NB; ++i) {
      mbar_init(t_full + 8 * i, 1);
      mbar_init(t_empty + 8 * i, kCtEpi);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();  // tokens and parameters may come from the previous kernel
  pdl_launch_dependents();

  // W^T into the A operand: lane (output channel) o, column (input channel)
  // k holds W[k][o]; 16-byte chunks XOR-swizzled by the lane; lanes >= D zero
  for (int u = tid; u < NSER * (int)(A_SER / 16); u += kCtThreads)
    reinterpret_cast<uint4 *>(sA)[u] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  // W as stored ([in][out], 16-byte copies) into the still unused token
  // stages, then transposed in shared memory: thread (o, kc) gathers inputs
  // 8kc..8kc+7 of output o into one 16-byte chunk (the swizzle spreads 8
  // consecutive lanes over all banks)
  uint16_t *wtmp = reinterpret_cast<uint16_t *>(sX);
  for (int u = tid; u < NSER * D * D / 8; u += kCtThreads) {
    const int ser = u / (D * D / 8), rem = u % (D * D / 8);
    cp_async16(smem_u32(wtmp) + 16 * u, (ser ? a.Wb : a.Wa) + 8 * rem, 16u);
  }
  cp_async_wait_all();
  __syncthreads();
  for (int u = tid; u < NSER * D * (D / 8); u += kCtThreads) {
    const int ser = u / (D * (D / 8)), rem = u % (D * (D / 8));
    const int o = rem % D, kc = rem / D;
    const uint16_t *Ws = wtmp + ser * D * D;
    uint32_t pk[4];
#pragma unroll
    for (int t = 0; t < 4; ++t)
      pk[t] = (uint32_t)Ws[(8 * kc + 2 * t) * D + o] | ((uint32_t)Ws[(8 * kc + 2 * t + 1) * D + o] << 16);
    uint8_t *at = sA + ser * A_SER + (kc >> 3) * A_ATOM + o * 128 + (((kc & 7) ^ (o & 7)) << 4);
    *reinterpret_cast<uint4 *>(at) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t nt = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < a.units && ok; u += gridDim.x) {
        const int b = u / a.per_seq, t = u % a.per_seq;
        for (int jt = 0; jt < tiles_per_unit && ok; ++jt, ++nt) {
          long tok0;
          if (CSA) tok0 = 128L * t - kCtHalo;
          else if (a.m > 128) tok0 = (long)a.m * t + 128L * jt;
          else tok0 = 128L * t;
          const uint32_t s = nt % S;
          if (!(ok = mbar_wait(x_empty + 8 * s, ((nt / S) & 1) ^ 1, abort))) break;
          mbar_arrive_expect_tx(x_full + 8 * s, X_STAGE);
          const int row = (int)((long)b * a.n_max + tok0);  // may be negative: zero fill
#pragma unroll
          for (int ka = 0; ka < KATOMS; ++ka)
            tma_load_2d(smem_u32(sX + s * X_STAGE + ka * X_ATOM), &tmX, 64 * ka, row, x_full + 8 * s);
        }
      }
      if (!ok) {
        volatile int no_abort = 0;
        for (uint32_t n = (nt > (uint32_t)S ? nt - S : 0); n < nt; ++n)
          mbar_wait(x_full + 8 * (n % S), (n / S) & 1, &no_abort);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      uint32_t nt = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < a.units && ok; u += gridDim.x) {
        for (int jt = 0; jt < tiles_per_unit; ++jt, ++nt) {
          const uint32_t s = nt % S, buf = nt % NB;
          if (!(ok = mbar_wait(x_full + 8 * s, (nt / S) & 1, abort))) break;
          if (!(ok = mbar_wait(t_empty + 8 * buf, ((nt / NB) & 1) ^ 1, abort))) break;
          tc_fence_after();
          const uint32_t x0 = smem_u32(sX + s * X_STAGE);
#pragma unroll
          for (int ser = 0; ser < NSER; ++ser) {
            const uint32_t d = tmem + buf * BUF_COL + ser * SER_COL;
            const uint32_t a0 = smem_u32(sA + ser * A_SER);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint32_t aoff = (k >> 2) * A_ATOM + (k & 3) * 32;
              const uint32_t xoff = (k >> 2) * X_ATOM + (k & 3) * 32;
              umma_bf16(d, sdesc_kmajor_sw128(a0 + aoff), sdesc_kmajor_sw128(x0 + xoff), IDESC, k > 0);
            }
          }
          umma_commit(t_full + 8 * buf);
        }
      }
      umma_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3, half = (warp - 2) >> 2;
    const int c = quad * 32 + lane;          // channel = TMEM lane
    const bool live = quad * 32 < D;         // warp-uniform
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const int catom = (c & 63) >> 3, cwithin = (c & 7) * 2;
    float bias8[8];  // CSA biases times log2(e)
    if (CSA) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        bias8[j] = live ? __bfloat162float(a.bias[j * D + (c & (D - 1))]) * kLog2e : 0.f;
    }
    // x_s[c] of tile row r: row base + the swizzled chunk, which depends on
    // r % 8 only (tables of the 8 offsets; callers index them with constants)
    uint32_t swz[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) swz[k] = ((uint32_t)(catom ^ k) << 4) + (uint32_t)cwithin + (c >> 6) * X_ATOM;
    if (!CSA && a.m <= 128) {
      // bias[pos][c] * log2(e) into TMEM lane c, column BIAS_COL + pos; each
      // half writes half of the m positions
      if (live) {
        const int h0 = half * (a.m / 2);
        for (int p0 = h0; p0 < h0 + a.m / 2; p0 += 16) {
          uint32_t bv[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            bv[e] = __float_as_uint(__bfloat162float(a.bias[(size_t)(p0 + e) * D + c]) * kLog2e);
          tmem_st16(tmem + lane_off + BIAS_COL + p0, bv);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      asm volatile("bar.sync 1, %0;" ::"r"(kCtEpi * 32) : "memory");
      tc_fence_after();
    }
    auto xat = [&](const uint8_t *rowbase, int k) -> float {  // rowbase: row r's start, k = r % 8
      return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(rowbase + swz[k]));
    };
    // half 1's state of an entry that spans both halves, by entry parity
    __shared__ float xch[2][3][128];
    uint32_t nt = 0, nx = 0;
    bool alive = true;
    // HCA online state of the current entry (this half's tokens)
    float run_max = -INFINITY, den = 0.f, num = 0.f;
    // the next unit's sequence length is loaded one unit ahead
    int n_next = blockIdx.x < a.units ? __ldg(a.lens + blockIdx.x / a.per_seq) : 0;
    for (int u = blockIdx.x; u < a.units && alive; u += gridDim.x) {
      const int b = u / a.per_seq, t = u % a.per_seq;
      int n = n_next;
      if (u + (int)gridDim.x < a.units) n_next = __ldg(a.lens + (u + (int)gridDim.x) / a.per_seq);
      if (n < 0 || n > a.n_max) {
        if (t == 0 && c == 0 && half == 0) raise_dev_err(kDevErrLen);
        n = 0;
      }
      for (int jt = 0; jt < tiles_per_unit; ++jt, ++nt) {
        const uint32_t s = nt % S, buf = nt % NB;
        const bool ok = mbar_wait(t_full + 8 * buf, (nt / NB) & 1, abort);
        if (!__all_sync(0xffffffffu, ok)) {
          alive = false;
          break;
        }
        tc_fence_after();
        const uint32_t tb = tmem + lane_off + buf * BUF_COL;
        bool merge = false;  // an entry spanning both halves ends with this tile
        int merge_i = 0;
        if (CSA) {
          const long tok0 = 128L * t - kCtHalo;
          const int nc = (n + 3) / 4;
#pragma unroll 1
          for (int p = 2 * half; p < 2 * half + 2; ++p) {  // 8 entries per pass
            uint32_t za[48], zb[32];
            if (live) {
              tmem_ld16(tb + 32 * p, za);
              tmem_ld16(tb + 32 * p + 16, za + 16);
              tmem_ld16(tb + 32 * p + 32, za + 32);
              tmem_ld16(tb + SER_COL + 32 * p + 16, zb);
              tmem_ld16(tb + SER_COL + 32 * p + 32, zb + 16);
              tmem_wait_ld_regs<48>(za);
              tmem_wait_ld_regs<32>(zb);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const int i = 32 * t + 8 * p + q;
                if (i >= a.nc_max) break;
                float z[8];
                bool v[8];
                float mx = -INFINITY;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  const long sidx = tok0 + 12 + 32 * p + 4 * q + j;  // token of slot j
                  v[j] = i < nc && sidx >= 0 && sidx < n;
                  const float zz = j < 4 ? __uint_as_float(za[12 + 4 * q + j])
                                         : __uint_as_float(zb[4 * q + j - 4]);
                  z[j] = fmaf(zz, kLog2e, bias8[j]);
                  if (v[j]) mx = fmaxf(mx, z[j]);
                }
                float dsum = 0.f, nsum = 0.f;
                // tile row 12 + 32p + 4q + j: its r % 8 is (4 + 4q + j) % 8
                const uint8_t *rb = sX + s * X_STAGE + (12 + 32 * p + 4 * q) * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  if (!v[j]) continue;
                  const float pw = ex2(z[j] - mx);
                  dsum += pw;
                  nsum = fmaf(pw, xat(rb + j * 128, (4 + 4 * q + j) & 7), nsum);
                }
                const float res = dsum > 0.f ? nsum / dsum : 0.f;
                a.out[((size_t)b * a.nc_max + i) * D + c] = __float2bfloat16_rn(res);
              }
            }
          }
        } else {
          const int m = a.m;
          const long tok0 = (m > 128) ? (long)m * t + 128L * jt : 128L * t;
          const bool bias_tmem = m <= 128;  // warp-uniform
          // fold G consecutive tokens (tile columns colL.., entry slots pos0..)
          // of one entry into this thread's running (max, sum, pooled sum);
          // lim = how many of them lie inside the sequence
          auto fold = [&](auto Gc, int colL, int pos0, long lim) {
            constexpr int G = decltype(Gc)::value;
            constexpr int NCH = G / 8;  // independent chains
            uint32_t zt[G], bt[G];
#pragma unroll
            for (int q = 0; q < G / 16; ++q) tmem_ld16(tb + colL + 16 * q, zt + 16 * q);
            if (bias_tmem) {
#pragma unroll
              for (int q = 0; q < G / 16; ++q) tmem_ld16(tmem + lane_off + BIAS_COL + pos0 + 16 * q, bt + 16 * q);
            }
            tmem_wait_ld_regs<G>(zt);
            float z[G];
            if (bias_tmem) {
              tmem_wait_ld_regs<G>(bt);
#pragma unroll
              for (int jj = 0; jj < G; ++jj) z[jj] = fmaf(__uint_as_float(zt[jj]), kLog2e, __uint_as_float(bt[jj]));
            } else {
              const __nv_bfloat16 *bp = a.bias + (size_t)pos0 * D + c;
#pragma unroll
              for (int jj = 0; jj < G; ++jj)
                z[jj] = (__uint_as_float(zt[jj]) + __bfloat162float(bp[jj * D])) * kLog2e;
            }
            if (lim < G) {
#pragma unroll
              for (int jj = 0; jj < G; ++jj)
                if (jj >= lim) z[jj] = -INFINITY;
            }
            float cm[NCH];
#pragma unroll
            for (int k = 0; k < NCH; ++k) cm[k] = -INFINITY;
#pragma unroll
            for (int jj = 0; jj < G; ++jj) cm[jj % NCH] = fmaxf(cm[jj % NCH], z[jj]);
#pragma unroll
            for (int k = 1; k < NCH; ++k) cm[0] = fmaxf(cm[0], cm[k]);
            const float nmax = fmaxf(run_max, cm[0]);
            if (nmax == -INFINITY) return;
            const float alpha = ex2(run_max - nmax);  // 0 when run_max is -inf
            // rows colL.. start at a multiple of 32: row % 8 == jj % 8
            const uint8_t *rb = sX + s * X_STAGE + colL * 128;
            float dd[NCH], nn[NCH];
#pragma unroll
            for (int k = 0; k < NCH; ++k) dd[k] = nn[k] = 0.f;
#pragma unroll
            for (int jj = 0; jj < G; ++jj) {
              const float pw = ex2(z[jj] - nmax);  // 0 for masked tokens
              dd[jj % NCH] += pw;
              nn[jj % NCH] = fmaf(pw, xat(rb + jj * 128, jj & 7), nn[jj % NCH]);
            }
#pragma unroll
            for (int k = 1; k < NCH; ++k) {
              dd[0] += dd[k];
              nn[0] += nn[k];
            }
            den = fmaf(den, alpha, dd[0]);
            num = fmaf(num, alpha, nn[0]);
            run_max = nmax;
          };
          auto finish = [&](int i) {
            if (live && i < a.nc_max)
              a.out[((size_t)b * a.nc_max + i) * D + c] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
            run_max = -INFINITY;
            den = 0.f;
            num = 0.f;
          };
          if (m == 32) {  // two entries per half, one chunk each
#pragma unroll 1
            for (int ch = 2 * half; ch < 2 * half + 2; ++ch) {
              const long s0 = tok0 + 32 * ch;
              if (live) fold(std::integral_constant<int, 32>(), 32 * ch, 0, (long)n - s0);
              finish((int)(s0 / 32));
            }
          } else {  // the half's 64 tokens lie inside one entry
            const long s0 = tok0 + 64 * half;
            const int i = (int)(s0 / m);
            const int pos0 = (int)(s0 - (long)m * i);
            if (live) fold(std::integral_constant<int, 64>(), 64 * half, pos0, (long)n - s0);
            if (m == 64) {
              finish(i);
            } else if (pos0 + 64 + (1 - half) * 64 == m) {
              // the entry (both halves) ends with this tile: merge below
              merge = true;
              merge_i = i;
            }
          }
        }
        // TMEM and the token stage are free
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(t_empty + 8 * buf);
          mbar_arrive(x_empty + 8 * s);
        }
        if (merge) {  // uniform over the epilogue warps
          float *xs = &xch[nx & 1][0][0];
          if (half == 1) {
            xs[c] = run_max;
            xs[128 + c] = den;
            xs[256 + c] = num;
          }
          asm volatile("bar.sync 1, %0;" ::"r"(kCtEpi * 32) : "memory");
          if (half == 0 && live && merge_i < a.nc_max) {
            const float m1 = xs[c], d1 = xs[128 + c], n1 = xs[256 + c];
            const float M = fmaxf(run_max, m1);
            float dd = 0.f, nn = 0.f;
            if (M != -INFINITY) {
              const float w0 = ex2(run_max - M), w1 = ex2(m1 - M);
              dd = den * w0 + d1 * w1;
              nn = num * w0 + n1 * w1;
            }
            a.out[((size_t)b * a.nc_max + merge_i) * D + c] = __float2bfloat16_rn(dd > 0.f ? nn / dd : 0.f);
          }
          ++nx;
          run_max = -INFINITY;
          den = 0.f;
          num = 0.f;
        }
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
