// csa_api.cu -- the C ABI (include/csa.h): host-side validation, launch
// configuration and error reporting for the CSA / HCA kernels.
//
// The whole library is this one translation unit: every kernel header is
// included here, so the device error word has one definition and no device
// linking is needed.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <type_traits>
#include <mutex>
#include <string>
#include <unordered_map>
#include <vector>

#include "csa.h"

#include "common.cuh"
#include "compress.cuh"
#include "compress_tc.cuh"
#include "compress_step.cuh"
#include "mxfp4.cuh"
#include "index_score_fma.cuh"
#include "index_score_tc.cuh"
#include "topk.cuh"
#include "attend_fma.cuh"
#include "attend_tc.cuh"
#include "fp8.cuh"
#include "rope.cuh"

namespace {

thread_local std::string g_last_error;

int fail(int code, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------------------
// optional per-kernel timing (csa_set_kernel_timing): CUDA events recorded
// on the call's stream around every kernel the call launches
// ---------------------------------------------------------------------------
struct TimingSlot {
  cudaEvent_t a = nullptr, b = nullptr;
  int dev = -1;
};
thread_local bool g_timing = false;
// CTAs of the persistent scoring kernel (0: one per SM); the layer-pair
// step lowers it to leave SMs to the HCA attention running beside it
thread_local int g_score_ctas = 0;
thread_local std::vector<TimingSlot> g_slots;
thread_local int g_nlaunch = 0;

void begin_call() { g_nlaunch = 0; }

struct KernelTimer {
  cudaStream_t st;
  int slot = -1;
  explicit KernelTimer(cudaStream_t s) : st(s) {
    if (!g_timing) return;
    int dev = 0;
    cudaGetDevice(&dev);
    if ((int)g_slots.size() <= g_nlaunch) g_slots.resize(g_nlaunch + 1);
    TimingSlot &ts = g_slots[g_nlaunch];
    if (ts.dev != dev) {
      if (ts.a) cudaEventDestroy(ts.a);
      if (ts.b) cudaEventDestroy(ts.b);
      cudaEventCreate(&ts.a);
      cudaEventCreate(&ts.b);
      ts.dev = dev;
    }
    slot = g_nlaunch++;
    cudaEventRecord(ts.a, st);
  }
  ~KernelTimer() {
    if (slot >= 0) cudaEventRecord(g_slots[slot].b, st);
  }
};

int launch_status(const char *what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(CSA_ERR_LAUNCH, "%s: launch failed: %s", what, cudaGetErrorString(e));
  return CSA_OK;
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device).
// Applied whenever dynamic memory is used: static plus dynamic shared memory
// above 48 KB needs the opt-in even when the dynamic part alone is smaller.
std::mutex g_attr_mu;
std::unordered_map<std::string, size_t> g_attr_done;

template <typename K>
int ensure_smem(K kernel, size_t bytes, const char *what) {
  if (bytes == 0) return CSA_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(CSA_ERR_CUDA, "%s: cudaGetDevice failed", what);
  char key[64];
  snprintf(key, sizeof(key), "%p/%d", reinterpret_cast<const void *>(kernel), dev);
  std::lock_guard<std::mutex> lk(g_attr_mu);
  auto it = g_attr_done.find(key);
  if (it != g_attr_done.end() && it->second >= bytes) return CSA_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess)
    return fail(CSA_ERR_CUDA, "%s: cannot reserve %zu B of shared memory: %s", what, bytes,
                cudaGetErrorString(e));
  g_attr_done[key] = bytes;
  return CSA_OK;
}

// Launch `kernel` on a 1-D grid of clusters of `cs` CTAs (cs == 1: a plain
// launch).
// The tensor-core path's kernels are launched with programmatic stream
// serialisation (they start early and wait in-kernel for their predecessor).
template <typename... KArgs, typename... Args>
int launch_cluster(void (*kernel)(KArgs...), int cs, unsigned grid, unsigned block, size_t smem,
                   cudaStream_t stream, const char *what, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(block, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cs > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cs;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  KernelTimer timer(stream);
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(CSA_ERR_LAUNCH, "%s: launch failed: %s", what, cudaGetErrorString(e));
  }
  return CSA_OK;
}

// Number of SMs of the current device (cached per device).
int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

// cuTensorMapEncodeTiled, fetched from the driver through the runtime (no
// link-time dependency on libcuda).
typedef CUresult (*encode_tiled_fn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                    const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                    const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

encode_tiled_fn get_encode_tiled() {
  static encode_tiled_fn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<encode_tiled_fn>(p);
  });
  return fn;
}

// 2-D bf16 tensor [outer][inner] (row-major), box [box_outer][box_inner],
// 128-byte swizzle, zero fill outside the tensor.
int encode_bf16_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                   uint32_t box_inner, uint32_t box_outer, const char *what) {
  encode_tiled_fn enc = get_encode_tiled();
  if (!enc) return fail(CSA_ERR_CUDA, "%s: cuTensorMapEncodeTiled is unavailable", what);
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSA_ERR_CUDA, "%s: tensor map encoding failed (%d)", what, (int)r);
  return CSA_OK;
}

// 2-D byte tensor [outer][inner], box [box_outer][box_inner], no swizzle.
int encode_u8_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                 uint32_t box_outer, const char *what) {
  encode_tiled_fn enc = get_encode_tiled();
  if (!enc) return fail(CSA_ERR_CUDA, "%s: cuTensorMapEncodeTiled is unavailable", what);
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSA_ERR_CUDA, "%s: tensor map encoding failed (%d)", what, (int)r);
  return CSA_OK;
}

int check_dtype(csa_dtype dt, const char *what) {
  if (dt != CSA_F32 && dt != CSA_BF16) return fail(CSA_ERR_DTYPE, "%s: unknown dtype %d", what, (int)dt);
  return CSA_OK;
}

constexpr int kMaxIndexEntries = csa::kTopkMaxCluster * csa::kTopkSliceCap;  // 327680

int topk_cluster_size(int nc_max) {
  int cs = 1;
  while (cs < csa::kTopkMaxCluster && (long)cs * 8192 < nc_max) cs *= 2;
  while ((long)cs * csa::kTopkSliceCap < nc_max) cs *= 2;  // never beyond the cap (validated)
  return cs;
}

int attend_cluster_size(long max_keys) {
  int cs = 1;
  while (cs < 8 && (long)cs * 64 * 2 <= max_keys) cs *= 2;
  return cs;
}

// ---------------------------------------------------------------------------
// compressors
// ---------------------------------------------------------------------------
// bf16 compressors with d in {64, 128} (HCA: strides that keep 32-token
// chunks inside one entry) run on the tensor cores.
template <bool CSA, int D>
int launch_compress_tc(const void *x, const int32_t *lens, int B, int n_max, int m, const void *Wa,
                       const void *Wb, const void *bias, void *out, int nc_max, cudaStream_t st,
                       const char *what) {
  constexpr int NTOK = CSA ? 128 + csa::kCtHalo : 128;
  constexpr size_t A_SER = (size_t)(D / 64) * 128 * 128, X_STAGE = (size_t)(D / 64) * NTOK * 128;
  constexpr int NSER = CSA ? 2 : 1, NB = CSA ? 1 : 2;
  if (nc_max == 0 || B == 0) return CSA_OK;
  CUtensorMap tmX;
  int rc = encode_bf16_2d(&tmX, x, D, (uint64_t)B * n_max, 64, NTOK, what);
  if (rc) return rc;
  // the token stages also hold W while it is transposed
  const size_t budget = 227 * 1024 - 1024 - NSER * A_SER - 4096;
  const int stages = (int)std::min<size_t>(5, budget / X_STAGE);
  if ((size_t)stages * X_STAGE < NSER * (size_t)D * D * 2)
    return fail(CSA_ERR_UNSUPPORTED, "%s: shared memory too small", what);
  const size_t smem = 1024 + NSER * A_SER + stages * X_STAGE + 8 * (2 * stages + 2 * NB + 1);
  auto kern = csa::k_compress_tc<CSA, D>;
  rc = ensure_smem(kern, smem, what);
  if (rc) return rc;
  csa::CompressTcArgs a;
  a.Wa = static_cast<const __nv_bfloat16 *>(Wa);
  a.Wb = static_cast<const __nv_bfloat16 *>(Wb);
  a.bias = static_cast<const __nv_bfloat16 *>(bias);
  a.lens = lens;
  a.out = static_cast<__nv_bfloat16 *>(out);
  a.n_max = n_max;
  a.nc_max = nc_max;
  a.m = m;
  if (CSA) a.per_seq = (nc_max + 31) / 32;
  else if (m > 128) a.per_seq = nc_max;
  else a.per_seq = (int)(((long)nc_max * m + 127) / 128);
  a.units = B * a.per_seq;
  a.stages = stages;
  const unsigned grid = (unsigned)std::min(a.units, num_sms());
  return launch_cluster(kern, 1, grid, csa::kCtThreads, smem, st, what, tmX, a);
}

// decode-time compressors: grid = sequences, block = channels
template <typename T, int D>
int launch_compress_step(bool is_csa, const void *tok, int n_tok, const int32_t *lens, int B, int m,
                         const void *Wa, const void *Wb, const void *bias, void *cache, int nc_max,
                         cudaStream_t st, const char *what) {
  auto X = static_cast<const T *>(tok);
  auto A = static_cast<const T *>(Wa);
  auto Z = static_cast<const T *>(bias);
  auto O = static_cast<T *>(cache);
  if (is_csa)
    return launch_cluster(csa::k_csa_compress_step<T, D>, 1, (unsigned)B, D, 0, st, what, X, n_tok,
                          lens, A, static_cast<const T *>(Wb), Z, O, nc_max);
  return launch_cluster(csa::k_hca_compress_step<T, D>, csa::kStepCluster, (unsigned)B * csa::kStepCluster,
                        D, 0, st, what, X, n_tok, lens, m, A, Z, O, nc_max);
}

template <typename T>
int compress_step_d(bool is_csa, const void *tok, int n_tok, const int32_t *lens, int B, int d, int m,
                    const void *Wa, const void *Wb, const void *bias, void *cache, int nc_max,
                    cudaStream_t st, const char *what) {
  switch (d) {
    case 32: return launch_compress_step<T, 32>(is_csa, tok, n_tok, lens, B, m, Wa, Wb, bias, cache, nc_max, st, what);
    case 64: return launch_compress_step<T, 64>(is_csa, tok, n_tok, lens, B, m, Wa, Wb, bias, cache, nc_max, st, what);
    default: return launch_compress_step<T, 128>(is_csa, tok, n_tok, lens, B, m, Wa, Wb, bias, cache, nc_max, st, what);
  }
}

template <typename T>
int launch_csa_compress(const void *x, const int32_t *lens, int B, int n_max, int d, const void *Wa,
                        const void *Wb, const void *b8, void *out, cudaStream_t st) {
  const int nc_max = (n_max + 3) / 4;
  const bool tc_rows_ok = (long)B * n_max < (1L << 30);  // TMA row coordinates fit in int32
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    if (d == 64 && tc_rows_ok) return launch_compress_tc<true, 64>(x, lens, B, n_max, 4, Wa, Wb, b8, out, nc_max, st, "csa_compress");
    if (d == 128 && tc_rows_ok) return launch_compress_tc<true, 128>(x, lens, B, n_max, 4, Wa, Wb, b8, out, nc_max, st, "csa_compress");
  }
  dim3 grid((nc_max + csa::kCsaEntries - 1) / csa::kCsaEntries, B);
  auto X = static_cast<const T *>(x);
  auto A = static_cast<const T *>(Wa);
  auto Bw = static_cast<const T *>(Wb);
  auto Z = static_cast<const T *>(b8);
  auto O = static_cast<T *>(out);
  KernelTimer timer(st);
  switch (d) {
    case 32: csa::k_csa_compress<T, 32><<<grid, 32, 0, st>>>(X, lens, n_max, A, Bw, Z, O, nc_max); break;
    case 64: csa::k_csa_compress<T, 64><<<grid, 64, 0, st>>>(X, lens, n_max, A, Bw, Z, O, nc_max); break;
    default: csa::k_csa_compress<T, 128><<<grid, 128, 0, st>>>(X, lens, n_max, A, Bw, Z, O, nc_max); break;
  }
  return launch_status("csa_compress");
}

template <typename T>
int launch_hca_compress(const void *x, const int32_t *lens, int B, int n_max, int d, int m,
                        const void *W, const void *bias, void *out, cudaStream_t st) {
  const int nc_max = (int)(((long)n_max + m - 1) / m);
  const bool tc_ok = csa::hca_tc_stride_ok(m) && (long)B * n_max < (1L << 30);
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    if (tc_ok && d == 64)
      return launch_compress_tc<false, 64>(x, lens, B, n_max, m, W, nullptr, bias, out, nc_max, st, "hca_compress");
    if (tc_ok && d == 128)
      return launch_compress_tc<false, 128>(x, lens, B, n_max, m, W, nullptr, bias, out, nc_max, st, "hca_compress");
  }
  dim3 grid(nc_max, B);
  auto X = static_cast<const T *>(x);
  auto Wp = static_cast<const T *>(W);
  auto Z = static_cast<const T *>(bias);
  auto O = static_cast<T *>(out);
  KernelTimer timer(st);
  switch (d) {
    case 32: csa::k_hca_compress<T, 32><<<grid, 32, 0, st>>>(X, lens, n_max, m, Wp, Z, O, nc_max); break;
    case 64: csa::k_hca_compress<T, 64><<<grid, 64, 0, st>>>(X, lens, n_max, m, Wp, Z, O, nc_max); break;
    default: csa::k_hca_compress<T, 128><<<grid, 128, 0, st>>>(X, lens, n_max, m, Wp, Z, O, nc_max); break;
  }
  return launch_status("hca_compress");
}

// ---------------------------------------------------------------------------
// indexer scores + top-k
// ---------------------------------------------------------------------------
template <typename T, int DI>
int launch_index_fma(const void *qI, const void *w, const void *kI, const int32_t *lens,
                     const int32_t *q_pos, int R, int Tq, int HI, int nc_max, float *scores,
                     cudaStream_t st) {
  const int tiles = (nc_max + csa::kIdxFmaTile - 1) / csa::kIdxFmaTile;
  const size_t smem = sizeof(float) * ((size_t)HI * DI + ((HI + 3) & ~3) +
                                       (size_t)csa::kIdxFmaTile * (DI + 1));
  auto kern = csa::k_index_score_fma<T, DI>;
  int rc = ensure_smem(kern, smem, "csa_index_topk");
  if (rc) return rc;
  dim3 grid(tiles, R);
  KernelTimer timer(st);
  kern<<<grid, csa::kIdxFmaTile, smem, st>>>(static_cast<const T *>(qI), static_cast<const T *>(w),
                                             static_cast<const T *>(kI), lens, q_pos, Tq, HI,
                                             nc_max, scores);
  return launch_status("csa_index_topk (scores)");
}

// The tensor-core scoring kernel with G query rows per unit (N1 head slots
// each; N1 * G <= 256).
template <int N1, int G, int DI>
int launch_index_tc(const void *qI, const void *w, const void *kI, const int32_t *lens,
                    const int32_t *q_pos, int R, int Tq, int HI, int nc_max, float *scores,
                    bool fill, cudaStream_t st) {
  constexpr int N = N1 * G;
  const char *what = "csa_index_scores";
  CUtensorMap tmK, tmQ;
  const int B = R / Tq;
  int rc = encode_bf16_2d(&tmK, kI, DI, (uint64_t)B * nc_max, 64, csa::kTcRows, what);
  if (rc) return rc;
  rc = encode_bf16_2d(&tmQ, qI, DI, (uint64_t)R * HI, 64, N, what);
  if (rc) return rc;
  constexpr size_t A_STAGE = (size_t)csa::kTcRows * DI * 2, B_SLOT = (size_t)N * DI * 2;
  const size_t budget = 227 * 1024 - 1024 - 2 * B_SLOT - 1024 - (G > 1 ? 2 * N * 4 : 0);
  const int stages = (int)std::min<size_t>(5, budget / A_STAGE);
  const size_t smem = 1024 + stages * A_STAGE + 2 * B_SLOT + 8 * (2 * stages + 9);
  auto kern = csa::k_index_score_tc<N1, G, DI>;
  rc = ensure_smem(kern, smem, what);
  if (rc) return rc;
  csa::IndexTcArgs a;
  a.w = static_cast<const __nv_bfloat16 *>(w);
  a.lens = lens;
  a.q_pos = q_pos;
  a.scores = scores;
  a.Tq = Tq;
  a.HI = HI;
  a.nc_max = nc_max;
  a.R = R;
  a.G = G;
  a.gpb = (Tq + G - 1) / G;
  a.U = B * a.gpb;
  a.stages = stages;
  a.fill_invisible = fill ? 1 : 0;
  const int ctas = g_score_ctas > 0 ? std::min(g_score_ctas, num_sms()) : num_sms();
  return launch_cluster(kern, 1, (unsigned)ctas, csa::kTcThreads, smem, st, what, tmK, tmQ, a);
}

// Decode (one query row per sequence): one row per unit, the heads padded to
// a power of two.  Several rows per sequence with HI a power of two from 16
// to 128: units of G rows sharing each key tile (N = G HI = 256, or 64 for
// HI = 16).
template <int DI>
int launch_index_tc_n(const void *qI, const void *w, const void *kI, const int32_t *lens,
                      const int32_t *q_pos, int R, int Tq, int HI, int nc_max, float *scores,
                      bool fill, cudaStream_t st) {
  if (Tq >= 2) {
    switch (HI) {
      case 16: return launch_index_tc<16, 4, DI>(qI, w, kI, lens, q_pos, R, Tq, HI, nc_max, scores, fill, st);
      case 32: return launch_index_tc<32, 4, DI>(qI, w, kI, lens, q_pos, R, Tq, HI, nc_max, scores, fill, st);
      case 64: return launch_index_tc<64, 4, DI>(qI, w, kI, lens, q_pos, R, Tq, HI, nc_max, scores, fill, st);
      case 128: return launch_index_tc<128, 2, DI>(qI, w, kI, lens, q_pos, R, Tq, HI, nc_max, scores, fill, st);
      default: break;
    }
  }
  if (HI <= 16) return launch_index_tc<16, 1, DI>(qI, w, kI, lens, q_pos, R, Tq, HI, nc_max, scores, fill, st);
  if (HI <= 32) return launch_index_tc<32, 1, DI>(qI, w, kI, lens, q_pos, R, Tq, HI, nc_max, scores, fill, st);
  if (HI <= 64) return launch_index_tc<64, 1, DI>(qI, w, kI, lens, q_pos, R, Tq, HI, nc_max, scores, fill, st);
  return launch_index_tc<128, 1, DI>(qI, w, kI, lens, q_pos, R, Tq, HI, nc_max, scores, fill, st);
}

// Indexer scores over an MXFP4 key cache (one query row per unit).
template <int N, int DI>
int launch_index_fp4(const void *qI, const void *w, const uint8_t *codes, const uint8_t *scales,
                     const int32_t *lens, const int32_t *q_pos, int R, int Tq, int HI, int nc_max,
                     float *scores, bool fill, cudaStream_t st) {
  const char *what = "csa_index_topk_mxfp4";
  CUtensorMap tmC, tmQ;
  const int B = R / Tq;
  int rc = encode_u8_2d(&tmC, codes, DI / 2, (uint64_t)B * nc_max, DI / 2, csa::kTcRows, what);
  if (rc) return rc;
  rc = encode_bf16_2d(&tmQ, qI, DI, (uint64_t)R * HI, 64, N, what);
  if (rc) return rc;
  constexpr size_t A_STAGE = (size_t)csa::kTcRows * DI * 2, C_STAGE = (size_t)csa::kTcRows * DI / 2,
                   B_SLOT = (size_t)N * DI * 2;
  const size_t smem = 1024 + 3 * A_STAGE + 2 * B_SLOT + 6 * C_STAGE + 8 * (2 * 6 + 2 * 3 + 9);
  auto kern = csa::k_index_score_fp4<N, DI>;
  rc = ensure_smem(kern, smem, what);
  if (rc) return rc;
  csa::IndexTcArgs a;
  a.w = static_cast<const __nv_bfloat16 *>(w);
  a.lens = lens;
  a.q_pos = q_pos;
  a.scores = scores;
  a.Tq = Tq;
  a.HI = HI;
  a.nc_max = nc_max;
  a.R = R;
  a.G = 1;
  a.gpb = Tq;
  a.U = R;
  a.stages = 3;
  a.fill_invisible = fill ? 1 : 0;
  return launch_cluster(kern, 1, (unsigned)num_sms(), csa::kF4Threads, smem, st, what, tmC, tmQ, a, scales);
}

template <int DI>
int launch_index_fp4_n(const void *qI, const void *w, const uint8_t *codes, const uint8_t *scales,
                       const int32_t *lens, const int32_t *q_pos, int R, int Tq, int HI, int nc_max,
                       float *scores, bool fill, cudaStream_t st) {
  if (HI <= 16) return launch_index_fp4<16, DI>(qI, w, codes, scales, lens, q_pos, R, Tq, HI, nc_max, scores, fill, st);
  if (HI <= 32) return launch_index_fp4<32, DI>(qI, w, codes, scales, lens, q_pos, R, Tq, HI, nc_max, scores, fill, st);
  if (HI <= 64) return launch_index_fp4<64, DI>(qI, w, codes, scales, lens, q_pos, R, Tq, HI, nc_max, scores, fill, st);
  return launch_index_fp4<128, DI>(qI, w, codes, scales, lens, q_pos, R, Tq, HI, nc_max, scores, fill, st);
}

template <int CS, int NT>
int launch_topk_nt(const float *scores, const int32_t *lens, const int32_t *q_pos, int R,
                   int Tq, int nc_max, int k, int32_t *idx_out, cudaStream_t st) {
  const int per = (nc_max + CS - 1) / CS;
  const size_t smem = csa::topk_dyn_bytes(per > 0 ? per : 1);
  auto kern = csa::k_topk<CS, NT>;
  int rc = ensure_smem(kern, smem, "csa_index_topk");
  if (rc) return rc;
  return launch_cluster(kern, CS, (unsigned)CS * R, NT, smem, st, "csa_index_topk (select)", scores,
                        lens, q_pos, Tq, nc_max, k, idx_out);
}

// Rows of up to 4096 keys per CTA take 256-thread CTAs (several per SM);
// longer slices 1024 threads.
template <int CS>
int launch_topk(const float *scores, const int32_t *lens, const int32_t *q_pos, int R,
                int Tq, int nc_max, int k, int32_t *idx_out, cudaStream_t st) {
  if ((nc_max + CS - 1) / CS <= 4096)
    return launch_topk_nt<CS, 256>(scores, lens, q_pos, R, Tq, nc_max, k, idx_out, st);
  return launch_topk_nt<CS, csa::kTopkThreads>(scores, lens, q_pos, R, Tq, nc_max, k, idx_out, st);
}

// Whether this device can co-schedule a 16-CTA cluster of the top-k kernel
// (a non-portable cluster size; checked once per device).
bool topk16_supported(int nc_max) {
  static int cache[64] = {0};  // 0 unknown, 1 yes, 2 no
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return false;
  if (cache[dev] == 0) {
    auto kern = csa::k_topk<16>;
    const size_t smem = csa::topk_dyn_bytes(csa::kTopkSliceCap);
    int ok = 2;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(16, 1, 1);
      cfg.blockDim = dim3(csa::kTopkThreads, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = 16;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0) ok = 1;
    }
    cudaGetLastError();
    cache[dev] = ok;
  }
  (void)nc_max;
  return cache[dev] == 1;
}

// ---------------------------------------------------------------------------
// attention
// ---------------------------------------------------------------------------
template <typename T, int D>
int launch_attend_fma(const csa::AttendArgs &a, int R, long max_keys, cudaStream_t st,
                      const char *what) {
  const int cs = attend_cluster_size(max_keys);
  const size_t smem = sizeof(float) * ((size_t)a.H * D + csa::kAttTile * (D + 1) + 2 * a.H) +
                      sizeof(int) * csa::kAttTile;
  void (*kern)(csa::AttendArgs) = nullptr;
  switch (cs) {
    case 1: kern = csa::k_attend_fma<T, D, 1>; break;
    case 2: kern = csa::k_attend_fma<T, D, 2>; break;
    case 4: kern = csa::k_attend_fma<T, D, 4>; break;
    default: kern = csa::k_attend_fma<T, D, 8>; break;
  }
  int rc = ensure_smem(kern, smem, what);
  if (rc) return rc;
  return launch_cluster(kern, cs, (unsigned)cs * R, csa::kAttThreads, smem, st, what, a);
}

// Tensor-core attention (bf16, d = 128): enough clusters to fill the GPU
// when the batch is small, one CTA per row when rows alone fill it.
int launch_attend_tc(const csa::AttendArgs &a, int R, cudaStream_t st, const char *what) {
  // one CTA per SM (its shared memory allows no second): the largest
  // cluster, up to 8, that keeps all R * cs CTAs in one wave
  int cs = 1;
  while (cs < 8 && (long)R * cs * 2 <= num_sms()) cs *= 2;
  void (*kern)(csa::AttendArgs) = nullptr;
  switch (cs) {
    case 1: kern = csa::k_attend_tc<1>; break;
    case 2: kern = csa::k_attend_tc<2>; break;
    case 4: kern = csa::k_attend_tc<4>; break;
    default: kern = csa::k_attend_tc<8>; break;
  }
  const size_t smem = csa::at_smem_bytes(cs, a.kv_fp8 != nullptr);
  int rc = ensure_smem(kern, smem, what);
  if (rc) return rc;
  // clusters: one per row; one CTA per row: persistent CTAs, one per SM,
  // each looping over rows (set-up and TMEM allocation once per SM)
  const unsigned grid = cs == 1 ? (unsigned)std::min(R, num_sms()) : (unsigned)cs * R;
  return launch_cluster(kern, cs, grid, csa::kAtThreads, smem, st, what, a);
}

// QK-norm / partial RoPE arguments of the fused attention entry points.
struct QkSpec {
  int flags = 0;  // CSA_NR_NORM | CSA_NR_ROTATE, 0: none
  const void *gamma = nullptr;
  float eps = 0.f;
  int rope_dim = 0;
  float rope_base = 0.f;
};

// FP8 entry planes of csa_attend_fp8 / hca_attend_fp8 (all NULL: kv_c).
struct F8Spec {
  const uint8_t *codes = nullptr;
  const uint8_t *scales = nullptr;
  const void *rope = nullptr;
};

// Validation shared by csa_norm_rope and the fused attention.
int check_norm_rope(const char *what, int d, int flags, float eps, int rope_dim, float rope_base,
                    const void *gamma) {
  if (flags & ~(CSA_NR_NORM | CSA_NR_ROTATE | CSA_NR_INVERSE))
    return fail(CSA_ERR_UNSUPPORTED, "%s: unknown flags 0x%x", what, flags);
  if ((flags & CSA_NR_NORM) && !(eps >= 0.f && eps < INFINITY))
    return fail(CSA_ERR_SHAPE, "%s: eps must be finite and >= 0", what);
  if (flags & CSA_NR_ROTATE) {
    if (rope_dim < 0 || rope_dim > d || (rope_dim & 1))
      return fail(CSA_ERR_UNSUPPORTED, "%s: rope_dim=%d must be even and in [0, d=%d]", what, rope_dim, d);
    if (!(rope_base > 0.f && rope_base < INFINITY))
      return fail(CSA_ERR_SHAPE, "%s: rope_base must be finite and > 0", what);
  }
  if (gamma && (reinterpret_cast<uintptr_t>(gamma) & 3))
    return fail(CSA_ERR_ALIGN, "%s: gamma must be 4-byte aligned", what);
  return CSA_OK;
}

int attend_common(const void *q, const void *kv_c, const void *kv_tok, int n_tok,
                  const int32_t *idx, const int32_t *lens, const int32_t *q_pos, int B, int Tq,
                  int H, int d, int nc_max, int k, int m, int window, float scale,
                  const float *sink, csa_dtype dt, void *out, void *stream, const char *what,
                  const QkSpec &qk = QkSpec(), const F8Spec &f8 = F8Spec()) {
  int rc = check_dtype(dt, what);
  if (rc) return rc;
  const bool fp8 = f8.codes || f8.scales || f8.rope;
  if (fp8) {
    if (dt != CSA_BF16 || d != 128)
      return fail(CSA_ERR_UNSUPPORTED, "%s: FP8 entries need bf16 and d = 128 (64 FP8 + 64 bf16 dims)", what);
    if (nc_max % 4) return fail(CSA_ERR_UNSUPPORTED, "%s: FP8 entries need nc_max %% 4 == 0", what);
    if (nc_max > 0 && (!f8.codes || !f8.scales || !f8.rope))
      return fail(CSA_ERR_NULL, "%s: an FP8 entry plane is NULL", what);
    if (nc_max > 0 && (!aligned16(f8.codes) || !aligned16(f8.rope) || (reinterpret_cast<uintptr_t>(f8.scales) & 3)))
      return fail(CSA_ERR_ALIGN, "%s: FP8 codes and rope planes 16-byte aligned, scales 4-byte", what);
    if ((long)B * nc_max >= (1L << 31)) return fail(CSA_ERR_UNSUPPORTED, "%s: B * nc_max >= 2^31", what);
  }
  if (qk.flags) {
    if (qk.flags & CSA_NR_INVERSE)
      return fail(CSA_ERR_UNSUPPORTED, "%s: the output's inverse rotation follows CSA_NR_ROTATE", what);
    rc = check_norm_rope(what, d, qk.flags, qk.eps, qk.rope_dim, qk.rope_base, qk.gamma);
    if (rc) return rc;
  }
  if (B < 0 || Tq < 0) return fail(CSA_ERR_SHAPE, "%s: B=%d and Tq=%d must be >= 0", what, B, Tq);
  if ((long)B * Tq == 0) return CSA_OK;
  if (!q || !kv_tok || !lens || !out || (idx == nullptr && k > 0) || (nc_max > 0 && !kv_c && !fp8))
    return fail(CSA_ERR_NULL, "%s: a required pointer is NULL", what);
  if (!aligned16(q) || !aligned16(kv_tok) || !aligned16(out) || (kv_c && !aligned16(kv_c)))
    return fail(CSA_ERR_ALIGN, "%s: tensors must be 16-byte aligned", what);
  if (d != 64 && d != 128) return fail(CSA_ERR_UNSUPPORTED, "%s: d=%d not in {64,128}", what, d);
  if (H < 1 || H > 128) return fail(CSA_ERR_UNSUPPORTED, "%s: H=%d not in [1,128]", what, H);
  if (window < 1 || window > 4096)
    return fail(CSA_ERR_UNSUPPORTED, "%s: window=%d not in [1,4096]", what, window);
  if (n_tok < 1) return fail(CSA_ERR_SHAPE, "%s: n_tok=%d must be >= 1", what, n_tok);
  if (nc_max < 0) return fail(CSA_ERR_SHAPE, "%s: nc_max=%d must be >= 0", what, nc_max);
  if ((long)B * Tq > (1L << 26)) return fail(CSA_ERR_UNSUPPORTED, "%s: too many query rows", what);
  csa::AttendArgs a;
  a.q = q;
  a.kv_c = kv_c;
  a.kv_tok = kv_tok;
  a.idx = idx;
  a.lens = lens;
  a.q_pos = q_pos;
  a.out = out;
  a.sink = sink;
  a.n_tok = n_tok;
  a.k = k;
  a.Tq = Tq;
  a.H = H;
  a.nc_max = nc_max;
  a.m = m;
  a.window = window;
  a.R = B * Tq;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
  a.scale_log2 = sc * 1.4426950408889634f;
  a.qk_flags = qk.flags;
  a.rope_r = (qk.flags & CSA_NR_ROTATE) ? qk.rope_dim : 0;
  a.q_gamma = (qk.flags & CSA_NR_NORM) ? qk.gamma : nullptr;
  a.q_eps = qk.eps;
  a.rope_log2_base = (qk.flags & CSA_NR_ROTATE) ? std::log2((double)qk.rope_base) : 0.0;
  a.kv_fp8 = fp8 ? f8.codes : nullptr;
  a.kv_sc = fp8 ? f8.scales : nullptr;
  a.kv_rope = fp8 ? f8.rope : nullptr;
  const int R = B * Tq;
  const long max_keys = (idx ? (long)k : (long)nc_max) + window;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == CSA_F32)
    return d == 64 ? launch_attend_fma<float, 64>(a, R, max_keys, st, what)
                   : launch_attend_fma<float, 128>(a, R, max_keys, st, what);
  if (d == 128) return launch_attend_tc(a, R, st, what);
  return launch_attend_fma<__nv_bfloat16, 64>(a, R, max_keys, st, what);
}

}  // namespace

// ===========================================================================
// extern "C" entry points
// ===========================================================================
extern "C" {

int csa_version(void) { return (0 << 16) | 2; }

int csa_set_kernel_timing(int enable) {
  g_timing = enable != 0;
  return CSA_OK;
}

int csa_kernel_timing(float *ms, int max_kernels) {
  const int n = g_nlaunch;
  for (int i = 0; i < n && i < max_kernels && ms; ++i) {
    cudaError_t e = cudaEventSynchronize(g_slots[i].b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms[i], g_slots[i].a, g_slots[i].b);
    if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "kernel timing: %s", cudaGetErrorString(e));
  }
  return n;
}

const char *csa_last_error(void) { return g_last_error.c_str(); }

int csa_check_device_error(void *stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "stream error: %s", cudaGetErrorString(e));
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, csa::g_dev_err, sizeof(int));
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "reading the device error word: %s", cudaGetErrorString(e));
  if (v == 0) return CSA_OK;
  const int zero = 0;
  cudaMemcpyToSymbol(csa::g_dev_err, &zero, sizeof(int));
  static const char *what[] = {"", "a query position outside its sequence",
                               "a sequence length outside [0, n_max]",
                               "visible entries exceed the cache rows",
                               "a query window larger than the token ring"};
  return fail(CSA_ERR_DEVICE, "device check failed: %s", (v > 0 && v < 5) ? what[v] : "unknown");
}

int csa_compress(const void *x, const int32_t *lens, int B, int n_max, int d, const void *W_a,
                 const void *W_b, const void *bias8, csa_dtype dt, void *out, void *stream) {
  begin_call();
  const char *what = "csa_compress";
  int rc = check_dtype(dt, what);
  if (rc) return rc;
  if (B < 0 || n_max < 0) return fail(CSA_ERR_SHAPE, "%s: B=%d, n_max=%d must be >= 0", what, B, n_max);
  if (d != 32 && d != 64 && d != 128) return fail(CSA_ERR_UNSUPPORTED, "%s: d=%d not in {32,64,128}", what, d);
  if (B == 0 || n_max == 0) return CSA_OK;
  if (B > 65535) return fail(CSA_ERR_UNSUPPORTED, "%s: B=%d > 65535", what, B);
  if (!x || !lens || !W_a || !W_b || !bias8 || !out) return fail(CSA_ERR_NULL, "%s: a required pointer is NULL", what);
  if (!aligned16(x) || !aligned16(W_a) || !aligned16(W_b) || !aligned16(bias8) || !aligned16(out))
    return fail(CSA_ERR_ALIGN, "%s: tensors must be 16-byte aligned", what);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == CSA_F32) return launch_csa_compress<float>(x, lens, B, n_max, d, W_a, W_b, bias8, out, st);
  return launch_csa_compress<__nv_bfloat16>(x, lens, B, n_max, d, W_a, W_b, bias8, out, st);
}

int hca_compress(const void *x, const int32_t *lens, int B, int n_max, int d, int m, const void *W,
                 const void *bias, csa_dtype dt, void *out, void *stream) {
  begin_call();
  const char *what = "hca_compress";
  int rc = check_dtype(dt, what);
  if (rc) return rc;
  if (B < 0 || n_max < 0) return fail(CSA_ERR_SHAPE, "%s: B=%d, n_max=%d must be >= 0", what, B, n_max);
  if (d != 32 && d != 64 && d != 128) return fail(CSA_ERR_UNSUPPORTED, "%s: d=%d not in {32,64,128}", what, d);
  if (m < 1 || m > 4096) return fail(CSA_ERR_UNSUPPORTED, "%s: m=%d not in [1,4096]", what, m);
  if (B == 0 || n_max == 0) return CSA_OK;
  if (B > 65535) return fail(CSA_ERR_UNSUPPORTED, "%s: B=%d > 65535", what, B);
  if (!x || !lens || !W || !bias || !out) return fail(CSA_ERR_NULL, "%s: a required pointer is NULL", what);
  if (!aligned16(x) || !aligned16(W) || !aligned16(bias) || !aligned16(out))
    return fail(CSA_ERR_ALIGN, "%s: tensors must be 16-byte aligned", what);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == CSA_F32) return launch_hca_compress<float>(x, lens, B, n_max, d, m, W, bias, out, st);
  return launch_hca_compress<__nv_bfloat16>(x, lens, B, n_max, d, m, W, bias, out, st);
}

static int compress_step_common(bool is_csa, const void *tok, int n_tok, const int32_t *lens, int B,
                                int d, int m, const void *Wa, const void *Wb, const void *bias,
                                csa_dtype dt, void *cache, int nc_max, void *stream,
                                const char *what) {
  begin_call();
  int rc = check_dtype(dt, what);
  if (rc) return rc;
  if (d != 32 && d != 64 && d != 128) return fail(CSA_ERR_UNSUPPORTED, "%s: d=%d not in {32,64,128}", what, d);
  if (!is_csa && (m < 1 || m > 4096)) return fail(CSA_ERR_UNSUPPORTED, "%s: m=%d not in [1,4096]", what, m);
  if (B < 0 || n_tok < 1 || nc_max < 0)
    return fail(CSA_ERR_SHAPE, "%s: B >= 0, n_tok >= 1, nc_max >= 0 required", what);
  if (B == 0 || nc_max == 0) return CSA_OK;
  if (!tok || !lens || !Wa || (is_csa && !Wb) || !bias || !cache)
    return fail(CSA_ERR_NULL, "%s: a required pointer is NULL", what);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == CSA_F32)
    return compress_step_d<float>(is_csa, tok, n_tok, lens, B, d, m, Wa, Wb, bias, cache, nc_max, st, what);
  return compress_step_d<__nv_bfloat16>(is_csa, tok, n_tok, lens, B, d, m, Wa, Wb, bias, cache, nc_max, st,
                                        what);
}

int csa_compress_step(const void *x_tok, int n_tok, const int32_t *lens, int B, int d, const void *W_a,
                      const void *W_b, const void *bias8, csa_dtype dt, void *cache, int nc_max,
                      void *stream) {
  return compress_step_common(true, x_tok, n_tok, lens, B, d, 4, W_a, W_b, bias8, dt, cache, nc_max,
                              stream, "csa_compress_step");
}

int hca_compress_step(const void *x_tok, int n_tok, const int32_t *lens, int B, int d, int m,
                      const void *W, const void *bias, csa_dtype dt, void *cache, int nc_max,
                      void *stream) {
  return compress_step_common(false, x_tok, n_tok, lens, B, d, m, W, nullptr, bias, dt, cache, nc_max,
                              stream, "hca_compress_step");
}

size_t csa_index_topk_workspace_size(int B, int Tq, int nc_max, int has_scores_out) {
  if (B <= 0 || Tq <= 0 || nc_max <= 0 || has_scores_out) return 0;
  const size_t bytes = sizeof(float) * (size_t)B * Tq * nc_max;
  return (bytes + 255) & ~(size_t)255;
}

}  // extern "C"

namespace {

// The tensor-core scoring kernel serves bf16 keys of 64 or 128 dims.
bool index_uses_tc(csa_dtype dt, int dI) { return dt == CSA_BF16 && (dI == 64 || dI == 128); }

int index_scores_impl(const void *q_idx, const void *w, const void *k_idx, const int32_t *lens,
                      const int32_t *q_pos, int B, int Tq, int HI, int dI, int nc_max,
                      csa_dtype dt, float *scores, bool fill, cudaStream_t st) {
  const int R = B * Tq;
  if (R == 0 || nc_max == 0) return CSA_OK;
  if (R > 65535) return fail(CSA_ERR_UNSUPPORTED, "csa_index_scores: B*Tq=%d > 65535", R);
  // bf16 with 128-byte key rows or wider: the tensor-core kernel
  if (index_uses_tc(dt, dI)) {
    if ((long)B * nc_max >= (1L << 31) || (long)R * HI >= (1L << 31))
      return fail(CSA_ERR_UNSUPPORTED, "csa_index_scores: tensor too large for 32-bit coordinates");
    return dI == 64 ? launch_index_tc_n<64>(q_idx, w, k_idx, lens, q_pos, R, Tq, HI, nc_max, scores, fill, st)
                    : launch_index_tc_n<128>(q_idx, w, k_idx, lens, q_pos, R, Tq, HI, nc_max, scores, fill, st);
  }
  if (dt == CSA_F32) {
    switch (dI) {
      case 32: return launch_index_fma<float, 32>(q_idx, w, k_idx, lens, q_pos, R, Tq, HI, nc_max, scores, st);
      case 64: return launch_index_fma<float, 64>(q_idx, w, k_idx, lens, q_pos, R, Tq, HI, nc_max, scores, st);
      default: return launch_index_fma<float, 128>(q_idx, w, k_idx, lens, q_pos, R, Tq, HI, nc_max, scores, st);
    }
  }
  switch (dI) {
    case 32: return launch_index_fma<__nv_bfloat16, 32>(q_idx, w, k_idx, lens, q_pos, R, Tq, HI, nc_max, scores, st);
    case 64: return launch_index_fma<__nv_bfloat16, 64>(q_idx, w, k_idx, lens, q_pos, R, Tq, HI, nc_max, scores, st);
    default: return launch_index_fma<__nv_bfloat16, 128>(q_idx, w, k_idx, lens, q_pos, R, Tq, HI, nc_max, scores, st);
  }
}

int topk_impl(const float *scores, const int32_t *lens, const int32_t *q_pos, int B,
              int Tq, int nc_max, int k, int32_t *idx_out, cudaStream_t st) {
  const int R = B * Tq;
  if (R == 0) return CSA_OK;
  // long rows: a 16-CTA cluster where the device can schedule one
  if (nc_max > 8 * 16384 && topk16_supported(nc_max))
    return launch_topk<16>(scores, lens, q_pos, R, Tq, nc_max, k, idx_out, st);
  switch (topk_cluster_size(nc_max)) {
    case 1: return launch_topk<1>(scores, lens, q_pos, R, Tq, nc_max, k, idx_out, st);
    case 2: return launch_topk<2>(scores, lens, q_pos, R, Tq, nc_max, k, idx_out, st);
    case 4: return launch_topk<4>(scores, lens, q_pos, R, Tq, nc_max, k, idx_out, st);
    default: return launch_topk<8>(scores, lens, q_pos, R, Tq, nc_max, k, idx_out, st);
  }
}

// shared argument checks of the indexer entry points
int check_index_args(const char *what, csa_dtype dt, int B, int Tq, int HI, int dI, int nc_max) {
  int rc = check_dtype(dt, what);
  if (rc) return rc;
  if (B < 0 || Tq < 0 || nc_max < 0) return fail(CSA_ERR_SHAPE, "%s: B, Tq, nc_max must be >= 0", what);
  if (HI < 1 || HI > 128) return fail(CSA_ERR_UNSUPPORTED, "%s: HI=%d not in [1,128]", what, HI);
  if (dI != 32 && dI != 64 && dI != 128) return fail(CSA_ERR_UNSUPPORTED, "%s: dI=%d not in {32,64,128}", what, dI);
  if (nc_max > kMaxIndexEntries)
    return fail(CSA_ERR_UNSUPPORTED, "%s: nc_max=%d > %d", what, nc_max, kMaxIndexEntries);
  if ((long)B * Tq > 65535) return fail(CSA_ERR_UNSUPPORTED, "%s: B*Tq=%ld > 65535", what, (long)B * Tq);
  return CSA_OK;
}

int check_topk_args(const char *what, int B, int Tq, int nc_max, int k) {
  if (B < 0 || Tq < 0 || nc_max < 0) return fail(CSA_ERR_SHAPE, "%s: B, Tq, nc_max must be >= 0", what);
  if (k < 1 || k > 4096) return fail(CSA_ERR_UNSUPPORTED, "%s: k=%d not in [1,4096]", what, k);
  if (nc_max > kMaxIndexEntries)
    return fail(CSA_ERR_UNSUPPORTED, "%s: nc_max=%d > %d", what, nc_max, kMaxIndexEntries);
  if ((long)B * Tq > 65535) return fail(CSA_ERR_UNSUPPORTED, "%s: B*Tq=%ld > 65535", what, (long)B * Tq);
  return CSA_OK;
}

}  // namespace

extern "C" {

int csa_index_scores(const void *q_idx, const void *w, const void *k_idx, const int32_t *lens,
                     const int32_t *q_pos, int B, int Tq, int HI, int dI, int nc_max,
                     csa_dtype dt, float *scores_out, void *stream) {
  const char *what = "csa_index_scores";
  begin_call();
  int rc = check_index_args(what, dt, B, Tq, HI, dI, nc_max);
  if (rc) return rc;
  if ((long)B * Tq == 0 || nc_max == 0) return CSA_OK;
  if (!q_idx || !w || !k_idx || !lens || !scores_out)
    return fail(CSA_ERR_NULL, "%s: a required pointer is NULL", what);
  if (!aligned16(q_idx) || !aligned16(w) || !aligned16(k_idx) || !aligned16(scores_out))
    return fail(CSA_ERR_ALIGN, "%s: tensors must be 16-byte aligned", what);
  return index_scores_impl(q_idx, w, k_idx, lens, q_pos, B, Tq, HI, dI, nc_max, dt, scores_out,
                           true, static_cast<cudaStream_t>(stream));
}

int csa_topk(const float *scores, const int32_t *lens, const int32_t *q_pos, int B, int Tq,
             int nc_max, int k, int32_t *idx_out, void *stream) {
  const char *what = "csa_topk";
  begin_call();
  int rc = check_topk_args(what, B, Tq, nc_max, k);
  if (rc) return rc;
  if ((long)B * Tq == 0) return CSA_OK;
  if (!lens || !idx_out || (nc_max > 0 && !scores)) return fail(CSA_ERR_NULL, "%s: a required pointer is NULL", what);
  if (scores && !aligned16(scores)) return fail(CSA_ERR_ALIGN, "%s: scores must be 16-byte aligned", what);
  return topk_impl(scores, lens, q_pos, B, Tq, nc_max, k, idx_out, static_cast<cudaStream_t>(stream));
}

int csa_index_topk(const void *q_idx, const void *w, const void *k_idx, const int32_t *lens,
                   const int32_t *q_pos, int B, int Tq, int HI, int dI, int nc_max, int k,
                   csa_dtype dt, int32_t *idx_out, float *scores_out, void *workspace,
                   size_t ws_bytes, void *stream) {
  const char *what = "csa_index_topk";
  begin_call();
  int rc = check_index_args(what, dt, B, Tq, HI, dI, nc_max);
  if (rc) return rc;
  rc = check_topk_args(what, B, Tq, nc_max, k);
  if (rc) return rc;
  if ((long)B * Tq == 0) return CSA_OK;
  if (!q_idx || !w || !lens || !idx_out || (nc_max > 0 && !k_idx))
    return fail(CSA_ERR_NULL, "%s: a required pointer is NULL", what);
  if (!aligned16(q_idx) || !aligned16(w) || (k_idx && !aligned16(k_idx)) ||
      (scores_out && !aligned16(scores_out)))
    return fail(CSA_ERR_ALIGN, "%s: tensors must be 16-byte aligned", what);
  const size_t need = csa_index_topk_workspace_size(B, Tq, nc_max, scores_out != nullptr);
  if (need > 0 && (!workspace || ws_bytes < need))
    return fail(CSA_ERR_WORKSPACE, "%s: workspace of %zu B needed, %zu given", what, need,
                workspace ? ws_bytes : (size_t)0);
  if (need > 0 && !aligned16(workspace)) return fail(CSA_ERR_ALIGN, "%s: workspace must be 16-byte aligned", what);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float *scores = scores_out ? scores_out : static_cast<float *>(workspace);
  rc = index_scores_impl(q_idx, w, k_idx, lens, q_pos, B, Tq, HI, dI, nc_max, dt, scores,
                         scores_out != nullptr, st);
  if (rc) return rc;
  return topk_impl(scores, lens, q_pos, B, Tq, nc_max, k, idx_out, st);
}

int csa_attend(const void *q, const void *kv_c, const void *kv_tok, int n_tok, const int32_t *idx,
               const int32_t *lens, const int32_t *q_pos, int B, int Tq, int H, int d, int nc_max,
               int k, int window, float scale, const float *sink, csa_dtype dt, void *out,
               void *stream) {
  begin_call();
  if (k < 1 || k > 4096) return fail(CSA_ERR_UNSUPPORTED, "csa_attend: k=%d not in [1,4096]", k);
  if (!idx && (long)B * Tq > 0) return fail(CSA_ERR_NULL, "csa_attend: idx is NULL");
  return attend_common(q, kv_c, kv_tok, n_tok, idx, lens, q_pos, B, Tq, H, d, nc_max, k, 4, window,
                       scale, sink, dt, out, stream, "csa_attend");
}

int hca_attend(const void *q, const void *kv_c, const void *kv_tok, int n_tok,
               const int32_t *lens, const int32_t *q_pos, int B, int Tq, int H, int d, int nc_max,
               int m, int window, float scale, const float *sink, csa_dtype dt, void *out,
               void *stream) {
  begin_call();
  if (m < 1 || m > 4096) return fail(CSA_ERR_UNSUPPORTED, "hca_attend: m=%d not in [1,4096]", m);
  if (nc_max > 65536) return fail(CSA_ERR_UNSUPPORTED, "hca_attend: nc_max=%d > 65536", nc_max);
  return attend_common(q, kv_c, kv_tok, n_tok, nullptr, lens, q_pos, B, Tq, H, d, nc_max, 0, m,
                       window, scale, sink, dt, out, stream, "hca_attend");
}

}  // extern "C"

// ---------------------------------------------------------------------------
// The CSA + HCA layer pair of one decode step as one call (the scheduler).
// "Anatomy of a Frontier Model", "The attention: compress, then select": V4
// interleaves CSA and HCA layers.  With both layers' queries given, the HCA
// attention shares nothing with the CSA layer's scoring, selection and
// attention, so it runs on a second stream beside them: the persistent
// scoring kernel is launched on all but a quarter of the SMs (at most one
// per HCA row), and the HCA attention fills the rest from a high-priority
// stream, ahead of the selection's early-launched CTAs.  Fork and join are
// event edges, so the call can be captured into a CUDA graph with both
// branches.
// ---------------------------------------------------------------------------
namespace {

struct PairCtx {
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_pair_mu;
PairCtx g_pair[64];

int pair_ctx(PairCtx **out, const char *what) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) return fail(CSA_ERR_CUDA, "%s: no usable device", what);
  std::lock_guard<std::mutex> lock(g_pair_mu);
  PairCtx &c = g_pair[dev];
  if (!c.side) {
    int least = 0, greatest = 0;
    e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&c.side, cudaStreamNonBlocking, greatest);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.join, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      c = PairCtx();
      return fail(CSA_ERR_CUDA, "%s: creating the pair stream: %s", what, cudaGetErrorString(e));
    }
  }
  *out = &c;
  return CSA_OK;
}

}  // namespace

extern "C" {

int csa_hca_pair_decode(const void *q_csa, const void *q_idx, const void *w, const void *k_idx, const void *kv_csa,
                        int nc_max, int HI, int dI, int k, const void *q_hca, const void *kv_hca, int nh_max, int m,
                        const void *kv_tok, int n_tok, const int32_t *lens, int B, int H, int d, int window,
                        int32_t *idx_out, void *out_csa, void *out_hca, void *workspace, size_t ws_bytes,
                        void *stream) {
  const char *what = "csa_hca_pair_decode";
  begin_call();
  const csa_dtype dt = CSA_BF16;
  int rc = check_index_args(what, dt, B, 1, HI, dI, nc_max);
  if (rc) return rc;
  rc = check_topk_args(what, B, 1, nc_max, k);
  if (rc) return rc;
  if (m < 1 || m > 4096) return fail(CSA_ERR_UNSUPPORTED, "%s: m=%d not in [1,4096]", what, m);
  if (nh_max < 0 || nh_max > 65536) return fail(CSA_ERR_UNSUPPORTED, "%s: nh_max=%d not in [0,65536]", what, nh_max);
  if (B == 0) return CSA_OK;
  if (!q_csa || !q_idx || !w || !lens || !idx_out || !out_csa || !out_hca || !q_hca || !kv_tok ||
      (nc_max > 0 && (!k_idx || !kv_csa)) || (nh_max > 0 && !kv_hca))
    return fail(CSA_ERR_NULL, "%s: a required pointer is NULL", what);
  if (!aligned16(q_idx) || !aligned16(w) || (k_idx && !aligned16(k_idx)))
    return fail(CSA_ERR_ALIGN, "%s: tensors must be 16-byte aligned", what);
  const size_t need = csa_index_topk_workspace_size(B, 1, nc_max, 0);
  if (need > 0 && (!workspace || ws_bytes < need || !aligned16(workspace)))
    return fail(CSA_ERR_WORKSPACE, "%s: a 16-byte aligned workspace of %zu B is needed", what, need);
  PairCtx *pc = nullptr;
  rc = pair_ctx(&pc, what);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float *scores = static_cast<float *>(workspace);
  // fork before the first CSA kernel: the HCA branch may start at once
  cudaError_t e = cudaEventRecord(pc->fork, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(pc->side, pc->fork, 0);
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "%s: fork: %s", what, cudaGetErrorString(e));
  const int sms = num_sms();
  g_score_ctas = sms - std::max(1, std::min(B, sms / 4));
  rc = index_scores_impl(q_idx, w, k_idx, lens, nullptr, B, 1, HI, dI, nc_max, dt, scores, false, st);
  g_score_ctas = 0;
  if (!rc)
    rc = attend_common(q_hca, kv_hca, kv_tok, n_tok, nullptr, lens, nullptr, B, 1, H, d, nh_max, 0, m, window,
                       0.f, nullptr, dt, out_hca, pc->side, what);
  if (!rc) rc = topk_impl(scores, lens, nullptr, B, 1, nc_max, k, idx_out, st);
  if (!rc)
    rc = attend_common(q_csa, kv_csa, kv_tok, n_tok, idx_out, lens, nullptr, B, 1, H, d, nc_max, k, 4, window,
                       0.f, nullptr, dt, out_csa, st, what);
  // join, whatever happened above: the caller's stream (or capture) stays whole
  e = cudaEventRecord(pc->join, pc->side);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, pc->join, 0);
  if (rc) return rc;
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "%s: join: %s", what, cudaGetErrorString(e));
  return CSA_OK;
}

int csa_quantize_fp8_entries(const void *kv, long rows, int d, int rope_dim, csa_dtype dt, uint8_t *fp8,
                             uint8_t *scales, void *rope, void *stream) {
  const char *what = "csa_quantize_fp8_entries";
  begin_call();
  int rc = check_dtype(dt, what);
  if (rc) return rc;
  if (d < 64 || d > 4096 || rope_dim < 0 || rope_dim > d || (d - rope_dim) % 64 || (rope_dim & 1))
    return fail(CSA_ERR_UNSUPPORTED, "%s: d=%d, rope_dim=%d: d - rope_dim must be a multiple of 64", what, d,
                rope_dim);
  if (rows < 0 || rows >= (1L << 31)) return fail(CSA_ERR_SHAPE, "%s: rows=%ld not in [0, 2^31)", what, rows);
  if (rows == 0) return CSA_OK;
  if (!kv || (d > rope_dim && (!fp8 || !scales)) || (rope_dim > 0 && !rope))
    return fail(CSA_ERR_NULL, "%s: a required pointer is NULL", what);
  if (!aligned16(kv) || (fp8 && (reinterpret_cast<uintptr_t>(fp8) & 1)) || (rope && !aligned16(rope)))
    return fail(CSA_ERR_ALIGN, "%s: kv and rope 16-byte aligned, fp8 2-byte aligned", what);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // eight elements per lane when a row is 8, 16 or 32 lanes and the planes
  // take 8- and 16-byte vectors
  const bool v8 = (d == 64 || d == 128 || d == 256) && !(reinterpret_cast<uintptr_t>(fp8) & 7);
  if (v8) {
    const long per_cta = 8L * (32 / (d / 8));
    const unsigned g8 = (unsigned)std::max(1L, std::min((rows + per_cta - 1) / per_cta, 8L * num_sms()));
    if (dt == CSA_F32)
      return launch_cluster(csa::k_quantize_fp8_entries_v8<float>, 1, g8, csa::kF8Threads, 0, st, what,
                            static_cast<const float *>(kv), rows, d, rope_dim, fp8, scales, static_cast<float *>(rope));
    return launch_cluster(csa::k_quantize_fp8_entries_v8<__nv_bfloat16>, 1, g8, csa::kF8Threads, 0, st, what,
                          static_cast<const __nv_bfloat16 *>(kv), rows, d, rope_dim, fp8, scales,
                          static_cast<__nv_bfloat16 *>(rope));
  }
  const unsigned grid = (unsigned)std::max(1L, std::min((rows + 7) / 8, 8L * num_sms()));
  if (dt == CSA_F32)
    return launch_cluster(csa::k_quantize_fp8_entries<float>, 1, grid, csa::kF8Threads, 0, st, what,
                          static_cast<const float *>(kv), rows, d, rope_dim, fp8, scales, static_cast<float *>(rope));
  return launch_cluster(csa::k_quantize_fp8_entries<__nv_bfloat16>, 1, grid, csa::kF8Threads, 0, st, what,
                        static_cast<const __nv_bfloat16 *>(kv), rows, d, rope_dim, fp8, scales,
                        static_cast<__nv_bfloat16 *>(rope));
}

int csa_attend_fp8(const void *q, const uint8_t *kv_fp8, const uint8_t *kv_scales, const void *kv_rope,
                   const void *kv_tok, int n_tok, const int32_t *idx, const int32_t *lens, const int32_t *q_pos,
                   int B, int Tq, int H, int d, int nc_max, int k, int window, float scale, const float *sink,
                   csa_dtype dt, void *out, void *stream) {
  begin_call();
  if (k < 1 || k > 4096) return fail(CSA_ERR_UNSUPPORTED, "csa_attend_fp8: k=%d not in [1,4096]", k);
  if (!idx && (long)B * Tq > 0) return fail(CSA_ERR_NULL, "csa_attend_fp8: idx is NULL");
  F8Spec f8;
  f8.codes = kv_fp8;
  f8.scales = kv_scales;
  f8.rope = kv_rope;
  return attend_common(q, nullptr, kv_tok, n_tok, idx, lens, q_pos, B, Tq, H, d, nc_max, k, 4, window, scale,
                       sink, dt, out, stream, "csa_attend_fp8", QkSpec(), f8);
}

int hca_attend_fp8(const void *q, const uint8_t *kv_fp8, const uint8_t *kv_scales, const void *kv_rope,
                   const void *kv_tok, int n_tok, const int32_t *lens, const int32_t *q_pos, int B, int Tq, int H,
                   int d, int nc_max, int m, int window, float scale, const float *sink, csa_dtype dt, void *out,
                   void *stream) {
  begin_call();
  if (m < 1 || m > 4096) return fail(CSA_ERR_UNSUPPORTED, "hca_attend_fp8: m=%d not in [1,4096]", m);
  if (nc_max > 65536) return fail(CSA_ERR_UNSUPPORTED, "hca_attend_fp8: nc_max=%d > 65536", nc_max);
  F8Spec f8;
  f8.codes = kv_fp8;
  f8.scales = kv_scales;
  f8.rope = kv_rope;
  return attend_common(q, nullptr, kv_tok, n_tok, nullptr, lens, q_pos, B, Tq, H, d, nc_max, 0, m, window,
                       scale, sink, dt, out, stream, "hca_attend_fp8", QkSpec(), f8);
}

int csa_norm_rope(const void *x, void *y, long R, int G, int d, const int32_t *pos, const int32_t *lens,
                  int Tq, int pos_stride, int pos_offset, const void *gamma, float eps, int rope_dim,
                  float rope_base, int flags, csa_dtype dt, void *stream) {
  const char *what = "csa_norm_rope";
  begin_call();
  int rc = check_dtype(dt, what);
  if (rc) return rc;
  if (d != 64 && d != 128) return fail(CSA_ERR_UNSUPPORTED, "%s: d=%d not in {64,128}", what, d);
  if (R < 0 || G < 1) return fail(CSA_ERR_SHAPE, "%s: R=%ld must be >= 0 and G=%d >= 1", what, R, G);
  if ((flags & CSA_NR_INVERSE) && !(flags & CSA_NR_ROTATE))
    return fail(CSA_ERR_UNSUPPORTED, "%s: CSA_NR_INVERSE needs CSA_NR_ROTATE", what);
  rc = check_norm_rope(what, d, flags, eps, rope_dim, rope_base, gamma);
  if (rc) return rc;
  if (!pos && Tq < 1) return fail(CSA_ERR_SHAPE, "%s: Tq=%d must be >= 1 without pos", what, Tq);
  if (R == 0) return CSA_OK;
  if (!x || !y) return fail(CSA_ERR_NULL, "%s: x and y must not be NULL", what);
  if (!aligned16(x) || !aligned16(y)) return fail(CSA_ERR_ALIGN, "%s: x and y must be 16-byte aligned", what);
  const long rows = R * (long)G;
  if (rows / G != R || rows >= (1L << 31)) return fail(CSA_ERR_UNSUPPORTED, "%s: R*G >= 2^31 rows", what);
  csa::NormRopeArgs a;
  a.x = x;
  a.y = y;
  a.rows = rows;
  a.G = G;
  a.pos = pos;
  a.lens = pos ? nullptr : lens;
  a.Tq = Tq < 1 ? 1 : Tq;
  a.stride = pos_stride;
  a.offset = pos_offset;
  a.gamma = (flags & CSA_NR_NORM) ? gamma : nullptr;
  a.eps = eps;
  a.r = (flags & CSA_NR_ROTATE) ? rope_dim : 0;
  a.flags = flags;
  a.log2_base = (flags & CSA_NR_ROTATE) ? std::log2((double)rope_base) : 0.0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long want = (rows + 8 * csa::kNrUnroll - 1) / (8 * csa::kNrUnroll);  // 8 warps per CTA
  const unsigned grid = (unsigned)std::max(1L, std::min(want, 8L * num_sms()));  // one wave
  if (dt == CSA_F32)
    return d == 64 ? launch_cluster(csa::k_norm_rope<float, 64>, 1, grid, csa::kNrThreads, 0, st, what, a)
                   : launch_cluster(csa::k_norm_rope<float, 128>, 1, grid, csa::kNrThreads, 0, st, what, a);
  return d == 64 ? launch_cluster(csa::k_norm_rope<__nv_bfloat16, 64>, 1, grid, csa::kNrThreads, 0, st, what, a)
                 : launch_cluster(csa::k_norm_rope<__nv_bfloat16, 128>, 1, grid, csa::kNrThreads, 0, st, what, a);
}

int csa_attend_rope(const void *q, const void *kv_c, const void *kv_tok, int n_tok, const int32_t *idx,
                    const int32_t *lens, const int32_t *q_pos, int B, int Tq, int H, int d, int nc_max,
                    int k, int window, float scale, const float *sink, const void *q_gamma, float eps,
                    int rope_dim, float rope_base, int flags, csa_dtype dt, void *out, void *stream) {
  begin_call();
  if (k < 1 || k > 4096) return fail(CSA_ERR_UNSUPPORTED, "csa_attend_rope: k=%d not in [1,4096]", k);
  if (!idx && (long)B * Tq > 0) return fail(CSA_ERR_NULL, "csa_attend_rope: idx is NULL");
  QkSpec qk;
  qk.flags = flags;
  qk.gamma = q_gamma;
  qk.eps = eps;
  qk.rope_dim = rope_dim;
  qk.rope_base = rope_base;
  return attend_common(q, kv_c, kv_tok, n_tok, idx, lens, q_pos, B, Tq, H, d, nc_max, k, 4, window,
                       scale, sink, dt, out, stream, "csa_attend_rope", qk);
}

int hca_attend_rope(const void *q, const void *kv_c, const void *kv_tok, int n_tok,
                    const int32_t *lens, const int32_t *q_pos, int B, int Tq, int H, int d, int nc_max,
                    int m, int window, float scale, const float *sink, const void *q_gamma, float eps,
                    int rope_dim, float rope_base, int flags, csa_dtype dt, void *out, void *stream) {
  begin_call();
  if (m < 1 || m > 4096) return fail(CSA_ERR_UNSUPPORTED, "hca_attend_rope: m=%d not in [1,4096]", m);
  if (nc_max > 65536) return fail(CSA_ERR_UNSUPPORTED, "hca_attend_rope: nc_max=%d > 65536", nc_max);
  QkSpec qk;
  qk.flags = flags;
  qk.gamma = q_gamma;
  qk.eps = eps;
  qk.rope_dim = rope_dim;
  qk.rope_base = rope_base;
  return attend_common(q, kv_c, kv_tok, n_tok, nullptr, lens, q_pos, B, Tq, H, d, nc_max, 0, m,
                       window, scale, sink, dt, out, stream, "hca_attend_rope", qk);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// csa_index_topk_noalloc: csa_index_topk with its score scratch in a fixed
// array of device memory that the library itself holds.
//
// For callers that may not allocate device memory while they run: a serving
// engine that has handed nearly all of the GPU's memory to its own pool, a
// custom allocator that forbids allocations outside it, or code running
// where cudaMalloc / cudaFree would synchronise the device or are not
// allowed.  It calls no cudaMalloc, cudaFree or other allocating routine.
//
// The array below is loaded with the library and every GPU that loads it
// keeps it (8 MiB) until the process exits.  Host code must not hand its name
// to a kernel (on the host that name stands for a host-side shadow, not for
// the device memory): the device address comes from cudaGetSymbolAddress,
// looked up once per device with that device current, on the first call
// made on that device.  That lookup may load the module, so the first call
// on a device should come before any stream capture.
//
// All calls share the one array and it keeps what the previous call left in
// it.  Nothing in it needs to start at zero: the scoring kernel rewrites
// every visible entry of every row before the selection reads it, and the
// selection reads visible entries only.  Calls that overlap on the GPU (two
// streams, two host threads) race on the array; the caller serialises them.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScoreFloats = size_t(2) << 20;  // 8 MiB: B*Tq*nc_max <= 2,097,152

static __device__ __align__(256) float g_noalloc_scores[kNoAllocScoreFloats];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
float *g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of g_noalloc_scores on the current device (looked up once).
int noalloc_scores_ptr(float **out, const char *what) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "%s: cudaGetDevice: %s", what, cudaGetErrorString(e));
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return fail(CSA_ERR_UNSUPPORTED, "%s: device ordinal %d >= %d", what, dev, kNoAllocMaxDevices);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scores);
    if (e != cudaSuccess || !p)
      return fail(CSA_ERR_CUDA, "%s: cudaGetSymbolAddress on device %d: %s", what, dev,
                  cudaGetErrorString(e));
    g_noalloc_ptr[dev] = static_cast<float *>(p);
  }
  *out = g_noalloc_ptr[dev];
  return CSA_OK;
}

}  // namespace

extern "C" {

size_t csa_index_topk_noalloc_max_elems(void) { return kNoAllocScoreFloats; }

int csa_index_topk_noalloc(const void *q_idx, const void *w, const void *k_idx, const int32_t *lens,
                           const int32_t *q_pos, int B, int Tq, int HI, int dI, int nc_max, int k,
                           csa_dtype dt, int32_t *idx_out, void *stream) {
  const char *what = "csa_index_topk_noalloc";
  begin_call();
  int rc = check_index_args(what, dt, B, Tq, HI, dI, nc_max);
  if (rc) return rc;
  rc = check_topk_args(what, B, Tq, nc_max, k);
  if (rc) return rc;
  if ((long)B * Tq == 0) return CSA_OK;
  const size_t elems = (size_t)B * Tq * nc_max;
  if (elems > kNoAllocScoreFloats)
    return fail(CSA_ERR_WORKSPACE,
                "%s: B*Tq*nc_max = %zu scores exceed the fixed scratch of %zu (8 MiB); "
                "use csa_index_topk with a workspace",
                what, elems, kNoAllocScoreFloats);
  if (!q_idx || !w || !lens || !idx_out || (nc_max > 0 && !k_idx))
    return fail(CSA_ERR_NULL, "%s: a required pointer is NULL", what);
  if (!aligned16(q_idx) || !aligned16(w) || (k_idx && !aligned16(k_idx)))
    return fail(CSA_ERR_ALIGN, "%s: tensors must be 16-byte aligned", what);
  float *scores = nullptr;
  rc = noalloc_scores_ptr(&scores, what);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = index_scores_impl(q_idx, w, k_idx, lens, q_pos, B, Tq, HI, dI, nc_max, dt, scores, false, st);
  if (rc) return rc;
  return topk_impl(scores, lens, q_pos, B, Tq, nc_max, k, idx_out, st);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// MXFP4 indexer keys
// ---------------------------------------------------------------------------
extern "C" {

int csa_quantize_mxfp4(const void *k_idx, int B, int nc_max, int dI, csa_dtype dt, uint8_t *codes,
                       uint8_t *scales, void *stream) {
  const char *what = "csa_quantize_mxfp4";
  begin_call();
  int rc = check_dtype(dt, what);
  if (rc) return rc;
  if (dI != 64 && dI != 128) return fail(CSA_ERR_UNSUPPORTED, "%s: dI=%d not in {64,128}", what, dI);
  if (B < 0 || nc_max < 0) return fail(CSA_ERR_SHAPE, "%s: B, nc_max must be >= 0", what);
  const long blocks = (long)B * nc_max * (dI / 32);
  if (blocks == 0) return CSA_OK;
  if (!k_idx || !codes || !scales) return fail(CSA_ERR_NULL, "%s: a required pointer is NULL", what);
  if (!aligned16(k_idx) || !aligned16(codes)) return fail(CSA_ERR_ALIGN, "%s: keys and codes must be 16-byte aligned", what);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned grid = (unsigned)((blocks + 255) / 256);
  if (dt == CSA_F32)
    return launch_cluster(csa::k_quantize_mxfp4<float>, 1, grid, 256, 0, st, what,
                          static_cast<const float *>(k_idx), blocks, codes, scales);
  return launch_cluster(csa::k_quantize_mxfp4<__nv_bfloat16>, 1, grid, 256, 0, st, what,
                        static_cast<const __nv_bfloat16 *>(k_idx), blocks, codes, scales);
}

int csa_index_topk_mxfp4(const void *q_idx, const void *w, const uint8_t *codes, const uint8_t *scales,
                         const int32_t *lens, const int32_t *q_pos, int B, int Tq, int HI, int dI,
                         int nc_max, int k, int32_t *idx_out, float *scores_out, void *workspace,
                         size_t ws_bytes, void *stream) {
  const char *what = "csa_index_topk_mxfp4";
  begin_call();
  int rc = check_index_args(what, CSA_BF16, B, Tq, HI, dI, nc_max);
  if (rc) return rc;
  if (dI != 64 && dI != 128) return fail(CSA_ERR_UNSUPPORTED, "%s: dI=%d not in {64,128}", what, dI);
  rc = check_topk_args(what, B, Tq, nc_max, k);
  if (rc) return rc;
  if ((long)B * Tq == 0) return CSA_OK;
  if (!q_idx || !w || !lens || !idx_out || (nc_max > 0 && (!codes || !scales)))
    return fail(CSA_ERR_NULL, "%s: a required pointer is NULL", what);
  if (!aligned16(q_idx) || !aligned16(w) || (codes && !aligned16(codes)) ||
      (scales && (reinterpret_cast<uintptr_t>(scales) & 3)) || (scores_out && !aligned16(scores_out)))
    return fail(CSA_ERR_ALIGN, "%s: tensors must be 16-byte aligned (scales 4-byte)", what);
  const size_t need = csa_index_topk_workspace_size(B, Tq, nc_max, scores_out != nullptr);
  if (need > 0 && (!workspace || ws_bytes < need))
    return fail(CSA_ERR_WORKSPACE, "%s: workspace of %zu B needed, %zu given", what, need,
                workspace ? ws_bytes : (size_t)0);
  if (need > 0 && !aligned16(workspace)) return fail(CSA_ERR_ALIGN, "%s: workspace must be 16-byte aligned", what);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float *scores = scores_out ? scores_out : static_cast<float *>(workspace);
  const int R = B * Tq;
  if (nc_max > 0) {
    if ((long)B * nc_max >= (1L << 31) || (long)R * HI >= (1L << 31))
      return fail(CSA_ERR_UNSUPPORTED, "%s: tensor too large for 32-bit coordinates", what);
    rc = dI == 64 ? launch_index_fp4_n<64>(q_idx, w, codes, scales, lens, q_pos, R, Tq, HI, nc_max, scores,
                                           scores_out != nullptr, st)
                  : launch_index_fp4_n<128>(q_idx, w, codes, scales, lens, q_pos, R, Tq, HI, nc_max, scores,
                                            scores_out != nullptr, st);
    if (rc) return rc;
  }
  return topk_impl(scores, lens, q_pos, B, Tq, nc_max, k, idx_out, st);
}

}  // extern "C"
