"""B200 (sm_100a) Compressed Sparse Attention / Heavily Compressed Attention.

A thin ctypes binding of ``libcsa.so`` (declared in ``include/csa.h``).  Each
function marshals PyTorch CUDA tensors into the C call of the same name; every
step of the computation runs in the library's CUDA kernels.  PyTorch provides
device memory and streams only.  There is no CPU path: if the library is not
built, or a tensor is not a contiguous CUDA tensor, the call raises.

Entry points (method definitions are stated in ``include/csa.h``):
  csa_compress    CSA overlapping compressor (stride 4, 8-token windows)
  hca_compress    HCA compressor (stride m, no overlap)
  csa_compress_step / hca_compress_step  the entry a decode token completes
  csa_index_topk  lightning-indexer scores + per-query top-k
  csa_index_topk_noalloc  the same without a workspace (fixed device scratch)
  csa_attend      MQA attention over the selected entries + sliding window
  hca_attend      MQA attention over every visible HCA entry + sliding window
"""
from __future__ import annotations

import ctypes
import os

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libcsa.so")

F32 = 0
BF16 = 1

_lib = None


class CsaError(RuntimeError):
    """A library call returned a negative status."""

    def __init__(self, status: int, message: str):
        super().__init__(f"status {status}: {message}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded libcsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m compressed_sparse_long_03_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.csa_version.restype = I
        L.csa_set_kernel_timing.argtypes = [I]
        L.csa_set_kernel_timing.restype = I
        L.csa_kernel_timing.argtypes = [ctypes.POINTER(ctypes.c_float), I]
        L.csa_kernel_timing.restype = I
        L.csa_last_error.restype = ctypes.c_char_p
        L.csa_check_device_error.argtypes = [P]
        L.csa_compress.argtypes = [P, P, I, I, I, P, P, P, I, P, P]
        L.hca_compress.argtypes = [P, P, I, I, I, I, P, P, I, P, P]
        L.csa_compress_step.argtypes = [P, I, P, I, I, P, P, P, I, P, I, P]
        L.hca_compress_step.argtypes = [P, I, P, I, I, I, P, P, I, P, I, P]
        L.csa_index_topk_workspace_size.argtypes = [I, I, I, I]
        L.csa_index_topk_workspace_size.restype = S
        L.csa_index_topk.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, S, P]
        L.csa_index_topk_noalloc.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, P, P]
        L.csa_index_topk_noalloc_max_elems.argtypes = []
        L.csa_index_topk_noalloc_max_elems.restype = S
        L.csa_index_scores.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, P]
        L.csa_quantize_mxfp4.argtypes = [P, I, I, I, I, P, P, P]
        L.csa_index_topk_mxfp4.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P, P, P, S, P]
        L.csa_topk.argtypes = [P, P, P, I, I, I, I, P, P]
        L.csa_attend.argtypes = [P, P, P, I, P, P, P, I, I, I, I, I, I, I, F, P, I, P, P]
        L.hca_attend.argtypes = [P, P, P, I, P, P, I, I, I, I, I, I, I, F, P, I, P, P]
        L.csa_norm_rope.argtypes = [P, P, ctypes.c_long, I, I, P, P, I, I, I, P, F, I, F, I, I, P]
        L.csa_quantize_fp8_entries.argtypes = [P, ctypes.c_long, I, I, I, P, P, P, P]
        L.csa_hca_pair_decode.argtypes = [P, P, P, P, P, I, I, I, I, P, P, I, I, P, I, P, I, I, I, I, P, P, P,
                                          P, S, P]
        L.csa_attend_fp8.argtypes = [P, P, P, P, P, I, P, P, P, I, I, I, I, I, I, I, F, P, I, P, P]
        L.hca_attend_fp8.argtypes = [P, P, P, P, P, I, P, P, I, I, I, I, I, I, I, F, P, I, P, P]
        L.csa_attend_rope.argtypes = [P, P, P, I, P, P, P, I, I, I, I, I, I, I, F, P, P, F, I, F, I, I, P, P]
        L.hca_attend_rope.argtypes = [P, P, P, I, P, P, I, I, I, I, I, I, I, F, P, P, F, I, F, I, I, P, P]
        for name in ("csa_check_device_error", "csa_compress", "hca_compress", "csa_compress_step",
                     "hca_compress_step", "csa_quantize_mxfp4", "csa_index_topk_mxfp4", "csa_index_topk",
                     "csa_index_topk_noalloc", "csa_index_scores", "csa_topk", "csa_attend", "hca_attend"):
            getattr(L, name).restype = I
        _lib = L
    return _lib


def last_error() -> str:
    return lib().csa_last_error().decode()


def _check(rc: int) -> None:
    if rc != 0:
        raise CsaError(rc, last_error())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"float tensors are float32 or bfloat16, got {t.dtype}")


def _p(t):
    """Device pointer of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _i32(t):
    if t is not None and t.dtype != torch.int32:
        raise TypeError("lengths, positions and indices are int32")
    return _p(t)


def check_device_error(stream=None) -> None:
    """Synchronise the stream and raise if a kernel flagged an invalid length,
    position or window (the device error word is cleared)."""
    _check(lib().csa_check_device_error(_s(stream)))


def csa_compress(x, lens, W_a, W_b, bias8, out=None, stream=None):
    """x [B][n_max][d], lens [B] int32, W_a/W_b [d][d], bias8 [8][d]
    -> [B][ceil(n_max/4)][d] (rows past ceil(lens/4) zero)."""
    B, n_max, d = x.shape
    if out is None:
        out = torch.empty(B, (n_max + 3) // 4, d, dtype=x.dtype, device=x.device)
    _check(lib().csa_compress(_p(x), _i32(lens), B, n_max, d, _p(W_a), _p(W_b), _p(bias8), _dt(x),
                              _p(out), _s(stream)))
    return out


def hca_compress(x, lens, W, bias, m=128, out=None, stream=None):
    """x [B][n_max][d], W [d][d], bias [m][d] -> [B][ceil(n_max/m)][d]."""
    B, n_max, d = x.shape
    if out is None:
        out = torch.empty(B, (n_max + m - 1) // m, d, dtype=x.dtype, device=x.device)
    _check(lib().hca_compress(_p(x), _i32(lens), B, n_max, d, m, _p(W), _p(bias), _dt(x), _p(out),
                              _s(stream)))
    return out


def csa_compress_step(x_tok, lens, W_a, W_b, bias8, cache, stream=None):
    """Decode-time CSA compressor: for every sequence whose newest token
    completes a 4-token block, entry lens/4 - 1 of cache [B][nc_max][d] from
    the token ring x_tok [B][n_tok][d] (token s at row s % n_tok)."""
    B, n_tok, d = x_tok.shape
    _check(lib().csa_compress_step(_p(x_tok), n_tok, _i32(lens), B, d, _p(W_a), _p(W_b), _p(bias8),
                                   _dt(x_tok), _p(cache), cache.shape[1], _s(stream)))
    return cache


def hca_compress_step(x_tok, lens, W, bias, cache, m=128, stream=None):
    """Decode-time HCA compressor: entry lens/m - 1 of cache for every
    sequence whose newest token completes an m-token block."""
    B, n_tok, d = x_tok.shape
    _check(lib().hca_compress_step(_p(x_tok), n_tok, _i32(lens), B, d, m, _p(W), _p(bias), _dt(x_tok),
                                   _p(cache), cache.shape[1], _s(stream)))
    return cache


def index_topk_workspace_size(B, Tq, nc_max, has_scores_out=False) -> int:
    return int(lib().csa_index_topk_workspace_size(B, Tq, nc_max, int(bool(has_scores_out))))


def index_topk_workspace(B, Tq, nc_max, has_scores_out=False, device="cuda"):
    """A workspace for csa_index_topk (reusable across calls on one stream)."""
    n = index_topk_workspace_size(B, Tq, nc_max, has_scores_out)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=device)


def set_kernel_timing(enable: bool) -> None:
    """Record CUDA events around every kernel of subsequent calls on this
    host thread (serialises them; for per-kernel measurements)."""
    _check(lib().csa_set_kernel_timing(int(bool(enable))))


def kernel_timing(max_kernels: int = 16):
    """Durations (ms) of the kernels launched by the last call on this host
    thread, in launch order (needs set_kernel_timing(True))."""
    buf = (ctypes.c_float * max_kernels)()
    n = lib().csa_kernel_timing(buf, max_kernels)
    if n < 0:
        raise CsaError(n, last_error())
    return [buf[i] for i in range(min(n, max_kernels))]


def csa_index_topk(q_idx, w, k_idx, lens, k, q_pos=None, idx_out=None, scores_out=None,
                   workspace=None, stream=None):
    """q_idx [B][Tq][HI][dI], w [B][Tq][HI], k_idx [B][nc_max][dI]
    -> idx [B][Tq][k] int32 (ascending, -1 padded); fills scores_out
    [B][Tq][nc_max] float32 when given."""
    B, Tq, HI, dI = q_idx.shape
    nc_max = k_idx.shape[1]
    if idx_out is None:
        idx_out = torch.empty(B, Tq, k, dtype=torch.int32, device=q_idx.device)
    need = index_topk_workspace_size(B, Tq, nc_max, scores_out is not None)
    if workspace is None and need:
        workspace = index_topk_workspace(B, Tq, nc_max, scores_out is not None, q_idx.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().csa_index_topk(_p(q_idx), _p(w), _p(k_idx), _i32(lens), _i32(q_pos), B, Tq, HI, dI,
                                nc_max, k, _dt(q_idx), _i32(idx_out), _p(scores_out), _p(workspace),
                                ws_bytes, _s(stream)))
    return idx_out


def index_topk_noalloc_max_elems() -> int:
    """Largest B*Tq*nc_max that csa_index_topk_noalloc accepts."""
    return int(lib().csa_index_topk_noalloc_max_elems())


def csa_index_topk_noalloc(q_idx, w, k_idx, lens, k, idx_out, q_pos=None, stream=None):
    """csa_index_topk for callers that may not allocate device memory: the
    scores go to the library's fixed device scratch instead of a workspace,
    and the caller passes idx_out [B][Tq][k] int32.  Neither this function
    nor the C call allocates.  Calls share the scratch, so calls that overlap
    on the GPU race; the first call on a device belongs before any stream
    capture."""
    B, Tq, HI, dI = q_idx.shape
    nc_max = k_idx.shape[1]
    if tuple(idx_out.shape) != (B, Tq, k) or idx_out.dtype != torch.int32:
        raise ValueError("idx_out must be an int32 tensor of shape [B][Tq][k]")
    _check(lib().csa_index_topk_noalloc(_p(q_idx), _p(w), _p(k_idx), _i32(lens), _i32(q_pos), B, Tq,
                                        HI, dI, nc_max, k, _dt(q_idx), _i32(idx_out), _s(stream)))
    return idx_out


def _u8(t):
    if t is not None and t.dtype != torch.uint8:
        raise TypeError("codes and scales are uint8")
    return _p(t)


def csa_quantize_mxfp4(k_idx, codes=None, scales=None, stream=None):
    """Indexer keys [B][nc_max][dI] (bf16 or fp32) -> MXFP4 (codes uint8
    [B][nc_max][dI/2], scales uint8 [B][nc_max][dI/32])."""
    B, nc, dI = k_idx.shape
    if codes is None:
        codes = torch.empty(B, nc, dI // 2, dtype=torch.uint8, device=k_idx.device)
    if scales is None:
        scales = torch.empty(B, nc, dI // 32, dtype=torch.uint8, device=k_idx.device)
    _check(lib().csa_quantize_mxfp4(_p(k_idx), B, nc, dI, _dt(k_idx), _u8(codes), _u8(scales), _s(stream)))
    return codes, scales


def csa_index_topk_mxfp4(q_idx, w, codes, scales, lens, k, q_pos=None, idx_out=None, scores_out=None,
                         workspace=None, stream=None):
    """csa_index_topk over an MXFP4 indexer-key cache (codes [B][nc_max][dI/2],
    scales [B][nc_max][dI/32]); q_idx and w bf16."""
    B, Tq, HI, dI = q_idx.shape
    nc_max = codes.shape[1]
    if idx_out is None:
        idx_out = torch.empty(B, Tq, k, dtype=torch.int32, device=q_idx.device)
    need = index_topk_workspace_size(B, Tq, nc_max, scores_out is not None)
    if workspace is None and need:
        workspace = index_topk_workspace(B, Tq, nc_max, scores_out is not None, q_idx.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().csa_index_topk_mxfp4(_p(q_idx), _p(w), _u8(codes), _u8(scales), _i32(lens), _i32(q_pos),
                                      B, Tq, HI, dI, nc_max, k, _i32(idx_out), _p(scores_out),
                                      _p(workspace), ws_bytes, _s(stream)))
    return idx_out


def csa_index_scores(q_idx, w, k_idx, lens, q_pos=None, scores_out=None, stream=None):
    """Indexer scores only -> scores [B][Tq][nc_max] float32 (-inf where
    not visible)."""
    B, Tq, HI, dI = q_idx.shape
    nc_max = k_idx.shape[1]
    if scores_out is None:
        scores_out = torch.empty(B, Tq, nc_max, dtype=torch.float32, device=q_idx.device)
    _check(lib().csa_index_scores(_p(q_idx), _p(w), _p(k_idx), _i32(lens), _i32(q_pos), B, Tq, HI, dI,
                                  nc_max, _dt(q_idx), _p(scores_out), _s(stream)))
    return scores_out


def csa_topk(scores, lens, k, q_pos=None, idx_out=None, stream=None):
    """Top-k selection over given scores [B][Tq][nc_max] -> idx [B][Tq][k]."""
    B, Tq, nc_max = scores.shape
    if scores.dtype != torch.float32:
        raise TypeError("scores are float32")
    if idx_out is None:
        idx_out = torch.empty(B, Tq, k, dtype=torch.int32, device=scores.device)
    _check(lib().csa_topk(_p(scores), _i32(lens), _i32(q_pos), B, Tq, nc_max, k, _i32(idx_out),
                          _s(stream)))
    return idx_out


def _f32(t):
    """Device pointer of a contiguous float32 CUDA tensor (None -> NULL)."""
    if t is not None and t.dtype != torch.float32:
        raise TypeError("expected a float32 tensor")
    return _p(t)


def csa_attend(q, kv_c, kv_tok, idx, lens, q_pos=None, window=128, scale=0.0, out=None,
               stream=None, sink=None):
    """q [B][Tq][H][d], kv_c [B][nc_max][d], kv_tok [B][n_tok][d] (ring),
    idx [B][Tq][k], sink [H] float32 or None -> out [B][Tq][H][d]."""
    B, Tq, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    _check(lib().csa_attend(_p(q), _p(kv_c), _p(kv_tok), kv_tok.shape[1], _i32(idx), _i32(lens),
                            _i32(q_pos), B, Tq, H, d, kv_c.shape[1], idx.shape[-1], window,
                            float(scale), _f32(sink), _dt(q), _p(out), _s(stream)))
    return out


def hca_attend(q, kv_c, kv_tok, lens, q_pos=None, m=128, window=128, scale=0.0, out=None,
               stream=None, sink=None):
    """q [B][Tq][H][d], kv_c [B][nc_max][d], kv_tok [B][n_tok][d] (ring),
    sink [H] float32 or None -> out [B][Tq][H][d]."""
    B, Tq, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    _check(lib().hca_attend(_p(q), _p(kv_c), _p(kv_tok), kv_tok.shape[1], _i32(lens), _i32(q_pos),
                            B, Tq, H, d, kv_c.shape[1], m, window, float(scale), _f32(sink), _dt(q),
                            _p(out), _s(stream)))
    return out


# QK-norm and partial RoPE (csa_norm_rope flags)
NR_NORM = 1
NR_ROTATE = 2
NR_INVERSE = 4


def csa_norm_rope(x, y=None, pos=None, lens=None, Tq=1, pos_stride=1, pos_offset=0, gamma=None, eps=1e-6,
                  rope_dim=64, rope_base=10000.0, flags=NR_NORM | NR_ROTATE, stream=None):
    """x [R][G][d] (or [..., G, d]) -> y = RMSNorm and/or RoPE of every head
    vector (in place when y is x); the position of row group r is pos[r],
    else lens[r // Tq] - Tq + r % Tq, else pos_stride * (r % Tq) + pos_offset."""
    *lead, G, d = x.shape
    R = 1
    for n in lead:
        R *= n
    if y is None:
        y = torch.empty_like(x)
    _check(lib().csa_norm_rope(_p(x), _p(y), R, G, d, _i32(pos), _i32(lens), int(Tq), int(pos_stride),
                               int(pos_offset), _p(gamma), float(eps), int(rope_dim), float(rope_base),
                               int(flags), _dt(x), _s(stream)))
    return y


def csa_attend_rope(q, kv_c, kv_tok, idx, lens, q_pos=None, window=128, scale=0.0, out=None, stream=None,
                    sink=None, q_gamma=None, eps=1e-6, rope_dim=64, rope_base=10000.0,
                    flags=NR_NORM | NR_ROTATE):
    """csa_attend with the query's QK-norm / RoPE and the output's inverse
    rotation fused into the attention kernel."""
    B, Tq, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    _check(lib().csa_attend_rope(_p(q), _p(kv_c), _p(kv_tok), kv_tok.shape[1], _i32(idx), _i32(lens),
                                 _i32(q_pos), B, Tq, H, d, kv_c.shape[1], idx.shape[-1], window, float(scale),
                                 _f32(sink), _p(q_gamma), float(eps), int(rope_dim), float(rope_base),
                                 int(flags), _dt(q), _p(out), _s(stream)))
    return out


def hca_attend_rope(q, kv_c, kv_tok, lens, q_pos=None, m=128, window=128, scale=0.0, out=None, stream=None,
                    sink=None, q_gamma=None, eps=1e-6, rope_dim=64, rope_base=10000.0,
                    flags=NR_NORM | NR_ROTATE):
    """hca_attend with the query's QK-norm / RoPE and the output's inverse
    rotation fused into the attention kernel."""
    B, Tq, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    _check(lib().hca_attend_rope(_p(q), _p(kv_c), _p(kv_tok), kv_tok.shape[1], _i32(lens), _i32(q_pos),
                                 B, Tq, H, d, kv_c.shape[1], m, window, float(scale), _f32(sink),
                                 _p(q_gamma), float(eps), int(rope_dim), float(rope_base), int(flags), _dt(q),
                                 _p(out), _s(stream)))
    return out


def csa_quantize_fp8_entries(kv, rope_dim=64, stream=None):
    """Entries kv [..., d] -> (E4M3 codes [..., d - rope_dim] uint8, UE8M0
    scales [..., (d - rope_dim) / 64] uint8, the last rope_dim dims [..., rope_dim])."""
    *lead, d = kv.shape
    rows = 1
    for n in lead:
        rows *= n
    q = d - rope_dim
    fp8 = torch.empty(*lead, q, dtype=torch.uint8, device=kv.device)
    sc = torch.empty(*lead, q // 64, dtype=torch.uint8, device=kv.device)
    rope = torch.empty(*lead, rope_dim, dtype=kv.dtype, device=kv.device)
    _check(lib().csa_quantize_fp8_entries(_p(kv), rows, d, int(rope_dim), _dt(kv), _u8(fp8), _u8(sc), _p(rope),
                                          _s(stream)))
    return fp8, sc, rope


def csa_attend_fp8(q, kv_fp8, kv_scales, kv_rope, kv_tok, idx, lens, q_pos=None, window=128, scale=0.0, out=None,
                   stream=None, sink=None):
    """csa_attend over FP8 entries: kv_fp8 [B][nc_max][64] uint8, kv_scales
    [B][nc_max] (or [B][nc_max][1]) uint8, kv_rope [B][nc_max][64] bf16."""
    B, Tq, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    _check(lib().csa_attend_fp8(_p(q), _u8(kv_fp8), _u8(kv_scales), _p(kv_rope), _p(kv_tok), kv_tok.shape[1],
                                _i32(idx), _i32(lens), _i32(q_pos), B, Tq, H, d, kv_fp8.shape[1], idx.shape[-1],
                                window, float(scale), _f32(sink), _dt(q), _p(out), _s(stream)))
    return out


def hca_attend_fp8(q, kv_fp8, kv_scales, kv_rope, kv_tok, lens, q_pos=None, m=128, window=128, scale=0.0,
                   out=None, stream=None, sink=None):
    """hca_attend over FP8 entries (planes as csa_attend_fp8)."""
    B, Tq, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    _check(lib().hca_attend_fp8(_p(q), _u8(kv_fp8), _u8(kv_scales), _p(kv_rope), _p(kv_tok), kv_tok.shape[1],
                                _i32(lens), _i32(q_pos), B, Tq, H, d, kv_fp8.shape[1], m, window, float(scale),
                                _f32(sink), _dt(q), _p(out), _s(stream)))
    return out


def csa_hca_pair_decode(q_csa, q_idx, w, k_idx, kv_csa, q_hca, kv_hca, kv_tok, lens, k, m=128, window=128,
                        idx_out=None, out_csa=None, out_hca=None, workspace=None, stream=None):
    """One decode step of a CSA + HCA layer pair in one call (the HCA
    attention beside the CSA layer on a second stream) -> (idx_out, out_csa,
    out_hca)."""
    B, _, H, d = q_csa.shape
    HI, dI = q_idx.shape[-2], q_idx.shape[-1]
    nc_max, nh_max = k_idx.shape[1], kv_hca.shape[1]
    if idx_out is None:
        idx_out = torch.empty(B, 1, k, dtype=torch.int32, device=q_csa.device)
    if out_csa is None:
        out_csa = torch.empty_like(q_csa)
    if out_hca is None:
        out_hca = torch.empty_like(q_hca)
    if workspace is None:
        workspace = index_topk_workspace(B, 1, nc_max, False)
    _check(lib().csa_hca_pair_decode(_p(q_csa), _p(q_idx), _p(w), _p(k_idx), _p(kv_csa), nc_max, HI, dI, int(k),
                                     _p(q_hca), _p(kv_hca), nh_max, int(m), _p(kv_tok), kv_tok.shape[1],
                                     _i32(lens), B, H, d, int(window), _i32(idx_out), _p(out_csa), _p(out_hca),
                                     _p(workspace), workspace.numel() * workspace.element_size(), _s(stream)))
    return idx_out, out_csa, out_hca
