"""NumPy front end of the fp64 CPU oracle for the CSA / HCA hot path.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the CPU-baseline
leg of the benchmark may use this package; the product library never does.
It shares no code with the CUDA path.

Every function takes NumPy arrays holding the exact input bits the GPU gets
(``float32`` for fp32 runs, ``uint16`` bf16 bit patterns for bf16 runs) and
returns float64 results computed in fp64 by ``csa_oracle.c``.  ``round_to``
rounds fp64 results to the run's storage dtype (round to nearest, ties to
even) for use as the next stage's input.

The definitions each function follows are stated in ``csa_oracle.c``; the
pages describe the method in prose only:
  * compress (CSA, stride 4, overlap 8; HCA, stride m): "Anatomy of a Frontier
    Model: Reading DeepSeek-V4 Through Part V", "The attention: compress, then
    select"; "The Exchange Rates of a Million Tokens", section 3.
  * indexer scores and top-k: same CSA bullet; Exchange Rates section 3.
  * attention over selected / all entries plus a 128-token window: the
    Anatomy page's "The skeleton, and what's kept" and its three details.

Parity pins: every function here is checked against closed forms, special
cases that reduce to library routines, brute force on tiny inputs and
invariants in ``tests/test_oracle_*.py``.
"""
import ctypes
import os

import numpy as np

from . import build as _build

F32 = 0
BF16 = 1

_lib = None


def _load():
    global _lib
    if _lib is None:
        # CSA_ORACLE_LIB: a deliberately broken build, used only by the
        # mutation test to show that the pins catch planted mistakes
        path = os.environ.get("CSA_ORACLE_LIB") or _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        L = ctypes.c_long
        D = ctypes.c_double
        lib.orc_round.argtypes = [P, ctypes.c_size_t, I, P]
        lib.orc_csa_compress.argtypes = [P, P, I, I, I, P, P, P, I, P]
        lib.orc_hca_compress.argtypes = [P, P, I, I, I, I, P, P, I, P]
        lib.orc_index_scores.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P]
        lib.orc_select_topk.argtypes = [P, P, L, I, I, P]
        lib.orc_visible.argtypes = [P, P, I, I, I, P]
        lib.orc_attend.argtypes = [P, P, P, I, P, P, P, I, I, I, I, I, I, I, I, D, P, I, P]
        lib.orc_quantize_mxfp4.argtypes = [P, I, L, I, P, P]
        lib.orc_dequant_mxfp4.argtypes = [P, P, L, I, P]
        lib.orc_norm_rope.argtypes = [P, L, I, I, P, P, D, I, D, I, I, P]
        lib.orc_quantize_fp8_entries.argtypes = [P, I, L, I, I, P, P, P]
        lib.orc_dequant_fp8_entries.argtypes = [P, P, P, I, L, I, I, P]
        lib.orc_set_threads.argtypes = [I]
        lib.orc_get_threads.restype = I
        for name in ("orc_round", "orc_csa_compress", "orc_hca_compress", "orc_index_scores",
                     "orc_select_topk", "orc_visible", "orc_attend"):
            getattr(lib, name).restype = I
        _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what}: oracle status {rc}")


def _dt_of(a):
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle inputs are float32 or bf16 bits (uint16), got {a.dtype}")


def _c(a, dtype=None):
    a = np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _same_dt(*arrs):
    dts = {_dt_of(a) for a in arrs}
    if len(dts) != 1:
        raise TypeError("all float inputs of one call share a dtype")
    return dts.pop()


def set_threads(n: int) -> None:
    _load().orc_set_threads(int(n))


def get_threads() -> int:
    return int(_load().orc_get_threads())


def round_to(x64, dt):
    """Round fp64 values to the storage dtype: float32, or bf16 bits (uint16)."""
    lib = _load()
    x64, px = _c(x64, np.float64)
    out = np.empty(x64.shape, np.float32 if dt == F32 else np.uint16)
    _check(lib.orc_round(px, x64.size, dt, out.ctypes.data_as(ctypes.c_void_p)), "round")
    return out


def values(a):
    """Exact float64 values of float32 / bf16-bit arrays."""
    if a.dtype == np.float32:
        return a.astype(np.float64)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(a, np.float64)


def csa_compress(x, lens, Wa, Wb, beta):
    """a1: x [B][n_max][d], lens [B], Wa/Wb [d][d] ([in][out]), beta [8][d]
    -> float64 [B][ceil(n_max/4)][d]."""
    lib = _load()
    dt = _same_dt(x, Wa, Wb, beta)
    B, n_max, d = x.shape
    x, px = _c(x)
    lens, pl = _c(lens, np.int32)
    Wa, pa = _c(Wa)
    Wb, pb = _c(Wb)
    beta, pbt = _c(beta)
    assert Wa.shape == (d, d) and Wb.shape == (d, d) and beta.shape == (8, d)
    out = np.empty((B, (n_max + 3) // 4, d), np.float64)
    _check(lib.orc_csa_compress(px, pl, B, n_max, d, pa, pb, pbt, dt,
                                out.ctypes.data_as(ctypes.c_void_p)), "csa_compress")
    return out


def hca_compress(x, lens, W, beta, m=128):
    """a2: x [B][n_max][d], W [d][d], beta [m][d] -> float64 [B][ceil(n_max/m)][d]."""
    lib = _load()
    dt = _same_dt(x, W, beta)
    B, n_max, d = x.shape
    x, px = _c(x)
    lens, pl = _c(lens, np.int32)
    W, pw = _c(W)
    beta, pbt = _c(beta)
    assert W.shape == (d, d) and beta.shape == (m, d)
    out = np.empty((B, (n_max + m - 1) // m, d), np.float64)
    _check(lib.orc_hca_compress(px, pl, B, n_max, d, m, pw, pbt, dt,
                                out.ctypes.data_as(ctypes.c_void_p)), "hca_compress")
    return out


def index_scores(qI, w, kI, lens, q_pos=None):
    """a3: qI [B][Tq][HI][dI], w [B][Tq][HI], kI [B][nc_max][dI]
    -> float64 scores [B][Tq][nc_max] (-inf where not visible)."""
    lib = _load()
    dt = _same_dt(qI, w, kI)
    B, Tq, HI, dI = qI.shape
    nc_max = kI.shape[1]
    qI, pq = _c(qI)
    w, pw = _c(w)
    kI, pk = _c(kI)
    lens, pl = _c(lens, np.int32)
    pp = None
    if q_pos is not None:
        q_pos, pp = _c(q_pos, np.int32)
    out = np.empty((B, Tq, nc_max), np.float64)
    _check(lib.orc_index_scores(pq, pw, pk, pl, pp, B, Tq, HI, dI, nc_max, dt,
                                out.ctypes.data_as(ctypes.c_void_p)), "index_scores")
    return out


def visible(lens, B, Tq, m, q_pos=None):
    """Visible-entry count floor((t+1)/m) for every query row -> int32 [B][Tq]."""
    lib = _load()
    lens, pl = _c(lens, np.int32)
    pp = None
    if q_pos is not None:
        q_pos, pp = _c(q_pos, np.int32)
    vis = np.empty((B, Tq), np.int32)
    _check(lib.orc_visible(pl, pp, B, Tq, m, vis.ctypes.data_as(ctypes.c_void_p)), "visible")
    return vis


def select_topk(scores, vis, k):
    """a4 selection rule: scores [..., nc_max] (any float dtype, compared as
    float64), vis [...] -> int32 idx [..., k], ascending, -1 padded."""
    lib = _load()
    lead = scores.shape[:-1]
    nc_max = scores.shape[-1]
    s, ps = _c(scores.reshape(-1, nc_max), np.float64)
    v, pv = _c(np.asarray(vis).reshape(-1), np.int32)
    R = s.shape[0]
    idx = np.empty((R, k), np.int32)
    _check(lib.orc_select_topk(ps, pv, R, nc_max, k, idx.ctypes.data_as(ctypes.c_void_p)),
           "select_topk")
    return idx.reshape(*lead, k)


def index_topk(qI, w, kI, lens, k, q_pos=None):
    """a3 + a4: returns (idx int32 [B][Tq][k], scores float64 [B][Tq][nc_max])."""
    B, Tq = qI.shape[:2]
    sc = index_scores(qI, w, kI, lens, q_pos)
    vis = visible(lens, B, Tq, 4, q_pos)
    return select_topk(sc, vis, k), sc


def attend(q, kv_c, kv_tok, lens, idx=None, q_pos=None, window=128, m=4, scale=0.0, sink=None):
    """a5 (idx given, CSA) / a6 (idx None, HCA with stride m): q [B][Tq][H][d],
    kv_c [B][nc_max][d], kv_tok [B][n_tok][d] (ring: token s at row s % n_tok),
    sink [H] per-head sink logits or None -> float64 [B][Tq][H][d]."""
    lib = _load()
    arrs = [q, kv_tok] + ([kv_c] if kv_c is not None and kv_c.size else [])
    dt = _same_dt(*arrs)
    B, Tq, H, d = q.shape
    n_tok = kv_tok.shape[1]
    q, pq = _c(q)
    kv_tok, pt = _c(kv_tok)
    if kv_c is None:
        kv_c = np.zeros((B, 0, d), q.dtype)
    kv_c, pc = _c(kv_c)
    nc_max = kv_c.shape[1]
    lens, pl = _c(lens, np.int32)
    pi, k = None, 0
    if idx is not None:
        idx, pi = _c(idx, np.int32)
        k = idx.shape[-1]
    pp = None
    if q_pos is not None:
        q_pos, pp = _c(q_pos, np.int32)
    ps = None
    if sink is not None:
        sink, ps = _c(np.asarray(sink, np.float64).reshape(H), np.float64)
    out = np.empty((B, Tq, H, d), np.float64)
    _check(lib.orc_attend(pq, pc if nc_max else None, pt, n_tok, pi, pl, pp, B, Tq, H, d,
                          nc_max, k, window, m, float(scale), ps, dt,
                          out.ctypes.data_as(ctypes.c_void_p)), "attend")
    return out


def quantize_mxfp4(k):
    """MXFP4 indexer keys: k [..., dI] (float32 or bf16 bits) -> (codes
    uint8 [..., dI/2], scales uint8 [..., dI/32])."""
    lib = _load()
    dt = _dt_of(k)
    k, pk = _c(k)
    dI = k.shape[-1]
    rows = k.size // dI
    codes = np.empty(k.shape[:-1] + (dI // 2,), np.uint8)
    scales = np.empty(k.shape[:-1] + (dI // 32,), np.uint8)
    _check(lib.orc_quantize_mxfp4(pk, dt, rows, dI, codes.ctypes.data_as(ctypes.c_void_p),
                                  scales.ctypes.data_as(ctypes.c_void_p)), "quantize_mxfp4")
    return codes, scales


def dequant_mxfp4(codes, scales):
    """(codes, scales) -> float64 [..., dI], the exact key values."""
    lib = _load()
    codes, pc = _c(codes, np.uint8)
    scales, ps = _c(scales, np.uint8)
    dI = codes.shape[-1] * 2
    rows = codes.size // (dI // 2)
    out = np.empty(codes.shape[:-1] + (dI,), np.float64)
    _check(lib.orc_dequant_mxfp4(pc, ps, rows, dI, out.ctypes.data_as(ctypes.c_void_p)), "dequant_mxfp4")
    return out


def norm_rope(x, pos, gamma=None, eps=1e-6, rope_dim=64, base=10000.0, norm=True, rotate=True,
              inverse=False):
    """QK-norm and partial RoPE of ``x`` ``[..., G, d]`` (the G heads of a
    row share its position ``pos[...]``, shape ``x.shape[:-2]``): RMSNorm per
    head with ``gamma`` ``[d]`` (ones when None), then a rotation of the last
    ``rope_dim`` dims by ``+pos`` (``-pos`` when ``inverse``); the readings are
    stated at ``orc_norm_rope``.  Returns float64 of the shape of ``x``."""
    dt = _dt_of(x)
    if gamma is not None:
        _same_dt(x, gamma)
    *lead, G, d = x.shape
    R = int(np.prod(lead)) if lead else 1
    p = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, np.int64), tuple(lead)).reshape(R))
    xc, px = _c(x)
    gc, pg = (None, None) if gamma is None else _c(gamma)
    out = np.empty(x.shape, np.float64)
    flags = (1 if norm else 0) | (2 if rotate else 0) | (4 if inverse else 0)
    _check(_load().orc_norm_rope(px, R, G, d, p.ctypes.data, pg, float(eps), int(rope_dim),
                                 float(base), flags, dt, out.ctypes.data), "norm_rope")
    return out


def quantize_fp8_entries(x, rope_dim=64):
    """Entries ``x`` ``[..., d]`` -> (fp8 codes ``[..., d - r]`` uint8, UE8M0
    scales ``[..., (d - r) / 64]`` uint8, rope dims ``[..., r]`` in x's
    dtype): the FP8 cache entry read stated at ``orc_quantize_fp8_entries``."""
    dt = _dt_of(x)
    *lead, d = x.shape
    rows = int(np.prod(lead)) if lead else 1
    q = d - rope_dim
    xc, px = _c(x)
    fp8 = np.zeros((*lead, q), np.uint8)
    sc = np.zeros((*lead, q // 64), np.uint8)
    rope = np.zeros((*lead, rope_dim), x.dtype)
    _check(_load().orc_quantize_fp8_entries(px, dt, rows, d, int(rope_dim), fp8.ctypes.data, sc.ctypes.data,
                                            rope.ctypes.data), "quantize_fp8_entries")
    return fp8, sc, rope


def dequant_fp8_entries(fp8, scales, rope):
    """Exact float64 values of FP8 entries (inverse layout of
    ``quantize_fp8_entries``)."""
    dt = _dt_of(rope)
    *lead, q = fp8.shape
    r = rope.shape[-1]
    d = q + r
    rows = int(np.prod(lead)) if lead else 1
    f, pf = _c(fp8, np.uint8)
    s_, ps = _c(scales, np.uint8)
    rp, pr = _c(rope)
    out = np.empty((*lead, d), np.float64)
    _check(_load().orc_dequant_fp8_entries(pf, ps, pr, dt, rows, d, r, out.ctypes.data), "dequant_fp8_entries")
    return out
