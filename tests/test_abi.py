"""The C-ABI library loads, exports every entry point include/csa.h declares,
and rejects invalid arguments on the host (status code + message) before any
CUDA call -- so these run without a GPU."""
import ctypes
import os
import re
import subprocess

import pytest

import compressed_sparse_long_03_b200 as csa
from compressed_sparse_long_03_b200 import build as csa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")

OK, E_NULL, E_ALIGN, E_SHAPE, E_DTYPE, E_UNSUP, E_WS = 0, -1, -2, -3, -4, -5, -6
P = ctypes.c_void_p
A16 = P(0x10000)       # aligned, never dereferenced by a rejected call
A4 = P(0x10004)        # misaligned


@pytest.fixture(scope="module")
def L():
    csa_build.build()
    return csa.lib()


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^CSA_API\s+[\w\s\*]*?\b(\w+)\s*\(", src, re.M)))


def test_header_declares_the_five_entry_points():
    names = declared_symbols()
    for n in ("csa_compress", "hca_compress", "csa_index_topk", "csa_attend", "hca_attend"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", csa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    for n in declared_symbols():
        assert n in exported, n
        assert hasattr(L, n)
    assert L.csa_version() >= 1


def err(L):
    return L.csa_last_error().decode()


def test_compress_validation(L):
    assert L.csa_compress(None, A16, 1, 8, 64, A16, A16, A16, 0, A16, None) == E_NULL
    assert "NULL" in err(L)
    assert L.csa_compress(A16, A16, 1, 8, 48, A16, A16, A16, 0, A16, None) == E_UNSUP
    assert "d=48" in err(L)
    assert L.csa_compress(A16, A16, 1, 8, 64, A16, A16, A16, 7, A16, None) == E_DTYPE
    assert L.csa_compress(A4, A16, 1, 8, 64, A16, A16, A16, 1, A16, None) == E_ALIGN
    assert L.csa_compress(A16, A16, -1, 8, 64, A16, A16, A16, 1, A16, None) == E_SHAPE
    assert L.csa_compress(None, None, 0, 8, 64, None, None, None, 1, None, None) == OK   # empty batch
    assert L.hca_compress(A16, A16, 1, 8, 64, 0, A16, A16, 1, A16, None) == E_UNSUP
    assert L.hca_compress(A16, A16, 1, 8, 64, 4097, A16, A16, 1, A16, None) == E_UNSUP
    assert L.hca_compress(A16, A16, 1, 8, 64, 128, A16, A4, 1, A16, None) == E_ALIGN


def idx_call(L, **kw):
    a = dict(q=A16, w=A16, k=A16, lens=A16, q_pos=None, B=1, Tq=1, HI=64, dI=128, nc=1000, kk=64,
             dt=1, idx=A16, sc=None, ws=A16, wsb=1 << 20)
    a.update(kw)
    return L.csa_index_topk(a["q"], a["w"], a["k"], a["lens"], a["q_pos"], a["B"], a["Tq"], a["HI"],
                            a["dI"], a["nc"], a["kk"], a["dt"], a["idx"], a["sc"], a["ws"], a["wsb"], None)


def test_index_topk_validation(L):
    assert idx_call(L, kk=0) == E_UNSUP
    assert idx_call(L, kk=4097) == E_UNSUP
    assert idx_call(L, HI=0) == E_UNSUP
    assert idx_call(L, dI=96) == E_UNSUP
    assert idx_call(L, nc=327681) == E_UNSUP
    assert idx_call(L, w=None) == E_NULL
    assert idx_call(L, q=A4) == E_ALIGN
    assert idx_call(L, ws=None) == E_WS
    assert idx_call(L, wsb=100) == E_WS
    assert "workspace" in err(L)
    assert idx_call(L, B=0) == OK
    assert idx_call(L, dt=3) == E_DTYPE
    need = L.csa_index_topk_workspace_size(2, 3, 1000, 0)
    assert need >= 2 * 3 * 1000 * 4 and need % 256 == 0
    assert L.csa_index_topk_workspace_size(2, 3, 1000, 1) == 0
    assert L.csa_index_topk_workspace_size(0, 3, 1000, 0) == 0


def att_call(L, fn="csa_attend", **kw):
    a = dict(q=A16, kv=A16, tok=A16, n_tok=128, idx=A16, lens=A16, q_pos=None, B=1, Tq=1, H=64,
             d=128, nc=1000, k=1024, m=128, window=128, scale=0.0, dt=1, out=A16)
    a.update(kw)
    if fn == "csa_attend":
        return L.csa_attend(a["q"], a["kv"], a["tok"], a["n_tok"], a["idx"], a["lens"], a["q_pos"],
                            a["B"], a["Tq"], a["H"], a["d"], a["nc"], a["k"], a["window"],
                            ctypes.c_float(a["scale"]), None, a["dt"], a["out"], None)
    return L.hca_attend(a["q"], a["kv"], a["tok"], a["n_tok"], a["lens"], a["q_pos"], a["B"], a["Tq"],
                        a["H"], a["d"], a["nc"], a["m"], a["window"], ctypes.c_float(a["scale"]),
                        None, a["dt"], a["out"], None)


def test_attend_validation(L):
    assert att_call(L, d=96) == E_UNSUP
    assert att_call(L, H=129) == E_UNSUP
    assert att_call(L, window=0) == E_UNSUP
    assert att_call(L, n_tok=0) == E_SHAPE
    assert att_call(L, k=0) == E_UNSUP
    assert att_call(L, idx=None) == E_NULL
    assert att_call(L, out=A4) == E_ALIGN
    assert att_call(L, dt=2) == E_DTYPE
    assert att_call(L, B=0) == OK
    assert att_call(L, "hca_attend", m=0) == E_UNSUP
    assert att_call(L, "hca_attend", nc=65537) == E_UNSUP
    assert att_call(L, "hca_attend", kv=None) == E_NULL
    assert att_call(L, "hca_attend", kv=None, nc=0, B=0) == OK


def test_binding_refuses_cpu_tensors(L):
    import torch
    x = torch.zeros(1, 8, 64)
    with pytest.raises(ValueError):
        csa.csa_compress(x, torch.zeros(1, dtype=torch.int32), torch.zeros(64, 64),
                         torch.zeros(64, 64), torch.zeros(8, 64))


def nr_call(L, **kw):
    a = dict(x=A16, y=A16, R=4, G=1, d=128, pos=None, lens=None, Tq=1, stride=1, offset=0, gamma=None,
             eps=1e-6, rope_dim=64, base=10000.0, flags=3, dt=1)
    a.update(kw)
    return L.csa_norm_rope(a["x"], a["y"], a["R"], a["G"], a["d"], a["pos"], a["lens"], a["Tq"], a["stride"],
                           a["offset"], a["gamma"], ctypes.c_float(a["eps"]), a["rope_dim"],
                           ctypes.c_float(a["base"]), a["flags"], a["dt"], None)


def test_norm_rope_validation(L):
    assert nr_call(L, d=96) == E_UNSUP
    assert nr_call(L, rope_dim=63) == E_UNSUP
    assert nr_call(L, rope_dim=130) == E_UNSUP
    assert nr_call(L, flags=8) == E_UNSUP
    assert nr_call(L, flags=4) == E_UNSUP          # inverse without rotation
    assert nr_call(L, eps=-1.0) == E_SHAPE
    assert nr_call(L, base=0.0) == E_SHAPE
    assert nr_call(L, G=0) == E_SHAPE
    assert nr_call(L, Tq=0) == E_SHAPE
    assert nr_call(L, x=None) == E_NULL
    assert nr_call(L, y=A4) == E_ALIGN
    assert nr_call(L, dt=3) == E_DTYPE
    assert nr_call(L, R=0) == OK
    # the fused attention refuses the inverse flag (the output's turn back follows the rotation)
    rc = L.csa_attend_rope(A16, A16, A16, 128, A16, A16, None, 1, 1, 4, 128, 8, 4, 128, ctypes.c_float(0.0),
                           None, None, ctypes.c_float(1e-6), 64, ctypes.c_float(1e4), 6, 1, A16, None)
    assert rc == E_UNSUP
    rc = L.hca_attend_rope(A16, A16, A16, 128, A16, None, 1, 1, 4, 128, 8, 128, 128, ctypes.c_float(0.0),
                           None, None, ctypes.c_float(1e-6), 63, ctypes.c_float(1e4), 2, 1, A16, None)
    assert rc == E_UNSUP


def test_fp8_entries_validation(L):
    q8 = L.csa_quantize_fp8_entries
    assert q8(A16, 4, 100, 64, 1, A16, A16, A16, None) == E_UNSUP       # 36 FP8 dims
    assert q8(A16, 4, 128, 63, 1, A16, A16, A16, None) == E_UNSUP
    assert q8(A16, -1, 128, 64, 1, A16, A16, A16, None) == E_SHAPE
    assert q8(None, 4, 128, 64, 1, A16, A16, A16, None) == E_NULL
    assert q8(A4, 4, 128, 64, 1, A16, A16, A16, None) == E_ALIGN
    assert q8(A16, 0, 128, 64, 1, A16, A16, A16, None) == OK

    def att(fn="csa_attend_fp8", d=128, nc=8, dt=1, codes=A16, scales=A16, rope=A16):
        if fn == "csa_attend_fp8":
            return L.csa_attend_fp8(A16, codes, scales, rope, A16, 128, A16, A16, None, 1, 1, 4, d, nc, 4, 128,
                                    ctypes.c_float(0.0), None, dt, A16, None)
        return L.hca_attend_fp8(A16, codes, scales, rope, A16, 128, A16, None, 1, 1, 4, d, nc, 128, 128,
                                ctypes.c_float(0.0), None, dt, A16, None)
    assert att(d=64) == E_UNSUP
    assert att(dt=0) == E_UNSUP
    assert att(nc=6) == E_UNSUP
    assert att(codes=None) == E_NULL
    assert att(rope=A4) == E_ALIGN
    assert att("hca_attend_fp8", nc=65540) == E_UNSUP


def test_pair_decode_validation(L):
    def pair(**kw):
        a = dict(nc=8, HI=4, dI=128, k=4, nh=4, m=128, B=1, H=4, d=128, ws=A16, ws_bytes=1 << 20, q=A16)
        a.update(kw)
        return L.csa_hca_pair_decode(a["q"], A16, A16, A16, A16, a["nc"], a["HI"], a["dI"], a["k"], A16, A16,
                                     a["nh"], a["m"], A16, 128, A16, a["B"], a["H"], a["d"], 128, A16, A16, A16,
                                     a["ws"], a["ws_bytes"], None)
    assert pair(m=0) == E_UNSUP
    assert pair(nh=70000) == E_UNSUP
    assert pair(dI=96) == E_UNSUP
    assert pair(HI=0) == E_UNSUP
    assert pair(q=None) == E_NULL
    assert pair(ws=None) == E_WS
    assert pair(ws_bytes=16) == E_WS
    assert pair(B=0) == OK
