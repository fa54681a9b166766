"""GPU parity of the decode-time compressors (csa_compress_step /
hca_compress_step) against the oracle's full compressors: a decode loop
appends one token per step to each sequence's token ring and calls the step
compressor; every entry a completed block produced must equal the oracle's
entry computed from the whole token array, and no other cache row may
change."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.helpers import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu

csa = pytest.importorskip("compressed_sparse_long_03_b200")
torch = pytest.importorskip("torch")

SENTINEL = 0x7F7F  # a bf16 / half-float bit pattern no entry produces here


def _ring(x, lens, n_tok):
    """Token rings of the current lengths: token s at row s % n_tok."""
    B, _, d = x.shape
    ring = np.zeros((B, n_tok, d), x.dtype)
    for b in range(B):
        for s in range(max(0, lens[b] - n_tok), lens[b]):
            ring[b, s % n_tok] = x[b, s]
    return ring


def _decode_loop(kind, dt, d, m, n_tok, start, steps, seed):
    B = len(start)
    N = max(start) + steps
    x = W.normal(seed, "x", (B, N, d), 1.0, dt)
    Wa = W.normal(seed, "Wa", (d, d), d ** -0.5, dt)
    Wb = W.normal(seed, "Wb", (d, d), d ** -0.5, dt)
    bias = W.normal(seed, "beta", ((8 if kind == "csa" else m), d), d ** -0.5, dt)
    stride = 4 if kind == "csa" else m
    nc = (N + stride - 1) // stride
    fill = np.full((B, nc, d), SENTINEL, np.uint16) if dt == "bf16" else np.full((B, nc, d), 7.0, np.float32)
    cache = to_dev(fill)
    dWa, dWb, dbias = to_dev(Wa), to_dev(Wb), to_dev(bias)
    lens = np.array(start, np.int32)
    for _ in range(steps):
        lens = lens + 1
        ring = to_dev(_ring(x, lens, n_tok))
        if kind == "csa":
            csa.csa_compress_step(ring, to_dev(lens), dWa, dWb, dbias, cache)
        else:
            csa.hca_compress_step(ring, to_dev(lens), dWa, dbias, cache, m=m)
    csa.check_device_error()
    got = to_host(cache)
    ref = (oracle.csa_compress(x, lens, Wa, Wb, bias) if kind == "csa"
           else oracle.hca_compress(x, lens, Wa, bias, m=m))
    for b in range(B):
        first = max(0, start[b] // stride)      # entries completed before the loop: untouched
        done = lens[b] // stride                # entries completed by now
        if done > first:
            assert_close(got[b:b + 1, first:done], ref[b:b + 1, first:done], dt, f"{kind} seq {b}")
        untouched = np.r_[0:first, done:nc]
        assert (got[b, untouched] == fill[b, untouched]).all()
    return got


@pytest.mark.parametrize("dt,d", [("bf16", 128), ("bf16", 64), ("f32", 32)])
def test_csa_compress_step_decode_loop(dt, d):
    _decode_loop("csa", dt, d, 4, n_tok=16, start=[0, 3, 9], steps=41, seed=600 + d)


@pytest.mark.parametrize("dt,d,m,n_tok", [("bf16", 128, 8, 8), ("bf16", 64, 32, 40), ("f32", 32, 5, 128)])
def test_hca_compress_step_decode_loop(dt, d, m, n_tok):
    _decode_loop("hca", dt, d, m, n_tok=n_tok, start=[0, m - 1, 2 * m + 3], steps=3 * m + 2, seed=700 + m)


def test_hca_compress_step_stride_128():
    _decode_loop("hca", "bf16", 128, 128, n_tok=128, start=[100, 127], steps=160, seed=811)


def test_compress_step_ring_too_small_is_a_device_error():
    d, B = 64, 1
    ring = torch.zeros(B, 4, d, dtype=torch.bfloat16, device="cuda")
    lens = torch.tensor([12], dtype=torch.int32, device="cuda")
    w = torch.zeros(d, d, dtype=torch.bfloat16, device="cuda")
    bias = torch.zeros(8, d, dtype=torch.bfloat16, device="cuda")
    cache = torch.zeros(B, 8, d, dtype=torch.bfloat16, device="cuda")
    csa.csa_compress_step(ring, lens, w, w, bias, cache)
    with pytest.raises(csa.CsaError):
        csa.check_device_error()
    assert (cache == 0).all()
