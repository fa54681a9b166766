"""GPU parity of csa_compress / hca_compress against the fp64 oracle, element
by element: several tiles, ragged lengths and partial tail blocks, and the
full-size prefill (8192 tokens) and HCA (131072 tokens x 32) workloads."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.helpers import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu

csa = pytest.importorskip("compressed_sparse_long_03_b200")


def _csa_case(dt, d, B, n_max, lens, seed, std):
    x = W.normal(seed, "x", (B, n_max, d), 1.0, dt)
    Wa = W.normal(seed, "Wa", (d, d), std, dt)
    Wb = W.normal(seed, "Wb", (d, d), std, dt)
    beta = W.normal(seed, "beta", (8, d), std, dt)
    return x, np.asarray(lens, np.int32), Wa, Wb, beta


@pytest.mark.parametrize("dt,d,std", [("f32", 64, 0.5), ("f32", 32, 0.5), ("bf16", 128, 128 ** -0.5),
                                      ("bf16", 64, 0.5)])
def test_csa_compress_ragged(dt, d, std):
    B, n_max = 4, 1003
    x, lens, Wa, Wb, beta = _csa_case(dt, d, B, n_max, [1003, 998, 7, 0], 11 + d, std)
    out = csa.csa_compress(to_dev(x), to_dev(lens), to_dev(Wa), to_dev(Wb), to_dev(beta))
    ref = oracle.csa_compress(x, lens, Wa, Wb, beta)
    got = to_host(out)
    assert got.shape == ref.shape == (B, (n_max + 3) // 4, d)
    assert_close(got, ref, dt, "csa_compress")
    # rows past ceil(lens/4) are exactly zero
    for b in range(B):
        assert np.all(W.bf16_to_f32(got[b, (lens[b] + 3) // 4:]) == 0) if dt == "bf16" else \
            np.all(got[b, (lens[b] + 3) // 4:] == 0)


@pytest.mark.parametrize("d", [64, 128])
def test_csa_compress_many_tiles_per_cta(d):
    """More 32-entry tiles than CTAs (each CTA loops), ragged tails."""
    B, n_max = 8, 20000
    lens = [20000, 19999, 16385, 4097, 128, 3, 1, 12345]
    x, lens, Wa, Wb, beta = _csa_case("bf16", d, B, n_max, lens, 77 + d, d ** -0.5)
    out = csa.csa_compress(to_dev(x), to_dev(lens), to_dev(Wa), to_dev(Wb), to_dev(beta))
    ref = oracle.csa_compress(x, lens, Wa, Wb, beta)
    assert_close(to_host(out), ref, "bf16", "csa_compress")


def test_csa_compress_full_prefill_workload():
    """Workload 2 (bf16, 8192 tokens, d=128): both the KV cache and the
    indexer-key cache, every row."""
    wl = W.make(2)
    lens = wl["lens"]
    for xk, a, b_, z in (("x", "Wa", "Wb", "beta"), ("kx", "kWa", "kWb", "kbeta")):
        out = csa.csa_compress(to_dev(wl[xk]), to_dev(lens), to_dev(wl[a]), to_dev(wl[b_]), to_dev(wl[z]))
        ref = oracle.csa_compress(wl[xk], lens, wl[a], wl[b_], wl[z])
        assert_close(to_host(out), ref, "bf16", f"csa_compress({xk})")


@pytest.mark.parametrize("dt,m,d", [("f32", 8, 64), ("bf16", 128, 128), ("bf16", 100, 64), ("f32", 1, 32),
                                    ("bf16", 32, 128), ("bf16", 64, 64), ("bf16", 256, 128),
                                    ("bf16", 384, 64)])
def test_hca_compress_ragged(dt, m, d):
    B, n_max = 3, 5 * m + 13
    seed = 40 + m
    x = W.normal(seed, "hca_x", (B, n_max, d), 1.0, dt)
    Wm = W.normal(seed, "hca_W", (d, d), d ** -0.5, dt)
    beta = W.normal(seed, "hca_beta", (m, d), d ** -0.5, dt)
    lens = np.array([n_max, 2 * m, m - 1], np.int32)
    out = csa.hca_compress(to_dev(x), to_dev(lens), to_dev(Wm), to_dev(beta), m=m)
    ref = oracle.hca_compress(x, lens, Wm, beta, m=m)
    assert_close(to_host(out), ref, dt, "hca_compress")


def test_hca_compress_full_workload_sampled():
    """Workload 3's compressor input (32 x 131072 tokens, d=128, m=128):
    every output row is computed on the GPU; 96 sampled rows (spread over the
    batch and the sequence) are compared with the oracle."""
    c = W.CONFIGS[3]
    wl = W.hca_tokens(W.seed_of(3), c["B"], c["n"], c["d"], "bf16", m=c["m"])
    out = to_host(csa.hca_compress(to_dev(wl["x"]), to_dev(wl["lens"]), to_dev(wl["W"]),
                                   to_dev(wl["beta"]), m=c["m"]))
    m = c["m"]
    g = np.random.default_rng(3)
    rows = [(int(b), int(i)) for b, i in zip(g.integers(0, c["B"], 96), g.integers(0, c["n"] // m, 96))]
    rows += [(0, 0), (c["B"] - 1, c["n"] // m - 1)]
    for b, i in rows:
        xs = wl["x"][b:b + 1, m * i:m * (i + 1)]
        ref = oracle.hca_compress(xs, np.array([m], np.int32), wl["W"], wl["beta"], m=m)
        assert_close(out[b:b + 1, i:i + 1], ref, "bf16", f"hca row ({b},{i})")
