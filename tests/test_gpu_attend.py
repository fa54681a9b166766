"""GPU parity of csa_attend / hca_attend against the fp64 oracle, element by
element, fed identical selected indices (stage-wise: the index list comes
from the test, never from the GPU path)."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.helpers import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu

csa = pytest.importorskip("compressed_sparse_long_03_b200")


def random_idx(seed, B, Tq, k, vis, nc_max, junk=True):
    """k slots per row: a random subset of the visible entries, plus (junk)
    -1 padding, invisible and out-of-range indices that must be ignored."""
    g = np.random.default_rng(seed)
    idx = np.full((B, Tq, k), -1, np.int32)
    for b in range(B):
        for tq in range(Tq):
            v = int(vis[b, tq])
            n = min(v, k - (8 if junk else 0))
            if n > 0:
                idx[b, tq, :n] = np.sort(g.choice(v, n, replace=False))
            if junk and k >= 8:
                idx[b, tq, k - 8:k - 4] = [v, v + 1, nc_max + 5, -7]  # never attended
                g.shuffle(idx[b, tq])
    return idx


@pytest.mark.parametrize("dt,d,H,k,nc,window,n_tok", [
    ("f32", 64, 8, 64, 256, 128, 1024),        # workload 1's shapes
    ("bf16", 128, 64, 1024, 5000, 128, 128),   # 1M decode shapes, smaller cache
    ("bf16", 128, 16, 512, 2048, 128, 8192),   # prefill shapes
    ("bf16", 64, 3, 40, 300, 37, 64),
    ("f32", 128, 128, 16, 100, 1, 1),
])
def test_csa_attend(dt, d, H, k, nc, window, n_tok):
    seed = d + H + k
    B, Tq = 3, 2
    lens = np.array([4 * nc, 4 * nc - 3, 4 * nc - 1001], np.int32)
    lens = np.maximum(lens, 2)
    q = W.normal(seed, "q", (B, Tq, H, d), 1.0, dt)
    kv = W.normal(seed, "kv", (B, nc, d), 1.0, dt)
    tok = W.normal(seed, "win", (B, n_tok, d), 1.0, dt)
    vis = oracle.visible(lens, B, Tq, 4)
    idx = random_idx(seed, B, Tq, k, vis, nc)
    out = csa.csa_attend(to_dev(q), to_dev(kv), to_dev(tok), to_dev(idx), to_dev(lens), window=window)
    csa.check_device_error()
    ref = oracle.attend(q, kv, tok, lens, idx=idx, window=window)
    assert_close(to_host(out), ref, dt, "csa_attend")


@pytest.mark.parametrize("H,B,Tq", [
    (4, 1, 2),      # 2 rows: 8-CTA clusters, fewer heads than CTAs (owners without heads)
    (100, 1, 37),   # 37 rows: 4-CTA clusters, a partly padded TMEM lane quadrant
    (128, 2, 37),   # 74 rows: 2-CTA clusters, every lane a head
    (64, 2, 150),   # 300 rows: one CTA per row, two key tiles per CTA
])
def test_csa_attend_cluster_shapes(H, B, Tq):
    """The tensor-core attention at every cluster size it launches with and at
    head counts that leave owners without heads or pad a lane quadrant."""
    seed = 900 + H + Tq
    d, k, nc, window, n_tok = 128, 256, 2000, 128, 8192
    lens = np.array([4 * nc, 4 * nc - 77][:B], np.int32)
    q = W.normal(seed, "q", (B, Tq, H, d), 1.0, "bf16")
    kv = W.normal(seed, "kv", (B, nc, d), 1.0, "bf16")
    tok = W.normal(seed, "win", (B, n_tok, d), 1.0, "bf16")
    vis = oracle.visible(lens, B, Tq, 4)
    idx = random_idx(seed, B, Tq, k, vis, nc)
    out = csa.csa_attend(to_dev(q), to_dev(kv), to_dev(tok), to_dev(idx), to_dev(lens), window=window)
    csa.check_device_error()
    ref = oracle.attend(q, kv, tok, lens, idx=idx, window=window)
    assert_close(to_host(out), ref, "bf16", "csa_attend")


@pytest.mark.parametrize("dt,d,H,m", [("bf16", 128, 64, 128), ("f32", 64, 8, 8), ("bf16", 128, 16, 4)])
def test_hca_attend_ragged(dt, d, H, m):
    seed = 3 * m + H
    B = 5
    lens = np.array([40000, 127, 128, 20000, 1], np.int32) if m == 128 else \
        np.array([4000, m - 1, m, 3001, 1], np.int32)
    nc = int((lens.max() + m - 1) // m)
    q = W.normal(seed, "q", (B, 1, H, d), 1.0, dt)
    kv = W.normal(seed, "hca_kv", (B, nc, d), 1.0, dt)
    tok = W.normal(seed, "win", (B, 128, d), 1.0, dt)
    out = csa.hca_attend(to_dev(q), to_dev(kv), to_dev(tok), to_dev(lens), m=m)
    csa.check_device_error()
    ref = oracle.attend(q, kv, tok, lens, idx=None, m=m)
    assert_close(to_host(out), ref, dt, "hca_attend")


def test_hca_attend_full_workload():
    """Workload 3 at full size: B=32, 1024 entries + 128 window, 64 heads."""
    wl = W.make(3)
    out = csa.hca_attend(to_dev(wl["q"]), to_dev(wl["hkv"]), to_dev(wl["win"]), to_dev(wl["lens"]), m=128)
    csa.check_device_error()
    ref = oracle.attend(wl["q"], wl["hkv"], wl["win"], wl["lens"], idx=None, m=128)
    assert_close(to_host(out), ref, "bf16", "hca_attend workload 3")


def test_csa_attend_full_1m_shapes():
    """Workload 4's attention stage at full size (B=4, 262,144-entry cache,
    k=1024, 64 heads, window ring of 128), indices from the test."""
    c = W.CONFIGS[4]
    wl = W.csa_cache(W.seed_of(4), c["B"], c["n"], c["H"], c["d"], c["HI"], c["dI"], "bf16", c["std_w"])
    vis = oracle.visible(wl["lens"], c["B"], 1, 4)
    idx = random_idx(4, c["B"], 1, c["k"], vis, wl.sizes["nc"], junk=False)
    out = csa.csa_attend(to_dev(wl["q"]), to_dev(wl["kv"]), to_dev(wl["win"]), to_dev(idx),
                         to_dev(wl["lens"]))
    csa.check_device_error()
    ref = oracle.attend(wl["q"], wl["kv"], wl["win"], wl["lens"], idx=idx)
    assert_close(to_host(out), ref, "bf16", "csa_attend workload 4")


def test_causal_prefill_rows_full_token_array():
    """Tq > 1 causal rows over the full token array (n_tok = n): windows that
    start at 0, partial windows, and no visible entries for t < 3."""
    seed, B, Tq, H, d, nc = 21, 1, 40, 16, 128, 600
    n = 4 * nc
    q_pos = np.sort(np.random.default_rng(seed).integers(0, n, (B, Tq))).astype(np.int32)
    q_pos[0, :5] = [0, 1, 3, 127, 128]
    lens = np.array([n], np.int32)
    q = W.normal(seed, "q", (B, Tq, H, d), 1.0, "bf16")
    kv = W.normal(seed, "kv", (B, nc, d), 1.0, "bf16")
    tok = W.normal(seed, "x", (B, n, d), 1.0, "bf16")
    vis = oracle.visible(lens, B, Tq, 4, q_pos)
    idx = random_idx(seed, B, Tq, 512, vis, nc)
    out = csa.csa_attend(to_dev(q), to_dev(kv), to_dev(tok), to_dev(idx), to_dev(lens),
                         q_pos=to_dev(q_pos))
    csa.check_device_error()
    ref = oracle.attend(q, kv, tok, lens, idx=idx, q_pos=q_pos)
    assert_close(to_host(out), ref, "bf16", "csa_attend prefill rows")


def test_deterministic_and_batch_invariant():
    seed, B, H, d, nc, k = 31, 4, 64, 128, 3000, 1024
    lens = np.array([4 * nc, 4 * nc - 17, 9000, 4 * nc - 2], np.int32)
    q = W.normal(seed, "q", (B, 1, H, d), 1.0, "bf16")
    kv = W.normal(seed, "kv", (B, nc, d), 1.0, "bf16")
    tok = W.normal(seed, "win", (B, 128, d), 1.0, "bf16")
    idx = random_idx(seed, B, 1, k, oracle.visible(lens, B, 1, 4), nc)
    args = [to_dev(a) for a in (q, kv, tok, idx, lens)]
    a = to_host(csa.csa_attend(*args))
    b = to_host(csa.csa_attend(*args))
    np.testing.assert_array_equal(a, b)
    one = to_host(csa.csa_attend(*[to_dev(x[2:3]) for x in (q, kv, tok, idx, lens)]))
    np.testing.assert_array_equal(one[0], a[2])


def test_invalid_window_ring_raises_device_error():
    B, H, d, nc = 1, 4, 64, 50
    q = W.normal(2, "q", (B, 1, H, d), 1.0, "f32")
    kv = W.normal(2, "kv", (B, nc, d), 1.0, "f32")
    tok = W.normal(2, "win", (B, 64, d), 1.0, "f32")  # ring of 64 < window 128
    lens = np.array([4 * nc], np.int32)
    out = csa.hca_attend(to_dev(q), to_dev(kv), to_dev(tok), to_dev(lens), m=4, window=128)
    with pytest.raises(csa.CsaError):
        csa.check_device_error()
    assert np.all(to_host(out) == 0)


@pytest.mark.parametrize("dt,d,H,B,Tq,hca", [
    ("bf16", 128, 64, 2, 1, False),   # tensor-core path, 8-CTA clusters
    ("bf16", 128, 16, 2, 150, False),  # tensor-core path, one CTA per row
    ("f32", 64, 8, 2, 3, False),      # CUDA-core path
    ("bf16", 64, 12, 2, 2, False),    # CUDA-core path, bf16
    ("bf16", 128, 64, 3, 1, True),    # HCA, tensor-core path
])
def test_attend_with_sink(dt, d, H, B, Tq, hca):
    """Per-head sink logits (one far below every logit, one far above, the
    rest moderate) on both attention kernels, against the oracle."""
    torch = pytest.importorskip("torch")
    seed = 300 + d + H + Tq
    k, nc, window, n_tok = 256, 1500, 128, 6000
    lens = np.array([4 * nc, 4 * nc - 9, 4 * nc - 100][:B], np.int32)
    q = W.normal(seed, "q", (B, Tq, H, d), 1.0, dt)
    kv = W.normal(seed, "kv", (B, nc, d), 1.0, dt)
    tok = W.normal(seed, "win", (B, n_tok, d), 1.0, dt)
    sink = (np.random.default_rng(seed).standard_normal(H) * 2.0).astype(np.float32)
    sink[0] = -1e30
    sink[-1] = 40.0
    dsink = torch.from_numpy(sink).cuda()
    if hca:
        m = 4
        out = csa.hca_attend(to_dev(q), to_dev(kv), to_dev(tok), to_dev(lens), m=m, window=window,
                             sink=dsink)
        ref = oracle.attend(q, kv, tok, lens, idx=None, m=m, window=window, sink=sink.astype(np.float64))
    else:
        vis = oracle.visible(lens, B, Tq, 4)
        idx = random_idx(seed, B, Tq, k, vis, nc)
        out = csa.csa_attend(to_dev(q), to_dev(kv), to_dev(tok), to_dev(idx), to_dev(lens),
                             window=window, sink=dsink)
        ref = oracle.attend(q, kv, tok, lens, idx=idx, window=window, sink=sink.astype(np.float64))
    csa.check_device_error()
    assert_close(to_host(out), ref, dt, "attend with sink")
