"""Pins of the oracle's attention over selected (CSA) / all (HCA) compressed
entries plus the sliding window, against PyTorch's textbook scaled
dot-product attention in fp64 (a library routine) on the explicit key list,
and against exact special cases.

Definitions: "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part
V": "The skeleton, and what's kept" (one KV head shared by all query heads,
the entry is both key and value), "The attention: compress, then select"
(CSA attends to its selected entries, HCA to all of them) and its first
detail (every layer also attends to the last 128 tokens).
"""
import numpy as np
import pytest
import torch

import oracle


def f32(a):
    return np.asarray(a, np.float32)


def sdpa(q_hd, keys, scale=None):
    """Textbook attention of H query rows over one shared K=V key list."""
    qt = torch.from_numpy(q_hd.astype(np.float64))[:, None, :]       # [H,1,d]
    kt = torch.from_numpy(keys.astype(np.float64))[None].expand(q_hd.shape[0], -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, scale=scale)
    return o[:, 0, :].numpy()


def setup(B=2, Tq=2, H=3, d=8, nc=12, n_tok=None, seed=0):
    g = np.random.default_rng(seed)
    lens = np.array([4 * nc - 1, 4 * nc - 6][:B], np.int32)
    n_tok = int(lens.max()) if n_tok is None else n_tok
    q = f32(g.standard_normal((B, Tq, H, d)))
    kv = f32(g.standard_normal((B, nc, d)))
    tok = f32(g.standard_normal((B, n_tok, d)))
    return q, kv, tok, lens


def keys_for(kv, tok, b, t, sel, window):
    w0 = max(0, t - window + 1)
    rows = [kv[b, i] for i in sel] + [tok[b, s % tok.shape[1]] for s in range(w0, t + 1)]
    return np.stack(rows)


@pytest.mark.parametrize("window", [1, 5, 128])
def test_csa_with_all_visible_selected_is_dense_attention(window):
    """k >= visible: CSA attention equals textbook attention over
    [C_0..C_{v-1}] followed by the window tokens."""
    q, kv, tok, lens = setup()
    B, Tq, H, d = q.shape
    k = 16
    q_pos = np.array([[lens[0] - 1, 20], [lens[1] - 1, 3]], np.int32)
    idx = np.full((B, Tq, k), -1, np.int32)
    for b in range(B):
        for tq in range(Tq):
            v = (q_pos[b, tq] + 1) // 4
            idx[b, tq, :v] = np.arange(v)
    out = oracle.attend(q, kv, tok, lens, idx=idx, q_pos=q_pos, window=window)
    for b in range(B):
        for tq in range(Tq):
            t = q_pos[b, tq]
            v = (t + 1) // 4
            ref = sdpa(q[b, tq], keys_for(kv, tok, b, t, range(v), window))
            np.testing.assert_allclose(out[b, tq], ref, rtol=1e-12, atol=1e-13)


def test_hca_dense_over_all_visible_entries():
    q, kv, tok, lens = setup(seed=1)
    m = 4
    out = oracle.attend(q, kv, tok, lens, idx=None, m=m, window=7)
    B, Tq = q.shape[:2]
    for b in range(B):
        for tq in range(Tq):
            t = lens[b] - Tq + tq
            ref = sdpa(q[b, tq], keys_for(kv, tok, b, t, range((t + 1) // m), 7))
            np.testing.assert_allclose(out[b, tq], ref, rtol=1e-12, atol=1e-13)


def test_hca_stride_128_visibility():
    g = np.random.default_rng(2)
    H, d, m = 2, 4, 128
    lens = np.array([3 * m + 5], np.int32)
    q = f32(g.standard_normal((1, 1, H, d)))
    kv = f32(g.standard_normal((1, 4, d)))
    tok = f32(g.standard_normal((1, 128, d)))
    out = oracle.attend(q, kv, tok, lens, idx=None, m=m)
    t = int(lens[0]) - 1
    ref = sdpa(q[0, 0], keys_for(kv, tok, 0, t, range(3), 128))
    np.testing.assert_allclose(out[0, 0], ref, rtol=1e-12, atol=1e-13)


def test_no_visible_entry_is_sliding_window_attention():
    """t < 4 (or n <= window with nothing selected): plain causal
    sliding-window attention over the raw tokens."""
    q, kv, tok, lens = setup(seed=3)
    q_pos = np.array([[0, 2], [1, 2]], np.int32)
    idx = np.full((2, 2, 4), -1, np.int32)
    out = oracle.attend(q, kv, tok, lens, idx=idx, q_pos=q_pos)
    for b in range(2):
        for tq in range(2):
            t = q_pos[b, tq]
            ref = sdpa(q[b, tq], tok[b, :t + 1])
            np.testing.assert_allclose(out[b, tq], ref, rtol=1e-12, atol=1e-13)


def test_single_key_returns_that_key():
    q, kv, tok, lens = setup(seed=4)
    out = oracle.attend(q, kv, tok, lens, idx=np.full((2, 2, 3), -1, np.int32),
                        q_pos=np.zeros((2, 2), np.int32))
    for b in range(2):
        np.testing.assert_array_equal(out[b], np.broadcast_to(tok[b, 0].astype(np.float64), out[b].shape))


def test_rows_sum_to_one():
    """With every key and value equal to the same constant row the output is
    that row: the attention weights of each head sum to 1."""
    B, Tq, H, d, nc = 1, 1, 4, 6, 8
    g = np.random.default_rng(5)
    q = f32(g.standard_normal((B, Tq, H, d)))
    c = f32(g.standard_normal(d))
    kv = np.broadcast_to(c, (B, nc, d)).copy()
    tok = np.broadcast_to(c, (B, 40, d)).copy()
    idx = np.array([[[0, 3, 5, -1]]], np.int32)
    out = oracle.attend(q, kv, tok, np.array([32], np.int32), idx=idx)
    np.testing.assert_allclose(out[0, 0], np.broadcast_to(c.astype(np.float64), (H, d)), rtol=1e-14, atol=1e-15)


def test_index_order_padding_invisible_and_duplicates():
    """The selected set is unordered (permuting idx changes nothing), -1 and
    entries that are not visible contribute nothing, and a listed duplicate
    contributes twice (textbook attention over the list with the duplicate)."""
    q, kv, tok, lens = setup(seed=6)
    q[:, 1] = q[:, 0]   # two query rows, same vector and position, permuted lists
    t = np.array([[30, 30], [30, 30]], np.int32)  # visible: 7 entries
    base = np.array([1, 4, 6, -1, 9, 11], np.int32)   # 9, 11 invisible
    idx = np.broadcast_to(base, (2, 2, 6)).copy()
    idx[:, 1] = base[::-1]
    out = oracle.attend(q, kv, tok, lens, idx=idx, q_pos=t)
    np.testing.assert_allclose(out[:, 0], out[:, 1], rtol=1e-14, atol=1e-15)
    ref = sdpa(q[0, 0], keys_for(kv, tok, 0, 30, [1, 4, 6], 128))
    np.testing.assert_allclose(out[0, 0], ref, rtol=1e-12, atol=1e-13)
    dup = np.array([[[1, 1, 4, -1]] * 2] * 2, np.int32)
    out2 = oracle.attend(q, kv, tok, lens, idx=dup, q_pos=t)
    ref2 = sdpa(q[0, 0], keys_for(kv, tok, 0, 30, [1, 1, 4], 128))
    np.testing.assert_allclose(out2[0, 0], ref2, rtol=1e-12, atol=1e-13)


def test_window_ring_equals_full_token_array():
    """A window ring of n_tok rows (token s at row s % n_tok) gives the same
    result as the full token array."""
    q, kv, tok, lens = setup(seed=7, n_tok=64)
    full = np.zeros((2, int(lens.max()), q.shape[-1]), np.float32)
    for s in range(full.shape[1]):
        full[:, s] = tok[:, s % 64]
    idx = np.array([[[0, 2, -1]] * 2] * 2, np.int32)
    a = oracle.attend(q, kv, tok, lens, idx=idx, window=40)
    b = oracle.attend(q, kv, full, lens, idx=idx, window=40)
    np.testing.assert_array_equal(a, b)


def test_explicit_scale():
    q, kv, tok, lens = setup(seed=8)
    idx = np.array([[[0, 5, 7]] * 2] * 2, np.int32)
    out = oracle.attend(q, kv, tok, lens, idx=idx, window=3, scale=0.5)
    t = int(lens[1]) - 1
    ref = sdpa(q[1, 1], keys_for(kv, tok, 1, t, [0, 5, 7], 3), scale=0.5)
    np.testing.assert_allclose(out[1, 1], ref, rtol=1e-12, atol=1e-13)


def test_bad_position_and_short_ring_are_errors():
    q, kv, tok, lens = setup(seed=9, n_tok=16)
    with pytest.raises(oracle.OracleError):
        oracle.attend(q, kv, tok, lens, idx=None, window=17)
    with pytest.raises(oracle.OracleError):
        oracle.attend(q, kv, tok, lens, idx=None, window=8, q_pos=np.full((2, 2), 60, np.int32))


# ---------------------------------------------------------------------------
# attention sink: "Anatomy of a Frontier Model", second of the "three
# details" (a learned per-head logit whose exponential joins the softmax
# denominator)
# ---------------------------------------------------------------------------
def test_sink_single_key_is_logistic_weight():
    """One key (query at t = 0: its own token, no entries): the output is the
    key times the logistic function of (logit - sink)."""
    q, kv, tok, lens = setup(seed=21)
    H, d = q.shape[2], q.shape[3]
    sink = np.array([-1.5, 0.0, 2.25])
    q_pos = np.zeros((2, 2), np.int32)
    out = oracle.attend(q, kv, tok, lens, idx=np.full((2, 2, 3), -1, np.int32), q_pos=q_pos, sink=sink)
    for b in range(2):
        for tq in range(2):
            v = tok[b, 0].astype(np.float64)
            for h in range(H):
                logit = float(q[b, tq, h].astype(np.float64) @ v) / np.sqrt(d)
                wgt = 1.0 / (1.0 + np.exp(sink[h] - logit))
                np.testing.assert_allclose(out[b, tq, h], wgt * v, rtol=1e-13, atol=1e-14)


def test_sink_limits():
    """A sink of -1e300 changes nothing; a sink far above every logit drives
    every output to zero."""
    q, kv, tok, lens = setup(seed=22)
    idx = np.array([[[0, 2, 5], [1, -1, 3]], [[4, 4, 0], [2, 7, 9]]], np.int32)
    base = oracle.attend(q, kv, tok, lens, idx=idx)
    low = oracle.attend(q, kv, tok, lens, idx=idx, sink=np.full(3, -1e300))
    np.testing.assert_array_equal(low, base)
    high = oracle.attend(q, kv, tok, lens, idx=idx, sink=np.full(3, 800.0))
    assert np.abs(high).max() < 1e-300


def test_sink_rescales_without_turning():
    """With a sink each head's output is the sink-free output times one
    factor in (0, 1): the sink carries no value, it only takes weight."""
    q, kv, tok, lens = setup(seed=23, d=16)
    idx = np.array([[[0, 2, 5], [1, -1, 3]], [[4, 4, 0], [2, 7, 9]]], np.int32)
    base = oracle.attend(q, kv, tok, lens, idx=idx)
    sunk = oracle.attend(q, kv, tok, lens, idx=idx, sink=np.array([0.3, -0.7, 1.1]))
    ratio = sunk / base
    spread = ratio.max(axis=-1) - ratio.min(axis=-1)
    assert spread.max() < 1e-12
    assert (ratio > 0).all() and (ratio < 1).all()
