"""Pins of the oracle's compressors (CSA stride 4 / overlap 8, HCA stride m)
against closed forms and limits that do not reuse the oracle's formula.

Definitions: "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part
V", "The attention: compress, then select" (CSA: 4 tokens per entry, 8-token
overlapping per-channel softmax pooling with position biases; HCA: 128 tokens
per entry, no overlap); "The Exchange Rates of a Million Tokens", section 3
(two series, one joint softmax).
"""
import numpy as np
import pytest

import oracle
from workloads import bf16_bits, bf16_to_f32

BIG = 60.0  # exp(-60) ~ 1e-26: a one-hot logit selects one token to fp64 precision


def rnd(shape, seed=0, lo=None, hi=None):
    g = np.random.default_rng(seed)
    if lo is None:
        return g.standard_normal(shape).astype(np.float32)
    return g.uniform(lo, hi, shape).astype(np.float32)


def zeros_params(d, slots=8):
    return (np.zeros((d, d), np.float32), np.zeros((d, d), np.float32),
            np.zeros((slots, d), np.float32))


# ---------------------------------------------------------------- CSA ----
def test_csa_uniform_weights_is_mean_pool_with_masking():
    """W=0, beta=0: every weight equal, so entry i is the plain mean of the
    valid tokens of blocks i-1 and i (entry 0: its own 4 tokens; a trailing
    partial block: what exists).  Rows past ceil(n/4) are zero."""
    B, n_max, d = 3, 13, 5
    x = rnd((B, n_max, d), 1)
    lens = np.array([13, 8, 6], np.int32)
    Wa, Wb, beta = zeros_params(d)
    out = oracle.csa_compress(x, lens, Wa, Wb, beta)
    assert out.shape == (B, 4, d)
    X = x.astype(np.float64)
    for b in range(B):
        n = lens[b]
        nc = -(-n // 4)
        for i in range(4):
            if i >= nc:
                assert np.all(out[b, i] == 0.0)
                continue
            lo, hi = max(0, 4 * (i - 1)), min(n, 4 * i + 4)
            np.testing.assert_allclose(out[b, i], X[b, lo:hi].mean(0), rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("j0", range(8))
def test_csa_one_hot_bias_selects_slot(j0):
    """beta[j0,:] = 60 (W=0) makes slot j0 take all the weight, so entry i is
    token 4(i-1)+j0: pins the slot -> token map, the overlap direction (entry
    i pools blocks i-1 and i) and the single joint softmax over both series.
    When slot j0 falls outside the sequence it is masked and the remaining
    valid tokens share equal weight."""
    B, n, d = 1, 18, 4
    x = rnd((B, n, d), 2)
    Wa, Wb, beta = zeros_params(d)
    beta[j0, :] = BIG
    out = oracle.csa_compress(x, np.array([n], np.int32), Wa, Wb, beta)
    X = x.astype(np.float64)[0]
    for i in range(-(-n // 4)):
        s = 4 * (i - 1) + j0
        if 0 <= s < n:
            np.testing.assert_allclose(out[0, i], X[s], rtol=1e-14, atol=1e-14)
        else:
            lo, hi = max(0, 4 * (i - 1)), min(n, 4 * i + 4)
            np.testing.assert_allclose(out[0, i], X[lo:hi].mean(0), rtol=1e-13, atol=1e-14)


def test_csa_per_channel_independence():
    """A different one-hot slot per channel selects a different token per
    channel: the pooling weights are per channel."""
    n, d = 16, 8
    x = rnd((1, n, d), 3)
    Wa, Wb, beta = zeros_params(d)
    slots = [c % 8 for c in range(d)]
    for c, j in enumerate(slots):
        beta[j, c] = BIG
    out = oracle.csa_compress(x, np.array([n], np.int32), Wa, Wb, beta)
    X = x.astype(np.float64)[0]
    for i in range(1, n // 4):
        for c, j in enumerate(slots):
            assert abs(out[0, i, c] - X[4 * (i - 1) + j, c]) < 1e-14


def _designated_inputs(n, d, seed):
    """Tokens <= 0 everywhere; the caller raises one entry to +1."""
    return rnd((1, n, d), seed, -1.0, 0.0)


@pytest.mark.parametrize("series", ["a", "b"])
def test_csa_series_a_is_previous_block_series_b_own_block(series):
    """Wa = 60*I (Wb = 0, beta = 0): the logit of channel c is 60*x_s[c] on
    the previous block and 0 on the own block.  With all tokens <= 0 except
    x_s*[c] = 1 for one token s* of the previous block, entry i equals 1 in
    channel c.  Symmetrically for Wb and the own block.  A swapped or
    mis-assigned series gives a value well below 1."""
    n, d, i = 16, 6, 2
    x = _designated_inputs(n, d, 4)
    Wa, Wb, beta = zeros_params(d)
    if series == "a":
        Wa[:] = BIG * np.eye(d)
        sstar = [4 * (i - 1) + (c % 4) for c in range(d)]
    else:
        Wb[:] = BIG * np.eye(d)
        sstar = [4 * i + (c % 4) for c in range(d)]
    for c, s in enumerate(sstar):
        x[0, s, c] = 1.0
    out = oracle.csa_compress(x, np.array([n], np.int32), Wa, Wb, beta)
    np.testing.assert_allclose(out[0, i], np.ones(d), rtol=0, atol=1e-14)


def test_csa_weight_orientation_in_out():
    """Only Wa[e0][c0] = 60: channel c0's logit over the previous block is
    60*x_s[e0].  With x_s*[e0] = 1 (all other tokens' e0 entries <= 0), channel
    c0 of entry i is x_s*[c0], and every other channel is the plain mean.
    A transposed weight would move the selection to channel e0."""
    n, d, i, e0, c0 = 16, 5, 3, 1, 3
    x = _designated_inputs(n, d, 5)
    s_star = 4 * (i - 1) + 2
    x[0, s_star, e0] = 1.0
    Wa, Wb, beta = zeros_params(d)
    Wa[e0, c0] = BIG
    out = oracle.csa_compress(x, np.array([n], np.int32), Wa, Wb, beta)
    X = x.astype(np.float64)[0]
    assert abs(out[0, i, c0] - X[s_star, c0]) < 1e-14
    mean = X[4 * (i - 1):4 * i + 4].mean(0)
    for c in range(d):
        if c != c0:
            assert abs(out[0, i, c] - mean[c]) < 1e-13


def test_csa_convex_combination_and_length():
    """Each output channel lies in the [min, max] of the pooled tokens, and the
    cache has ceil(n/4) rows."""
    for n in (1, 3, 4, 5, 31, 32):
        d = 6
        x = rnd((1, n, d), 6 + n)
        g = np.random.default_rng(n)
        Wa = g.normal(0, 2, (d, d)).astype(np.float32)
        Wb = g.normal(0, 2, (d, d)).astype(np.float32)
        beta = g.normal(0, 2, (8, d)).astype(np.float32)
        out = oracle.csa_compress(x, np.array([n], np.int32), Wa, Wb, beta)
        assert out.shape[1] == -(-n // 4)
        X = x.astype(np.float64)[0]
        for i in range(out.shape[1]):
            seg = X[max(0, 4 * (i - 1)):min(n, 4 * i + 4)]
            assert np.all(out[0, i] >= seg.min(0) - 1e-12)
            assert np.all(out[0, i] <= seg.max(0) + 1e-12)


def test_csa_bf16_decoding_matches_fp32_values():
    """bf16 bit patterns decode to the same real values as their fp32
    widening: the same problem given either way gives the same result."""
    n, d = 12, 4
    xf = bf16_to_f32(bf16_bits(rnd((1, n, d), 7)))
    g = np.random.default_rng(7)
    P = [bf16_to_f32(bf16_bits(g.normal(0, 1, s).astype(np.float32))) for s in ((d, d), (d, d), (8, d))]
    a = oracle.csa_compress(xf, np.array([n], np.int32), *P)
    b = oracle.csa_compress(bf16_bits(xf), np.array([n], np.int32), *[bf16_bits(p) for p in P])
    np.testing.assert_array_equal(a, b)


# ---------------------------------------------------------------- HCA ----
@pytest.mark.parametrize("m", [8, 128])
def test_hca_uniform_weights_is_block_mean(m):
    """W=0, beta=0: entry i is the mean of block i (no overlap), a partial
    last block pools what exists, rows past ceil(n/m) are zero."""
    d = 3
    n_max = 2 * m + m // 2 + 1
    x = rnd((2, n_max, d), 8)
    lens = np.array([n_max, m + 3], np.int32)
    W = np.zeros((d, d), np.float32)
    beta = np.zeros((m, d), np.float32)
    out = oracle.hca_compress(x, lens, W, beta, m=m)
    assert out.shape == (2, 3, d)
    X = x.astype(np.float64)
    for b in range(2):
        for i in range(3):
            lo, hi = m * i, min(int(lens[b]), m * (i + 1))
            if lo >= lens[b]:
                assert np.all(out[b, i] == 0)
            else:
                np.testing.assert_allclose(out[b, i], X[b, lo:hi].mean(0), rtol=1e-13, atol=1e-14)


def test_hca_one_hot_bias_and_orientation():
    """beta[j0] = 60 selects token m*i + j0; W[e0][c0] = 60 with a designated
    token selects by input channel e0 into output channel c0."""
    m, d, n = 16, 4, 48
    x = _designated_inputs(n, d, 9)
    W = np.zeros((d, d), np.float32)
    beta = np.zeros((m, d), np.float32)
    beta[5, :] = BIG
    out = oracle.hca_compress(x, np.array([n], np.int32), W, beta, m=m)
    X = x.astype(np.float64)[0]
    for i in range(3):
        np.testing.assert_allclose(out[0, i], X[m * i + 5], rtol=0, atol=1e-14)
    beta[:] = 0
    e0, c0, s_star = 2, 0, m + 11
    x[0, s_star, e0] = 1.0
    W[e0, c0] = BIG
    out = oracle.hca_compress(x, np.array([n], np.int32), W, beta, m=m)
    X = x.astype(np.float64)[0]
    assert abs(out[0, 1, c0] - X[s_star, c0]) < 1e-14
    np.testing.assert_allclose(out[0, 1, 1:], X[m:2 * m, 1:].mean(0), rtol=1e-13)


# ------------------------------------------------------------ rounding ----
def test_round_bf16_ties_to_even_and_no_double_rounding():
    v = np.array([1.0, 1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 + 2.0 ** -8 + 2.0 ** -40,
                  -(1 + 2.0 ** -8 + 2.0 ** -40), 2.0 ** -130, 3.4e38, 3.4e39, -0.0])
    got = bf16_to_f32(oracle.round_to(v, oracle.BF16)).astype(np.float64)
    want = [1.0, 1.0, 1 + 2.0 ** -6, 1 + 2.0 ** -7, -(1 + 2.0 ** -7), 2.0 ** -130,
            float(bf16_to_f32(bf16_bits(np.array([3.4e38], np.float32)))[0]), np.inf, -0.0]
    np.testing.assert_array_equal(got, want)
    assert np.signbit(got[-1])


def test_round_bf16_agrees_with_float32_rne_on_float32_values():
    """For values that are exact in float32 there is no double rounding, so
    the oracle's rounding must equal the integer-trick RNE of the input
    generator (an independent formulation)."""
    a = np.random.default_rng(11).standard_normal(100000).astype(np.float32) * 7
    np.testing.assert_array_equal(oracle.round_to(a.astype(np.float64), oracle.BF16), bf16_bits(a))
