"""Pins of the oracle's QK-norm and partial RoPE (``oracle.norm_rope``) and of
the chain they form with the attention: closed forms of RMSNorm and of the
rotation of unit vectors, the identity at position 0, the inverse, the
relative-position property, norm preservation, and two properties of the
whole chain (q and keys normalised and rotated, attention, output rotated
back by the query's position).

Definition: "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part
V", "The attention: compress, then select", third detail (queries and
compressed entries RMS-normalised per head; RoPE on the last dims only; the
output rotated back by its own position, leaving relative position only).
"""
import math

import numpy as np
import pytest

import oracle


def f32(a):
    return np.asarray(a, np.float32)


def unit(d, i):
    x = np.zeros((1, 1, d), np.float32)
    x[0, 0, i] = 1.0
    return x


def test_rmsnorm_closed_form():
    x = f32([[[3, 4, 0, 0]]])
    np.testing.assert_allclose(oracle.norm_rope(x, [7], eps=0.0, rope_dim=0)[0, 0], [0.6 * 2, 0.8 * 2, 0, 0],
                               rtol=0, atol=1e-15)  # rms = sqrt(25/4) = 2.5
    g = f32([1, 2, 3, 4])
    np.testing.assert_allclose(oracle.norm_rope(x, [7], gamma=g, eps=0.0, rope_dim=0)[0, 0], [1.2, 3.2, 0, 0],
                               rtol=0, atol=1e-15)
    ones = f32(np.ones((1, 1, 4)))
    np.testing.assert_allclose(oracle.norm_rope(ones, [0], eps=3.0, rope_dim=0)[0, 0], [0.5] * 4, rtol=0, atol=1e-15)


@pytest.mark.parametrize("p", [0, 1, 3, 1000, 1048575])
def test_rotation_of_unit_vectors(p):
    d, r, base = 8, 4, 10000.0
    # pair 0 of the rotated dims (dims 4, 5) turns at frequency 1, pair 1
    # (dims 6, 7) at base^(-2/4) = 0.01; dims 0..3 are not rotated
    for i, want in [(4, {4: math.cos(p), 5: math.sin(p)}),
                    (5, {4: -math.sin(p), 5: math.cos(p)}),
                    (6, {6: math.cos(0.01 * p), 7: math.sin(0.01 * p)}),
                    (7, {6: -math.sin(0.01 * p), 7: math.cos(0.01 * p)}),
                    (2, {2: 1.0})]:
        got = oracle.norm_rope(unit(d, i), [p], norm=False, rope_dim=r, base=base)[0, 0]
        ref = np.zeros(d)
        for k, v in want.items():
            ref[k] = v
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_base_sets_the_frequencies():
    got = oracle.norm_rope(unit(4, 2), [5], norm=False, rope_dim=4, base=100.0)[0, 0]
    np.testing.assert_allclose(got, [0, 0, math.cos(0.5), math.sin(0.5)], rtol=0, atol=1e-12)


def test_position_zero_is_the_identity_and_norm_comes_first():
    g = np.random.default_rng(1)
    x = f32(g.standard_normal((3, 2, 16)))
    normed = oracle.norm_rope(x, [0, 0, 0], rope_dim=0)
    np.testing.assert_array_equal(oracle.norm_rope(x, [0, 0, 0], rope_dim=8), normed)
    ms = (normed ** 2).mean(-1)
    np.testing.assert_allclose(ms, 1.0 / (1.0 + 1e-6 / (x.astype(np.float64) ** 2).mean(-1)), rtol=1e-12)


def test_inverse_undoes_forward_and_only_last_dims_move():
    g = np.random.default_rng(2)
    x = f32(g.standard_normal((5, 3, 16)))
    pos = np.array([0, 1, 17, 4096, 999_999])
    fwd = oracle.norm_rope(x, pos, norm=False, rope_dim=8)
    np.testing.assert_array_equal(fwd[..., :8], x[..., :8].astype(np.float64))
    back = oracle.norm_rope(f32(fwd), pos, norm=False, rope_dim=8, inverse=True)
    # fwd rounded to fp32 before the inverse: agreement to fp32 resolution
    np.testing.assert_allclose(back, x, rtol=0, atol=2e-6)
    np.testing.assert_allclose(np.linalg.norm(fwd, axis=-1), np.linalg.norm(x.astype(np.float64), axis=-1),
                               rtol=1e-13)


def test_dot_products_depend_on_relative_position_only():
    g = np.random.default_rng(3)
    q = f32(g.standard_normal((1, 1, 32)))
    k = f32(g.standard_normal((1, 1, 32)))

    def dot(t, s):
        a = oracle.norm_rope(q, [t], rope_dim=16)
        b = oracle.norm_rope(k, [s], rope_dim=16)
        return float((a * b).sum())

    for t, s, shift in [(10, 3, 1), (500, 7, 12345), (3, 10, 777)]:
        assert dot(t, s) == pytest.approx(dot(t + shift, s + shift), rel=1e-10, abs=1e-12)
    assert abs(dot(10, 3) - dot(10, 4)) > 1e-6  # the position does enter


def _chain(q, tok, lens, shift, window, gq, gk):
    """QK-norm + RoPE on the query (at its position t + shift) and on every
    window token (at s + shift), attention over the window only, output
    rotated back by t + shift."""
    B, Tq, H, d = q.shape
    t = lens - 1
    qr = oracle.round_to(oracle.norm_rope(q, (t + shift)[:, None], gamma=gq, rope_dim=d // 2), oracle.F32)
    s = np.arange(tok.shape[1])[None, :] + shift
    kr = oracle.round_to(oracle.norm_rope(tok[:, :, None, :], np.broadcast_to(s, tok.shape[:2]), gamma=gk,
                                          rope_dim=d // 2)[:, :, 0, :], oracle.F32)
    o = oracle.attend(qr, None, kr, lens, window=window, m=64)  # no entry visible
    return oracle.norm_rope(oracle.round_to(o, oracle.F32), (t + shift)[:, None], norm=False, rope_dim=d // 2,
                            inverse=True)


def test_chain_output_is_invariant_to_a_common_shift():
    g = np.random.default_rng(4)
    B, H, d, n = 2, 3, 16, 3
    q = f32(g.standard_normal((B, 1, H, d)))
    tok = f32(g.standard_normal((B, n, d)))
    gq, gk = f32(1 + 0.1 * g.standard_normal(d)), f32(1 + 0.1 * g.standard_normal(d))
    lens = np.array([3, 2], np.int32)
    a = _chain(q, tok, lens, 0, 8, gq, gk)
    for shift in (1, 4096, 1_000_000):
        np.testing.assert_allclose(_chain(q, tok, lens, shift, 8, gq, gk), a, rtol=0, atol=2e-6)


def test_chain_single_key_returns_the_normalised_key():
    # a window of one token: the query at t attends token t only, so the
    # output is that token normalised and rotated to t, rotated back by t
    g = np.random.default_rng(5)
    B, H, d = 1, 2, 16
    q = f32(g.standard_normal((B, 1, H, d)))
    tok = f32(g.standard_normal((B, 6, d)))
    gk = f32(1 + 0.1 * g.standard_normal(d))
    lens = np.array([6], np.int32)
    out = _chain(q, tok, lens, 0, 1, None, gk)
    ref = oracle.norm_rope(tok[:, 5:6, None, :], [0], gamma=gk, rope_dim=0)[:, :, 0, :]
    for h in range(H):
        np.testing.assert_allclose(out[0, 0, h], ref[0, 0], rtol=0, atol=3e-6)


def test_bad_arguments_are_errors():
    x = f32(np.ones((1, 1, 4)))
    with pytest.raises(oracle.OracleError):
        oracle.norm_rope(x, [0], rope_dim=3)
    with pytest.raises(oracle.OracleError):
        oracle.norm_rope(x, [0], rope_dim=6)
    with pytest.raises(oracle.OracleError):
        oracle.norm_rope(x, [0], eps=-1.0)
