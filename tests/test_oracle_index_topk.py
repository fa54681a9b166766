"""Pins of the oracle's lightning-indexer scores and top-k selection.

Definitions: "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part
V", "The attention: compress, then select", CSA bullet (a small indexer of
64 heads x 128 dims ranks the compressed blocks; each query attends to the
top 1,024 / 512) and "three details" (an entry exists once its block is
complete); "The Exchange Rates of a Million Tokens", section 3 (ReLU-gated
dot products, top-k).  Tie rule: lower index first (problem statement).
"""
import numpy as np
import pytest

import oracle


def f32(a):
    return np.asarray(a, np.float32)


def test_single_head_positive_dots_is_matvec():
    """HI=1, w=1 and every dot product positive: the score reduces to the
    plain matrix-vector product K q (a library routine)."""
    g = np.random.default_rng(0)
    nc, dI = 37, 16
    kI = f32(np.abs(g.standard_normal((1, nc, dI))))
    qI = f32(np.abs(g.standard_normal((1, 1, 1, dI))))
    w = f32(np.ones((1, 1, 1)))
    lens = np.array([4 * nc], np.int32)
    s = oracle.index_scores(qI, w, kI, lens)
    want = kI[0].astype(np.float64) @ qI[0, 0, 0].astype(np.float64)
    np.testing.assert_allclose(s[0, 0], want, rtol=1e-14)


@pytest.mark.parametrize("h", [0, 2])
def test_one_hot_head_weight_is_relu_of_one_head(h):
    """w = e_h picks head h alone: the score is max(0, K q_h), with negative
    dot products clipped to exactly 0 (the ReLU gate)."""
    g = np.random.default_rng(1)
    nc, HI, dI = 29, 3, 8
    kI = f32(g.standard_normal((1, nc, dI)))
    qI = f32(g.standard_normal((1, 1, HI, dI)))
    w = np.zeros((1, 1, HI), np.float32)
    w[0, 0, h] = 1.0
    s = oracle.index_scores(qI, w, kI, np.array([4 * nc], np.int32))
    dots = kI[0].astype(np.float64) @ qI[0, 0, h].astype(np.float64)
    np.testing.assert_allclose(s[0, 0], np.maximum(dots, 0.0), rtol=1e-14, atol=0)
    assert np.any(dots < 0) and np.all(s[0, 0][dots < 0] == 0.0)


def test_linear_in_head_weights_and_homogeneous_in_query():
    """score(w1 + w2) = score(w1) + score(w2), and doubling every indexer
    query doubles the score (ReLU is positively homogeneous): catches a
    missing head weight, a scale or a non-ReLU gate."""
    g = np.random.default_rng(2)
    nc, HI, dI = 50, 4, 12
    kI = f32(g.standard_normal((1, nc, dI)))
    qI = f32(g.standard_normal((1, 1, HI, dI)))
    w1 = f32(g.integers(-16, 17, (1, 1, HI)) / 8.0)   # coarse grid: w1 + w2 exact in fp32
    w2 = f32(g.integers(-16, 17, (1, 1, HI)) / 8.0)
    lens = np.array([4 * nc], np.int32)
    s1 = oracle.index_scores(qI, w1, kI, lens)
    s2 = oracle.index_scores(qI, w2, kI, lens)
    s12 = oracle.index_scores(qI, f32(w1 + w2), kI, lens)
    np.testing.assert_allclose(s12, s1 + s2, rtol=1e-12, atol=1e-12)
    s_2q = oracle.index_scores(f32(2 * qI), w1, kI, lens)
    np.testing.assert_array_equal(s_2q, 2 * s1)


def test_visibility_only_complete_blocks():
    """A query at position t sees entries i < floor((t+1)/4); the rest are
    -inf and their keys do not influence visible scores."""
    g = np.random.default_rng(3)
    nc, HI, dI = 10, 2, 4
    kI = f32(g.standard_normal((2, nc, dI)))
    qI = f32(g.standard_normal((2, 3, HI, dI)))
    w = f32(g.standard_normal((2, 3, HI)))
    lens = np.array([39, 17], np.int32)
    q_pos = np.array([[0, 3, 38], [4, 7, 16]], np.int32)
    s = oracle.index_scores(qI, w, kI, lens, q_pos)
    for b in range(2):
        for tq in range(3):
            v = (q_pos[b, tq] + 1) // 4
            assert np.all(np.isfinite(s[b, tq, :v]))
            assert np.all(s[b, tq, v:] == -np.inf)
    kI2 = kI.copy()
    kI2[:, 9:] = 100.0
    s2 = oracle.index_scores(qI, w, kI2, lens, q_pos)
    np.testing.assert_array_equal(s2[0, :2], s[0, :2])
    np.testing.assert_array_equal(s2[1], s[1])
    # default positions: the last Tq tokens of each sequence
    s_def = oracle.index_scores(qI, w, kI, lens)
    s_exp = oracle.index_scores(qI, w, kI, lens, np.array([[36, 37, 38], [14, 15, 16]], np.int32))
    np.testing.assert_array_equal(s_def, s_exp)


def test_query_position_outside_sequence_is_an_error():
    qI = np.zeros((1, 1, 1, 4), np.float32)
    with pytest.raises(oracle.OracleError):
        oracle.index_scores(qI, np.ones((1, 1, 1), np.float32), np.zeros((1, 4, 4), np.float32),
                            np.array([16], np.int32), np.array([[16]], np.int32))


# ------------------------------------------------------------------ top-k --
def rank_count_topk(scores, v, k):
    """Top-k by its definition: i is selected iff fewer than k visible j come
    before it in the order (score desc, index asc).  O(v^2), tiny inputs."""
    sel = []
    for i in range(v):
        before = sum(1 for j in range(v) if scores[j] > scores[i] or (scores[j] == scores[i] and j < i))
        if before < k:
            sel.append(i)
    return np.array(sel + [-1] * (k - len(sel)), np.int32)


@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_rank_count_definition_with_ties(seed):
    g = np.random.default_rng(seed)
    R, nc = 5, 40
    scores = g.integers(-3, 4, (R, nc)).astype(np.float64)  # many exact ties
    scores[:, ::7] *= -0.0 if seed % 2 else 1.0
    vis = g.integers(0, nc + 1, R).astype(np.int32)
    for k in (1, 3, 8, 40, 55):
        got = oracle.select_topk(scores, vis, k)
        for r in range(R):
            np.testing.assert_array_equal(got[r], rank_count_topk(scores[r], vis[r], k))


def test_topk_special_cases():
    nc = 20
    eq = np.full((1, nc), 0.25)
    np.testing.assert_array_equal(oracle.select_topk(eq, [nc], 6)[0], np.arange(6))
    sc = np.random.default_rng(9).standard_normal((1, nc))
    np.testing.assert_array_equal(oracle.select_topk(sc, [12], 16)[0],
                                  np.r_[np.arange(12), -np.ones(4)])
    np.testing.assert_array_equal(oracle.select_topk(sc, [0], 4)[0], -np.ones(4))
    z = np.zeros((1, 4))
    z[0, 0] = -0.0
    z[0, 2] = 0.0
    z[0, 1] = -1.0
    z[0, 3] = -1.0
    np.testing.assert_array_equal(oracle.select_topk(z, [4], 1)[0], [0])
    np.testing.assert_array_equal(oracle.select_topk(z, [4], 2)[0], [0, 2])


def test_topk_nan_is_rejected():
    with pytest.raises(oracle.OracleError):
        oracle.select_topk(np.array([[1.0, np.nan]]), [2], 1)


def test_index_topk_invisible_never_selected():
    g = np.random.default_rng(4)
    nc, HI, dI = 16, 2, 4
    kI = f32(g.standard_normal((1, nc, dI)))
    kI[0, 10:] = 50.0  # huge but invisible
    qI = f32(np.abs(g.standard_normal((1, 1, HI, dI))))
    w = f32(np.ones((1, 1, HI)))
    idx, sc = oracle.index_topk(qI, w, kI, np.array([40], np.int32), k=4)
    assert np.all(idx[0, 0] < 10) and np.all(np.diff(idx[0, 0]) > 0)
