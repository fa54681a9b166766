"""GPU parity of csa_index_topk against the fp64 oracle.

Scores are compared element by element; the selection is checked at two
levels: (i) bit-exact -- the oracle's selector applied to the GPU's own fp32
scores must give the GPU's index list exactly (isolates the selection kernel
from rounding); (ii) end to end -- GPU and oracle index sets may differ only
in entries whose oracle score lies within the score tolerance of the
oracle's k-th score."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.helpers import (assert_scores_close, to_dev, to_host, topk_set_difference_ok)

pytestmark = pytest.mark.gpu

csa = pytest.importorskip("compressed_sparse_long_03_b200")
torch = pytest.importorskip("torch")


def run_gpu(qI, w, kI, lens, k, q_pos=None):
    B, Tq = qI.shape[:2]
    nc = kI.shape[1]
    sc = torch.empty(B, Tq, nc, dtype=torch.float32, device="cuda")
    idx = csa.csa_index_topk(to_dev(qI), to_dev(w), to_dev(kI), to_dev(lens), k,
                             q_pos=None if q_pos is None else to_dev(q_pos), scores_out=sc)
    csa.check_device_error()
    return to_host(idx), to_host(sc)


def check_all(qI, w, kI, lens, k, dt, q_pos=None, expect_exact=False):
    B, Tq = qI.shape[:2]
    idx, sc = run_gpu(qI, w, kI, lens, k, q_pos)
    vis = oracle.visible(lens, B, Tq, 4, q_pos).reshape(-1)
    nc = kI.shape[1]
    # (i) selection bit-exact on the GPU's own scores
    ref_sel = oracle.select_topk(sc.reshape(-1, nc), vis, k)
    np.testing.assert_array_equal(idx.reshape(-1, k), ref_sel)
    # scores vs oracle, then (ii) end-to-end set agreement
    ref_idx, ref_sc = oracle.index_topk(qI, w, kI, lens, k, q_pos)
    assert_scores_close(sc.reshape(-1, nc), ref_sc.reshape(-1, nc), vis, dt)
    nd = topk_set_difference_ok(idx.reshape(-1, k), ref_idx.reshape(-1, k), ref_sc.reshape(-1, nc), k, dt)
    if expect_exact:
        assert nd == 0
    return idx, sc


@pytest.mark.parametrize("nc,Tq", [(300, 1), (1000, 2)])
def test_fp32_small(nc, Tq):
    """Workload 1's shapes (HI=4, dI=32, k=64, fp32), ragged lengths."""
    seed = 7 + nc
    B = 2
    lens = np.array([4 * nc, 4 * nc - 197], np.int32)
    qI = W.normal(seed, "qI", (B, Tq, 4, 32), 1.0, "f32")
    w = W.normal(seed, "w", (B, Tq, 4), 1.0, "f32")
    kI = W.normal(seed, "kI", (B, nc, 32), 1.0, "f32")
    check_all(qI, w, kI, lens, 64, "f32")


@pytest.mark.parametrize("nc", [5000, 16384 + 77, 30000, 70000])
def test_bf16_tiles_and_cluster_sizes(nc):
    """HI=64 x dI=128 bf16, k=1024: sizes that select 1, 2, 4 and 8 CTAs per
    query row, with partial last tiles."""
    seed = 100 + nc
    B = 3
    lens = np.array([4 * nc, 4 * nc - 4 * (nc // 3) - 1, 4 * nc - 5], np.int32)
    qI = W.normal(seed, "qI", (B, 1, 64, 128), 1.0, "bf16")
    w = W.normal(seed, "w", (B, 1, 64), 128 ** -0.5, "bf16")
    kI = W.normal(seed, "kI", (B, nc, 128), 1.0, "bf16")
    check_all(qI, w, kI, lens, 1024, "bf16")


@pytest.mark.parametrize("HI,dI", [(4, 128), (16, 64), (24, 128), (100, 64), (128, 128), (64, 32)])
def test_bf16_head_and_dim_shapes(HI, dI):
    """Indexer head counts that pad to 16/32/128 tensor-core columns, key
    widths of one and two 128-byte slices, and the 32-wide keys that take the
    CUDA-core kernel; several query rows per sequence at explicit positions."""
    seed = 1000 + HI + dI
    B, Tq, nc = 2, 3, 1000
    lens = np.array([4 * nc, 4 * nc - 333], np.int32)
    q_pos = np.array([[3999, 2500, 130], [3666, 515, 1]], np.int32)
    qI = W.normal(seed, "qI", (B, Tq, HI, dI), 1.0, "bf16")
    w = W.normal(seed, "w", (B, Tq, HI), 1.0 / HI, "bf16")
    kI = W.normal(seed, "kI", (B, nc, dI), 1.0, "bf16")
    check_all(qI, w, kI, lens, 200, "bf16", q_pos=q_pos)


@pytest.mark.parametrize("HI,dI", [(16, 128), (32, 64), (64, 128), (128, 64)])
def test_grouped_query_rows(HI, dI):
    """Several query rows of a sequence share each key tile (units of up to
    four rows): 7 rows per sequence (a partial last unit whose query block
    reaches into the next sequence's rows), two sequences of different
    lengths, positions out of order; scores of every row (-inf where not
    visible) and the selections checked."""
    seed = 2000 + HI + dI
    B, Tq, nc = 2, 7, 3000
    lens = np.array([4 * nc, 4 * nc - 5001], np.int32)
    q_pos = np.array([[11999, 20, 3, 7000, 4, 11998, 5555],
                      [6998, 0, 6000, 129, 131, 6997, 2]], np.int32)
    qI = W.normal(seed, "qI", (B, Tq, HI, dI), 1.0, "bf16")
    w = W.normal(seed, "w", (B, Tq, HI), 1.0 / HI, "bf16")
    kI = W.normal(seed, "kI", (B, nc, dI), 1.0, "bf16")
    idx, sc = check_all(qI, w, kI, lens, 300, "bf16", q_pos=q_pos)
    vis = oracle.visible(lens, B, Tq, 4, q_pos)
    for b in range(B):
        for tq in range(Tq):
            assert np.all(np.isneginf(sc[b, tq, vis[b, tq]:]))


def test_causal_rows_prefill_like():
    """Many query rows at increasing positions (v from 0 to > k): visibility
    and the v <= k / v == 0 paths."""
    seed = 5
    nc, Tq, k = 700, 48, 512
    lens = np.array([4 * nc], np.int32)
    q_pos = np.sort(np.random.default_rng(seed).integers(0, 4 * nc, (1, Tq))).astype(np.int32)
    q_pos[0, :4] = [0, 2, 3, 4]
    qI = W.normal(seed, "qI", (1, Tq, 64, 128), 1.0, "bf16")
    w = W.normal(seed, "w", (1, Tq, 64), 128 ** -0.5, "bf16")
    kI = W.normal(seed, "kI", (1, nc, 128), 1.0, "bf16")
    idx, _ = check_all(qI, w, kI, lens, k, "bf16", q_pos=q_pos)
    assert np.all(idx[0, 0] == -1)                   # t = 0: nothing visible
    assert idx[0, 3, 0] == 0 and np.all(idx[0, 3, 1:] == -1)   # t = 4: entry 0 only


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("nc", [20000, 3000])  # 1024- and 256-thread selection CTAs
def test_all_equal_scores_select_first_k(dt, nc):
    k = 1024
    row = W.normal(9, "kI", (1, 1, 128), 1.0, dt)
    kI = np.repeat(row, nc, axis=1)
    qI = W.normal(9, "qI", (1, 1, 64, 128), 1.0, dt)
    w = W.normal(9, "w", (1, 1, 64), 1.0, dt)
    idx, sc = check_all(qI, w, kI, np.array([4 * nc], np.int32), k, dt, expect_exact=True)
    np.testing.assert_array_equal(idx[0, 0], np.arange(k))


def test_exact_zero_ties_straddle_threshold():
    """Half the keys point away from every indexer query, so their scores are
    exactly 0 (every head's ReLU is 0); with positive head weights the rest
    score > 0, and k larger than the positive set forces the tie rule onto
    the zeros."""
    nc, k = 6000, 4000
    g = np.random.default_rng(12)
    q = np.abs(g.standard_normal((1, 1, 64, 128))).astype(np.float32)
    keys = np.abs(g.standard_normal((1, nc, 128))).astype(np.float32)
    neg = g.random(nc) < 0.5
    keys[0, neg] *= -1
    w = np.abs(g.standard_normal((1, 1, 64))).astype(np.float32) / 8
    qI, kI, wb = W.bf16_bits(q), W.bf16_bits(keys), W.bf16_bits(w)
    idx, sc = check_all(qI, wb, kI, np.array([4 * nc], np.int32), k, "bf16", expect_exact=True)
    zeros = np.where(sc[0, 0] == 0)[0]
    npos = int((~neg).sum())
    assert len(zeros) == int(neg.sum())
    np.testing.assert_array_equal(np.sort(idx[0, 0]),
                                  np.sort(np.r_[np.where(~neg)[0], zeros[:k - npos]]))


def test_needle_workload_full_size():
    """Workload 4 at full size (B=4, 262,144 entries, 64x128 bf16, k=1024):
    all rows checked at both levels, and every planted needle is selected."""
    wl = W.make(4)
    idx, sc = check_all(wl["qI"], wl["w"], wl["kI"], wl["lens"], wl.sizes["k"], "bf16")
    for b, p in enumerate(wl["needle_pos"]):
        assert int(p) in set(idx[b, 0].tolist())


def test_deterministic_and_batch_invariant():
    nc = 40000
    seed = 77
    B = 3
    lens = np.array([4 * nc, 4 * nc - 9, 4 * nc - 1000], np.int32)
    qI = W.normal(seed, "qI", (B, 1, 64, 128), 1.0, "bf16")
    w = W.normal(seed, "w", (B, 1, 64), 128 ** -0.5, "bf16")
    kI = W.normal(seed, "kI", (B, nc, 128), 1.0, "bf16")
    a_idx, a_sc = run_gpu(qI, w, kI, lens, 1024)
    b_idx, b_sc = run_gpu(qI, w, kI, lens, 1024)
    np.testing.assert_array_equal(a_idx, b_idx)
    np.testing.assert_array_equal(a_sc.view(np.uint32), b_sc.view(np.uint32))
    one_idx, one_sc = run_gpu(qI[1:2], w[1:2], kI[1:2], lens[1:2], 1024)
    np.testing.assert_array_equal(one_idx[0], a_idx[1])
    np.testing.assert_array_equal(one_sc[0].view(np.uint32), a_sc[1].view(np.uint32))


def test_invalid_position_raises_device_error():
    nc = 100
    qI = W.normal(1, "qI", (1, 1, 4, 32), 1.0, "f32")
    w = W.normal(1, "w", (1, 1, 4), 1.0, "f32")
    kI = W.normal(1, "kI", (1, nc, 32), 1.0, "f32")
    lens = np.array([4 * nc], np.int32)
    idx = csa.csa_index_topk(to_dev(qI), to_dev(w), to_dev(kI), to_dev(lens), 8,
                             q_pos=to_dev(np.array([[4 * nc]], np.int32)))
    with pytest.raises(csa.CsaError):
        csa.check_device_error()
    assert np.all(to_host(idx) == -1)
    csa.check_device_error()  # cleared


def test_index_topk_matches_split_calls_and_reuses_workspace():
    """csa_index_topk against csa_index_scores + csa_topk on the same inputs
    (identical indices), twice through one workspace, with rows that have
    fewer visible entries than k."""
    seed, B, nc, k = 55, 4, 50000, 1024
    lens = np.array([4 * nc, 4 * nc - 3, 100 * 4, 3], np.int32)
    qI = W.normal(seed, "qI", (B, 1, 64, 128), 1.0, "bf16")
    w = W.normal(seed, "w", (B, 1, 64), 128 ** -0.5, "bf16")
    kI = W.normal(seed, "kI", (B, nc, 128), 1.0, "bf16")
    d = [to_dev(a) for a in (qI, w, kI, lens)]
    ws = csa.index_topk_workspace(B, 1, nc, False)
    a1 = to_host(csa.csa_index_topk(*d, k, workspace=ws))
    a2 = to_host(csa.csa_index_topk(*d, k, workspace=ws))
    sc = csa.csa_index_scores(*d)
    b1 = to_host(csa.csa_topk(sc, d[3], k))
    csa.check_device_error()
    np.testing.assert_array_equal(a1, a2)
    np.testing.assert_array_equal(a1, b1)
    vis = oracle.visible(lens, B, 1, 4).reshape(-1)
    np.testing.assert_array_equal(a1.reshape(B, k), oracle.select_topk(to_host(sc).reshape(B, -1), vis, k))


def test_kernel_timing_hook():
    nc = 4096
    qI = W.normal(3, "qI", (1, 1, 64, 128), 1.0, "bf16")
    w = W.normal(3, "w", (1, 1, 64), 0.1, "bf16")
    kI = W.normal(3, "kI", (1, nc, 128), 1.0, "bf16")
    lens = np.array([4 * nc], np.int32)
    csa.set_kernel_timing(True)
    try:
        csa.csa_index_topk(to_dev(qI), to_dev(w), to_dev(kI), to_dev(lens), 64)
        t = csa.kernel_timing()
    finally:
        csa.set_kernel_timing(False)
    assert len(t) == 2 and all(x > 0 for x in t)
