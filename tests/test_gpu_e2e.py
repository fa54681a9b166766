"""End-to-end GPU parity of whole CSA / HCA layer steps on the five
workloads, against the fp64 oracle run on the same seeded inputs.

The GPU chain runs entirely on the device (compress -> index/top-k ->
attend); the oracle chain runs on the host.  Stage results are compared
where they are defined (caches element by element, index sets at level (ii));
the final outputs are compared per query row wherever the two index sets
agree, and, in addition, the GPU attention is fed the oracle's index set so
that every row's output is checked."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.helpers import (CHAIN_EPS, assert_close, assert_scores_close, to_dev, to_host,
                           topk_set_difference_ok)

pytestmark = pytest.mark.gpu

csa = pytest.importorskip("compressed_sparse_long_03_b200")
torch = pytest.importorskip("torch")


def test_workload1_csa_decode_fp32():
    wl = W.make(1)
    s = wl.sizes
    k, window = s["k"], s["window"]
    D = {n: to_dev(wl[n]) for n in wl.arrays}
    C = csa.csa_compress(D["x"], D["lens"], D["Wa"], D["Wb"], D["beta"])
    KI = csa.csa_compress(D["kx"], D["lens"], D["kWa"], D["kWb"], D["kbeta"])
    sc = torch.empty(s["B"], 1, s["nc"], dtype=torch.float32, device="cuda")
    idx = csa.csa_index_topk(D["qI"], D["w"], KI, D["lens"], k, scores_out=sc)
    out = csa.csa_attend(D["q"], C, D["x"], idx, D["lens"], window=window)
    csa.check_device_error()

    C_ref = oracle.csa_compress(wl["x"], wl["lens"], wl["Wa"], wl["Wb"], wl["beta"])
    KI_ref = oracle.csa_compress(wl["kx"], wl["lens"], wl["kWa"], wl["kWb"], wl["kbeta"])
    assert_close(to_host(C), C_ref, "f32", "KV cache")
    assert_close(to_host(KI), KI_ref, "f32", "indexer-key cache")
    C_r, KI_r = oracle.round_to(C_ref, oracle.F32), oracle.round_to(KI_ref, oracle.F32)
    ref_idx, ref_sc = oracle.index_topk(wl["qI"], wl["w"], KI_r, wl["lens"], k)
    vis = oracle.visible(wl["lens"], s["B"], 1, 4).reshape(-1)
    assert_scores_close(to_host(sc).reshape(1, -1), ref_sc.reshape(1, -1), vis, "f32")
    nd = topk_set_difference_ok(to_host(idx).reshape(1, -1), ref_idx.reshape(1, -1),
                                ref_sc.reshape(1, -1), k, "f32")
    ref_out = oracle.attend(wl["q"], C_r, wl["x"], wl["lens"], idx=ref_idx, window=window)
    if nd == 0:
        assert_close(to_host(out), ref_out, "f32", "layer output")
    out2 = csa.csa_attend(D["q"], to_dev(C_r), D["x"], to_dev(ref_idx), D["lens"], window=window)
    assert_close(to_host(out2), ref_out, "f32", "layer output (oracle indices)")


def test_workload2_csa_prefill_sampled_rows():
    """8192 causal queries on the GPU; 24 query rows (early, window-edge and
    late positions) recomputed by the oracle."""
    wl = W.make(2)
    s = wl.sizes
    k, window = s["k"], s["window"]
    D = {n: to_dev(wl[n]) for n in wl.arrays}
    C = csa.csa_compress(D["x"], D["lens"], D["Wa"], D["Wb"], D["beta"])
    KI = csa.csa_compress(D["kx"], D["lens"], D["kWa"], D["kWb"], D["kbeta"])
    sc = torch.empty(1, s["Tq"], s["nc"], dtype=torch.float32, device="cuda")
    idx = csa.csa_index_topk(D["qI"], D["w"], KI, D["lens"], k, scores_out=sc)
    out = csa.csa_attend(D["q"], C, D["x"], idx, D["lens"], window=window)
    csa.check_device_error()
    idx, sc, out = to_host(idx), to_host(sc), to_host(out)

    C_r = oracle.round_to(oracle.csa_compress(wl["x"], wl["lens"], wl["Wa"], wl["Wb"], wl["beta"]), oracle.BF16)
    KI_r = oracle.round_to(oracle.csa_compress(wl["kx"], wl["lens"], wl["kWa"], wl["kWb"], wl["kbeta"]), oracle.BF16)
    g = np.random.default_rng(2)
    rows = np.unique(np.r_[[0, 2, 3, 4, 126, 127, 128, 2047, 2048, 2051, 8191],
                           g.integers(0, s["n"], 13)]).astype(np.int32)
    q_pos = rows[None, :]
    sub = lambda a: a[:, rows]
    ref_idx, ref_sc = oracle.index_topk(sub(wl["qI"]), sub(wl["w"]), KI_r, wl["lens"], k, q_pos)
    vis = oracle.visible(wl["lens"], 1, len(rows), 4, q_pos).reshape(-1)
    # the chain: scores from the GPU-built cache (bound CHAIN_EPS), the
    # selection bit-exact on the GPU's own scores
    assert_scores_close(sc[0, rows], ref_sc[0], vis, "bf16", eps=CHAIN_EPS["bf16"])
    np.testing.assert_array_equal(idx[0, rows], oracle.select_topk(sc[0, rows], vis, k))
    topk_set_difference_ok(idx[0, rows], ref_idx[0], ref_sc[0], k, "bf16", eps=CHAIN_EPS["bf16"])
    # stage-wise: the GPU indexer on the oracle's cache, at the tight bound
    sc2 = to_host(csa.csa_index_scores(to_dev(sub(wl["qI"])), to_dev(sub(wl["w"])), to_dev(KI_r),
                                       D["lens"], q_pos=to_dev(q_pos)))
    assert_scores_close(sc2[0], ref_sc[0], vis, "bf16")
    ref_out = oracle.attend(sub(wl["q"]), C_r, wl["x"], wl["lens"], idx=ref_idx, q_pos=q_pos, window=window)
    for j, r in enumerate(rows):
        if set(idx[0, r]) == set(ref_idx[0, j]):
            assert_close(out[0, r:r + 1], ref_out[0, j:j + 1], "bf16", f"row {r}")
    # every sampled row with the oracle's indices, through the GPU attention
    out2 = csa.csa_attend(to_dev(sub(wl["q"])), to_dev(C_r), D["x"], to_dev(ref_idx), D["lens"],
                          q_pos=to_dev(q_pos), window=window)
    assert_close(to_host(out2), ref_out, "bf16", "sampled rows (oracle indices)")


def test_workload5_pair_sampled_sequences():
    """B=64 ragged contexts: the CSA step (index/top-k + attend) and the HCA
    step of the layer pair on the GPU; 6 sequences recomputed by the oracle."""
    wl = W.make(5)
    s = wl.sizes
    k, window, m = s["k"], s["window"], s["m"]
    D = {n: to_dev(wl[n]) for n in wl.arrays}
    sc = torch.empty(s["B"], 1, s["nc"], dtype=torch.float32, device="cuda")
    idx = csa.csa_index_topk(D["qI"], D["w"], D["kI"], D["lens"], k, scores_out=sc)
    out_c = csa.csa_attend(D["q"], D["kv"], D["win"], idx, D["lens"], window=window)
    out_h = csa.hca_attend(D["q2"], D["hkv"], D["win"], D["lens"], m=m, window=window)
    csa.check_device_error()
    idx, sc, out_c, out_h = map(to_host, (idx, sc, out_c, out_h))
    for b in (0, 1, 17, 31, 50, 63):
        sl = slice(b, b + 1)
        ref_idx, ref_sc = oracle.index_topk(wl["qI"][sl], wl["w"][sl], wl["kI"][sl], wl["lens"][sl], k)
        vis = oracle.visible(wl["lens"][sl], 1, 1, 4).reshape(-1)
        assert_scores_close(sc[sl].reshape(1, -1), ref_sc.reshape(1, -1), vis, "bf16")
        np.testing.assert_array_equal(idx[sl].reshape(1, -1),
                                      oracle.select_topk(sc[sl].reshape(1, -1), vis, k))
        nd = topk_set_difference_ok(idx[sl].reshape(1, -1), ref_idx.reshape(1, -1),
                                    ref_sc.reshape(1, -1), k, "bf16")
        ref_c = oracle.attend(wl["q"][sl], wl["kv"][sl], wl["win"][sl], wl["lens"][sl], idx=ref_idx,
                              window=window)
        if nd == 0:
            assert_close(out_c[sl], ref_c, "bf16", f"CSA seq {b}")
        ref_h = oracle.attend(wl["q2"][sl], wl["hkv"][sl], wl["win"][sl], wl["lens"][sl], idx=None,
                              m=m, window=window)
        assert_close(out_h[sl], ref_h, "bf16", f"HCA seq {b}")
