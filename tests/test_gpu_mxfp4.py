"""GPU parity of the MXFP4 indexer keys: the quantiser bit-exact against the
oracle's, and the indexer over FP4 keys against the oracle's indexer on the
oracle-dequantised keys (scores element by element, the selection
bit-exact on the GPU's own scores and set-equal to the oracle's within the
score tolerance), up to the full 1M-token decode workload."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.helpers import assert_scores_close, to_dev, to_host, topk_set_difference_ok

pytestmark = pytest.mark.gpu

csa = pytest.importorskip("compressed_sparse_long_03_b200")
torch = pytest.importorskip("torch")


def edge_keys(dI):
    """fp32 keys whose blocks hit every rounding case: midpoints, just off
    midpoints, saturation, zeros of both signs, an all-zero block, tiny and
    large scales."""
    g = np.random.default_rng(3)
    rows = []
    for X in (-20, -1, 0, 3, 30):
        row = g.standard_normal(dI).astype(np.float32)
        for blk in range(dI // 32):
            b = np.zeros(32, np.float32)
            b[0] = 4.0
            b[1:8] = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
            b[8:12] = [0.2501, 0.7499, 5.01, 7.9]
            b[12] = -0.0
            b[13:20] = -b[1:8]
            b[20:] = g.uniform(-6, 6, 12)
            row[32 * blk:32 * blk + 32] = b * np.float32(2.0 ** X)
        rows.append(row)
    rows.append(np.zeros(dI, np.float32))
    return np.stack(rows)[None]


@pytest.mark.parametrize("dt,dI", [("bf16", 128), ("bf16", 64), ("f32", 128)])
def test_quantize_bit_exact(dt, dI):
    k = W.normal(40 + dI, "kI", (3, 777, dI), 1.0, dt)
    if dt == "f32":
        e = edge_keys(dI)
        k = np.concatenate([k, np.repeat(e, 3, axis=0)[:, :, :]], axis=1)
    codes, scales = csa.csa_quantize_mxfp4(to_dev(k))
    c_ref, s_ref = oracle.quantize_mxfp4(k)
    np.testing.assert_array_equal(to_host(scales), s_ref)
    np.testing.assert_array_equal(to_host(codes), c_ref)


def check_fp4(qI, w, kI, lens, k, q_pos=None):
    B, Tq = qI.shape[:2]
    nc = kI.shape[1]
    codes, scales = csa.csa_quantize_mxfp4(to_dev(kI))
    sc = torch.empty(B, Tq, nc, dtype=torch.float32, device="cuda")
    idx = csa.csa_index_topk_mxfp4(to_dev(qI), to_dev(w), codes, scales, to_dev(lens), k,
                                   q_pos=None if q_pos is None else to_dev(q_pos), scores_out=sc)
    csa.check_device_error()
    idx, sc = to_host(idx), to_host(sc)
    c_ref, s_ref = oracle.quantize_mxfp4(kI)
    kdq = W.bf16_bits(oracle.dequant_mxfp4(c_ref, s_ref).astype(np.float32))  # exact bf16 values
    vis = oracle.visible(lens, B, Tq, 4, q_pos).reshape(-1)
    np.testing.assert_array_equal(idx.reshape(-1, k), oracle.select_topk(sc.reshape(-1, nc), vis, k))
    ref_idx, ref_sc = oracle.index_topk(qI, w, kdq, lens, k, q_pos)
    assert_scores_close(sc.reshape(-1, nc), ref_sc.reshape(-1, nc), vis, "bf16")
    topk_set_difference_ok(idx.reshape(-1, k), ref_idx.reshape(-1, k), ref_sc.reshape(-1, nc), k, "bf16")
    return idx, sc


@pytest.mark.parametrize("HI,dI,nc", [(64, 128, 5000), (16, 64, 3000), (128, 128, 40000), (24, 128, 1000)])
def test_index_topk_mxfp4(HI, dI, nc):
    seed = 50 + HI + dI
    B, Tq = 2, 2
    lens = np.array([4 * nc, 4 * nc - 777], np.int32)
    q_pos = np.array([[4 * nc - 1, 333], [4 * nc - 778, 4 * nc - 2000]], np.int32)
    qI = W.normal(seed, "qI", (B, Tq, HI, dI), 1.0, "bf16")
    w = W.normal(seed, "w", (B, Tq, HI), 1.0 / HI, "bf16")
    kI = W.normal(seed, "kI", (B, nc, dI), 1.0, "bf16")
    check_fp4(qI, w, kI, lens, 512, q_pos=q_pos)


def test_index_topk_mxfp4_full_1m_workload():
    """The 1M-token decode workload with its indexer keys quantised to MXFP4:
    every row checked, and every planted needle still selected."""
    wl = W.make(4)
    s = wl.sizes
    idx, _ = check_fp4(wl["qI"], wl["w"], wl["kI"], wl["lens"], s["k"])
    for b, p in enumerate(wl["needle_pos"]):
        assert p in set(idx[b, 0].tolist())
