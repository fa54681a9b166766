"""GPU tests of the layer-pair scheduler (csa_hca_pair_decode) on the ragged
CSA + HCA pair workload (B = 64, n_b ~ U{65536..262144}): its results equal
those of the three separate calls bit for bit (the same kernels on the same
inputs; the scoring kernel's reduced grid does not change which tile
computes an entry), match the oracle on sampled sequences, and replay from
a CUDA graph captured with both branches.

Definition: "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part
V", "The attention: compress, then select" (interleaved CSA and HCA layers).
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.helpers import assert_close, to_dev, to_host, topk_set_difference_ok

pytestmark = pytest.mark.gpu

csa = pytest.importorskip("compressed_sparse_long_03_b200")
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def pair():
    wl = W.make(5)
    D = {n: to_dev(wl[n]) for n in wl.arrays}
    return wl, D


def _run_pair(wl, D, **kw):
    s = wl.sizes
    return csa.csa_hca_pair_decode(D["q"], D["qI"], D["w"], D["kI"], D["kv"], D["q2"], D["hkv"], D["win"],
                                   D["lens"], s["k"], m=s["m"], window=s["window"], **kw)


def test_pair_equals_the_separate_calls(pair):
    wl, D = pair
    s = wl.sizes
    idx, out_c, out_h = _run_pair(wl, D)
    csa.check_device_error()
    ref_idx = csa.csa_index_topk(D["qI"], D["w"], D["kI"], D["lens"], s["k"])
    ref_c = csa.csa_attend(D["q"], D["kv"], D["win"], ref_idx, D["lens"], window=s["window"])
    ref_h = csa.hca_attend(D["q2"], D["hkv"], D["win"], D["lens"], m=s["m"], window=s["window"])
    csa.check_device_error()
    assert torch.equal(idx, ref_idx)
    assert torch.equal(out_c, ref_c)
    assert torch.equal(out_h, ref_h)


def test_pair_against_the_oracle(pair):
    wl, D = pair
    s = wl.sizes
    k, window, m = s["k"], s["window"], s["m"]
    idx, out_c, out_h = map(to_host, _run_pair(wl, D))
    csa.check_device_error()
    for b in (0, 33, 63):
        sl = slice(b, b + 1)
        ref_idx, ref_sc = oracle.index_topk(wl["qI"][sl], wl["w"][sl], wl["kI"][sl], wl["lens"][sl], k)
        nd = topk_set_difference_ok(idx[sl].reshape(1, -1), ref_idx.reshape(1, -1), ref_sc.reshape(1, -1), k,
                                    "bf16")
        # stage-wise: the CSA attention over the GPU's own selection
        ref_c = oracle.attend(wl["q"][sl], wl["kv"][sl], wl["win"][sl], wl["lens"][sl], idx=idx[sl],
                              window=window)
        assert_close(out_c[sl], ref_c, "bf16", f"CSA seq {b} ({nd} boundary swaps)")
        ref_h = oracle.attend(wl["q2"][sl], wl["hkv"][sl], wl["win"][sl], wl["lens"][sl], idx=None, m=m,
                              window=window)
        assert_close(out_h[sl], ref_h, "bf16", f"HCA seq {b}")


def test_pair_replays_from_a_cuda_graph(pair):
    wl, D = pair
    s = wl.sizes
    B = s["B"]
    idx = torch.empty(B, 1, s["k"], dtype=torch.int32, device="cuda")
    out_c = torch.empty_like(D["q"])
    out_h = torch.empty_like(D["q2"])
    ws = csa.index_topk_workspace(B, 1, s["nc"], False)

    def step():
        _run_pair(wl, D, idx_out=idx, out_csa=out_c, out_hca=out_h, workspace=ws)

    step()  # creates the library's second stream before the capture
    torch.cuda.synchronize()
    eager = (idx.clone(), out_c.clone(), out_h.clone())
    for t in (idx, out_c, out_h):
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    csa.check_device_error()
    assert torch.equal(idx, eager[0]) and torch.equal(out_c, eager[1]) and torch.equal(out_h, eager[2])
