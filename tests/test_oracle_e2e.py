"""End-to-end pin of the oracle's CSA layer on tiny inputs, against a closed
form that does not use the oracle: with W=0 and beta=0 the compressor is a
mean pool (NumPy), and with k >= the visible entries the layer is textbook
attention (PyTorch fp64) over the pooled entries plus the window.

Definitions: "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part
V", "The attention: compress, then select" and its three details.
"""
import numpy as np
import torch

import oracle


def test_csa_layer_closed_form_tiny():
    g = np.random.default_rng(42)
    B, n, H, d, HI, dI, window = 2, 23, 3, 8, 2, 4, 6
    lens = np.array([23, 18], np.int32)
    x = g.standard_normal((B, n, d)).astype(np.float32)
    kx = g.standard_normal((B, n, dI)).astype(np.float32)
    q = g.standard_normal((B, 1, H, d)).astype(np.float32)
    qI = g.standard_normal((B, 1, HI, dI)).astype(np.float32)
    w = g.standard_normal((B, 1, HI)).astype(np.float32)
    z = lambda k: np.zeros((k, k), np.float32)
    C = oracle.csa_compress(x, lens, z(d), z(d), np.zeros((8, d), np.float32))
    KI = oracle.csa_compress(kx, lens, z(dI), z(dI), np.zeros((8, dI), np.float32))
    Cr = oracle.round_to(C, oracle.F32)
    KIr = oracle.round_to(KI, oracle.F32)
    k = 16
    idx, _ = oracle.index_topk(qI, w, KIr, lens, k)
    out = oracle.attend(q, Cr, x, lens, idx=idx, window=window)
    X = x.astype(np.float64)
    for b in range(B):
        t = int(lens[b]) - 1
        v = (t + 1) // 4
        assert list(idx[b, 0][:v]) == list(range(v)) and np.all(idx[b, 0][v:] == -1)
        pooled = [X[b, max(0, 4 * (i - 1)):min(int(lens[b]), 4 * i + 4)].mean(0) for i in range(v)]
        pooled = np.array(pooled, np.float32).astype(np.float64)  # the cache is stored in fp32
        keys = np.concatenate([pooled, X[b, t - window + 1:t + 1]])
        qt = torch.from_numpy(q[b, 0].astype(np.float64))[:, None]
        kt = torch.from_numpy(keys)[None].expand(H, -1, -1)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt)[:, 0].numpy()
        np.testing.assert_allclose(out[b, 0], ref, rtol=1e-6, atol=1e-7)
