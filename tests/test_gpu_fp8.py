"""GPU parity of FP8 cache entries against the fp64 oracle: the quantiser
bit for bit (codes, scales and the kept RoPE dims, edge values included),
and the attention over FP8 entries (csa_attend_fp8, hca_attend_fp8) against
the oracle's attention over the dequantised entries, stage-wise and through
the GPU quantiser at the 1M-decode shapes.

Definition: "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part
V", "The KV cache, recomputed".
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.helpers import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu

csa = pytest.importorskip("compressed_sparse_long_03_b200")
torch = pytest.importorskip("torch")


def _edge_rows(d, dt):
    """Rows that exercise the format's corners: a zero block, values that
    saturate, values below the smallest subnormal step, -0.0, ties."""
    x = np.zeros((6, d), np.float32)
    x[1, :64] = np.linspace(-500, 500, 64)            # amax 500: X = 0, |x| > 448 saturates
    x[2, :64] = 2.0 ** -12
    x[2, 0] = 300.0                                    # X = 0: 2^-12 rounds to 0
    x[3, :64] = -0.0
    x[3, 1] = 1.0
    x[4, :64] = np.array([256.0, 1.0625, 1.1875, 17.0, 2.0 ** -10, 3 * 2.0 ** -10] + [0.0] * 58)
    x[5, :] = 3.0 * 2.0 ** 100
    return x if dt == "f32" else W.bf16_bits(x)


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("d,r", [(128, 64), (256, 64), (64, 0), (192, 64)])
def test_quantize_fp8_bit_exact(dt, d, r):
    x = W.normal(40 + d + r, "kv", (1000, d), 2.0, dt)
    x = np.concatenate([x, _edge_rows(d, dt)])
    fp8, sc, rope = csa.csa_quantize_fp8_entries(to_dev(x), rope_dim=r)
    csa.check_device_error()
    ref = oracle.quantize_fp8_entries(x, rope_dim=r)
    np.testing.assert_array_equal(to_host(fp8), ref[0])
    np.testing.assert_array_equal(to_host(sc), ref[1])
    np.testing.assert_array_equal(to_host(rope), ref[2])


def _planes(seed, B, nc, d=128):
    kv = W.normal(seed, "kv", (B, nc, d), 1.0, "bf16")
    fp8, sc, rope = oracle.quantize_fp8_entries(kv, rope_dim=64)
    deq = oracle.round_to(oracle.dequant_fp8_entries(fp8, sc, rope), oracle.BF16)
    return fp8, sc, rope, deq


@pytest.mark.parametrize("H,B,Tq,k,nc", [
    (64, 1, 1, 1024, 5000),    # 1M-decode shapes: an 8-CTA cluster per row
    (100, 1, 37, 256, 600),    # 4-CTA clusters, a partly padded lane quadrant
    (64, 2, 150, 128, 300),    # one CTA per row, double-buffered tiles
])
def test_csa_attend_fp8(H, B, Tq, k, nc):
    seed, n_tok, d = 960 + H + Tq, 256, 128
    lens = np.array([4 * nc, 4 * nc - 3][:B], np.int32)
    q = W.normal(seed, "q", (B, Tq, H, d), 1.0, "bf16")
    tok = W.normal(seed, "win", (B, n_tok, d), 1.0, "bf16")
    fp8, sc, rope, deq = _planes(seed, B, nc)
    vis = oracle.visible(lens, B, Tq, 4)
    g = np.random.default_rng(seed)
    idx = np.full((B, Tq, k), -1, np.int32)
    for b in range(B):
        for tq in range(Tq):
            n = min(int(vis[b, tq]), k - 3)
            idx[b, tq, :n] = np.sort(g.choice(int(vis[b, tq]), n, replace=False))
    sink = g.standard_normal(H).astype(np.float32)
    out = csa.csa_attend_fp8(to_dev(q), to_dev(fp8), to_dev(sc), to_dev(rope), to_dev(tok), to_dev(idx),
                             to_dev(lens), sink=to_dev(sink))
    csa.check_device_error()
    ref = oracle.attend(q, deq, tok, lens, idx=idx, sink=sink)
    assert_close(to_host(out), ref, "bf16", "csa_attend_fp8")


def test_hca_attend_fp8():
    seed, B, H, nc, m, n_tok, d = 975, 4, 64, 300, 128, 128, 128
    lens = (m * nc - np.arange(B) * 77).astype(np.int32)
    q = W.normal(seed, "q", (B, 1, H, d), 1.0, "bf16")
    tok = W.normal(seed, "win", (B, n_tok, d), 1.0, "bf16")
    fp8, sc, rope, deq = _planes(seed, B, nc)
    out = csa.hca_attend_fp8(to_dev(q), to_dev(fp8), to_dev(sc), to_dev(rope), to_dev(tok), to_dev(lens), m=m)
    csa.check_device_error()
    ref = oracle.attend(q, deq, tok, lens, idx=None, m=m)
    assert_close(to_host(out), ref, "bf16", "hca_attend_fp8")


def test_fp8_decode_at_one_million_tokens():
    """The 1M-decode shapes end to end on the GPU: the bf16 entry cache
    quantised by csa_quantize_fp8_entries, then csa_attend_fp8 over 1024
    selected entries + the window, against the oracle's quantise / dequantise
    / attend; the GPU planes are also compared with the oracle's on sampled
    rows."""
    B, nc, H, d, k, n_tok = 2, 262144, 64, 128, 1024, 128
    lens = np.array([4 * nc, 4 * nc - 5], np.int32)
    kv = W.normal(991, "kv", (B, nc, d), 1.0, "bf16")
    q = W.normal(991, "q", (B, 1, H, d), 1.0, "bf16")
    tok = W.normal(991, "win", (B, n_tok, d), 1.0, "bf16")
    fp8, sc, rope = csa.csa_quantize_fp8_entries(to_dev(kv))
    g = np.random.default_rng(4)
    idx = np.stack([np.sort(g.choice(int(l) // 4, k, replace=False)) for l in lens]).astype(np.int32)[:, None]
    out = csa.csa_attend_fp8(to_dev(q), fp8, sc.view(B, nc), rope, to_dev(tok), to_dev(idx), to_dev(lens))
    csa.check_device_error()
    rows = idx[:, 0, :]
    sub = np.stack([kv[b, rows[b]] for b in range(B)])
    f_ref, s_ref, r_ref = oracle.quantize_fp8_entries(sub)
    f_gpu, s_gpu = to_host(fp8), to_host(sc)
    for b in range(B):
        np.testing.assert_array_equal(f_gpu[b, rows[b]], f_ref[b])
        np.testing.assert_array_equal(s_gpu[b, rows[b]], s_ref[b])
    deq = np.zeros((B, nc, d), np.uint16)
    dq_sub = oracle.round_to(oracle.dequant_fp8_entries(f_ref, s_ref, r_ref), oracle.BF16)
    for b in range(B):
        deq[b, rows[b]] = dq_sub[b]
    ref = oracle.attend(q, deq, tok, lens, idx=idx)
    assert_close(to_host(out), ref, "bf16", "1M FP8 decode")


def test_unsupported_shapes_are_errors():
    q = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16, device="cuda")
    tok = torch.zeros(1, 8, 128, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(1, 1, 4, dtype=torch.int32, device="cuda")
    lens = torch.tensor([8], dtype=torch.int32, device="cuda")
    f = torch.zeros(1, 6, 64, dtype=torch.uint8, device="cuda")        # nc_max = 6: not a multiple of 4
    s = torch.zeros(1, 8, dtype=torch.uint8, device="cuda")
    r = torch.zeros(1, 6, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(csa.CsaError):
        csa.csa_attend_fp8(q, f, s, r, tok, idx, lens)
    with pytest.raises(csa.CsaError):
        csa.csa_quantize_fp8_entries(torch.zeros(4, 100, dtype=torch.bfloat16, device="cuda"))
