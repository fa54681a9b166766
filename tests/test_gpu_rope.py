"""GPU parity of QK-norm and partial RoPE against the fp64 oracle: the
standalone kernel (csa_norm_rope) in every flag combination and position
rule, in place, at a million rows (sampled); and the attention with the
query's norm / rotation and the output's inverse rotation fused in
(csa_attend_rope, hca_attend_rope), stage-wise (caches prepared by the
oracle) and chained (caches prepared by csa_norm_rope on the GPU).

Definition: "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part
V", "The attention: compress, then select", third detail.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.helpers import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu

csa = pytest.importorskip("compressed_sparse_long_03_b200")
torch = pytest.importorskip("torch")

ODT = {"f32": oracle.F32, "bf16": oracle.BF16}
FLAGS = {"norm+rope": 3, "rope": 2, "norm": 1, "inverse": 6}


def _oracle_nr(x, pos, gamma, flags, rope_dim, base=10000.0, eps=1e-6):
    return oracle.norm_rope(x, pos, gamma=gamma, eps=eps, rope_dim=rope_dim, base=base,
                            norm=bool(flags & 1), rotate=bool(flags & 2), inverse=bool(flags & 4))


@pytest.mark.parametrize("dt,d", [("bf16", 128), ("bf16", 64), ("f32", 128), ("f32", 64)])
@pytest.mark.parametrize("flag", list(FLAGS))
@pytest.mark.parametrize("mode", ["pos", "lens", "strided"])
def test_norm_rope(dt, d, flag, mode):
    flags = FLAGS[flag]
    seed = 900 + d + flags
    R, G, rope_dim = 1000, 3, d // 2
    x = W.normal(seed, "x", (R, G, d), 1.0, dt)
    gamma = W.normal(seed, "q_gamma", (d,), 1.0, dt)
    g = np.random.default_rng(seed)
    kw = {}
    if mode == "pos":
        pos = g.integers(0, 1 << 21, R).astype(np.int32)
        kw = dict(pos=to_dev(pos))
    elif mode == "lens":
        Tq = 4
        lens = g.integers(Tq, 1 << 20, R // Tq).astype(np.int32)
        pos = (np.repeat(lens, Tq) - Tq + np.tile(np.arange(Tq), R // Tq)).astype(np.int64)
        kw = dict(lens=to_dev(lens), Tq=Tq)
    else:
        Tq, stride, off = 250, 128, 3
        pos = stride * (np.arange(R) % Tq) + off
        kw = dict(Tq=Tq, pos_stride=stride, pos_offset=off)
    y = csa.csa_norm_rope(to_dev(x), gamma=to_dev(gamma), rope_dim=rope_dim, flags=flags, **kw)
    csa.check_device_error()
    ref = _oracle_nr(x, pos, gamma, flags, rope_dim)
    assert_close(to_host(y), ref, dt, f"norm_rope {flag} {mode}")


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_norm_rope_in_place_and_full_rotation(dt):
    d, R, G = 128, 37, 5
    x = W.normal(31, "x", (R, G, d), 3.0, dt)
    pos = np.arange(R, dtype=np.int32) * 977
    t = to_dev(x)
    out = csa.csa_norm_rope(t, t, pos=to_dev(pos), rope_dim=d, rope_base=500.0, flags=3, eps=0.0)
    assert out.data_ptr() == t.data_ptr()
    csa.check_device_error()
    assert_close(to_host(t), _oracle_nr(x, pos, None, 3, d, base=500.0, eps=0.0), dt, "in place, r = d")


def test_norm_rope_million_rows_sampled():
    """A 1M-entry bf16 cache of stride 4 (positions 4 i up to 2^22): every
    row checked on 4096 sampled rows, and the unsampled rest checked by the
    norm of each row (rotation keeps it; RMSNorm with gamma = 1 sets the
    mean square to 1 / (1 + eps / ms))."""
    d, nc, B = 128, 1 << 19, 2
    x = W.normal(77, "x", (B * nc, 1, d), 1.0, "bf16")
    y = csa.csa_norm_rope(to_dev(x), Tq=nc, pos_stride=4, rope_dim=64, flags=3)
    csa.check_device_error()
    got = to_host(y)
    rows = np.random.default_rng(5).choice(B * nc, 4096, replace=False)
    pos = 4 * (rows % nc)
    assert_close(got[rows], _oracle_nr(x[rows], pos, None, 3, 64), "bf16", "sampled rows")
    ms = (oracle.values(got).reshape(B * nc, d) ** 2).mean(-1)
    assert np.abs(ms - 1.0).max() < 0.02


def _ring_positions(lens, n_tok):
    """Position of the token each ring row holds: the latest s < lens[b]
    with s = row (mod n_tok)."""
    j = np.arange(n_tok)[None, :]
    last = lens[:, None] - 1
    return np.where(last >= j, j + n_tok * ((last - j) // n_tok), 0)


def _stage_inputs(dt, d, H, B, Tq, nc, n_tok, m, seed, lens):
    """Raw q, and caches normalised and rotated by the oracle (rounded to
    dt): entry i at m i, window-ring rows at their tokens' positions."""
    q = W.normal(seed, "q", (B, Tq, H, d), 1.0, dt)
    kv = W.normal(seed, "kv", (B, nc, d), 1.0, dt)
    tok = W.normal(seed, "win", (B, n_tok, d), 1.0, dt)
    gq = W.normal(seed, "q_gamma", (d,), 1.0, dt)
    gk = W.normal(seed, "kv_gamma", (d,), 1.0, dt)
    kv_r = oracle.round_to(_oracle_nr(kv[:, :, None, :], m * np.arange(nc)[None, :].repeat(B, 0), gk, 3,
                                      64)[:, :, 0, :], ODT[dt])
    tok_r = oracle.round_to(_oracle_nr(tok[:, :, None, :], _ring_positions(lens, n_tok), gk, 3,
                                       64)[:, :, 0, :], ODT[dt])
    return q, kv, tok, gq, gk, kv_r, tok_r


def _oracle_attend_rope(q, kv_r, tok_r, gq, lens, dt, idx=None, m=4, window=128, sink=None):
    B, Tq = q.shape[:2]
    t = (lens[:, None] - Tq + np.arange(Tq)[None, :]).astype(np.int64)
    q_r = oracle.round_to(_oracle_nr(q, t, gq, 3, 64), ODT[dt])
    o = oracle.attend(q_r, kv_r, tok_r, lens, idx=idx, window=window, m=m, sink=sink)
    return oracle.norm_rope(o.astype(np.float32), t, norm=False, rope_dim=64, inverse=True)


@pytest.mark.parametrize("dt,d,H,B,Tq,k,nc", [
    ("bf16", 128, 64, 1, 1, 1024, 5000),    # 1M-decode shapes: an 8-CTA cluster per row
    ("bf16", 128, 100, 1, 37, 256, 600),    # 4-CTA clusters, a partly padded lane quadrant
    ("bf16", 128, 64, 2, 150, 128, 300),    # one CTA per row, double-buffered tiles
    ("bf16", 64, 8, 1, 3, 64, 256),         # CUDA-core kernel, bf16
    ("f32", 128, 16, 2, 2, 64, 400),        # CUDA-core kernel, fp32
])
def test_csa_attend_rope(dt, d, H, B, Tq, k, nc):
    seed = 950 + H + Tq
    n_tok = 256
    lens = np.array([4 * nc, 4 * nc - 3][:B], np.int32)
    q, kv, tok, gq, gk, kv_r, tok_r = _stage_inputs(dt, d, H, B, Tq, nc, n_tok, 4, seed, lens)
    vis = oracle.visible(lens, B, Tq, 4)
    g = np.random.default_rng(seed)
    idx = np.full((B, Tq, k), -1, np.int32)
    for b in range(B):
        for tq in range(Tq):
            n = min(int(vis[b, tq]), k - 3)
            idx[b, tq, :n] = np.sort(g.choice(int(vis[b, tq]), n, replace=False))
    sink = g.standard_normal(H).astype(np.float32)
    out = csa.csa_attend_rope(to_dev(q), to_dev(kv_r), to_dev(tok_r), to_dev(idx), to_dev(lens),
                              q_gamma=to_dev(gq), sink=to_dev(sink))
    csa.check_device_error()
    ref = _oracle_attend_rope(q, kv_r, tok_r, gq, lens, dt, idx=idx, sink=sink)
    assert_close(to_host(out), ref, dt, "csa_attend_rope")


@pytest.mark.parametrize("dt,d,H,B", [("bf16", 128, 64, 4), ("f32", 64, 8, 2)])
def test_hca_attend_rope(dt, d, H, B):
    seed, nc, m, n_tok = 970 + H, 300, 128, 128
    lens = (m * nc - np.arange(B) * 77).astype(np.int32)
    q, kv, tok, gq, gk, kv_r, tok_r = _stage_inputs(dt, d, H, B, 1, nc, n_tok, m, seed, lens)
    out = csa.hca_attend_rope(to_dev(q), to_dev(kv_r), to_dev(tok_r), to_dev(lens), m=m, q_gamma=to_dev(gq))
    csa.check_device_error()
    ref = _oracle_attend_rope(q, kv_r, tok_r, gq, lens, dt, m=m)
    assert_close(to_host(out), ref, dt, "hca_attend_rope")


def test_decode_chain_at_one_million_tokens():
    """The whole QK-norm / RoPE chain on the GPU at the 1M-decode shapes:
    csa_norm_rope prepares the entry cache (stride 4) and the window ring,
    csa_attend_rope normalises and rotates q and turns the output back;
    against the oracle chain on the same raw inputs (each cache element may
    be one bf16 ulp from the oracle's rounding: within the bf16 bound)."""
    dt, d, H, B, nc, k, n_tok = "bf16", 128, 64, 2, 262144, 1024, 128
    lens = np.array([4 * nc, 4 * nc - 5], np.int32)
    q, kv, tok, gq, gk, kv_r, tok_r = _stage_inputs(dt, d, H, B, 1, nc, n_tok, 4, 990, lens)
    # one head vector per row: [B][rows][1][d]
    d_kv = csa.csa_norm_rope(to_dev(kv).view(B, nc, 1, d), gamma=to_dev(gk), Tq=nc, pos_stride=4, rope_dim=64,
                             flags=3).view(B, nc, d)
    ring_pos = _ring_positions(lens, n_tok).astype(np.int32)
    d_tok = csa.csa_norm_rope(to_dev(tok).view(B, n_tok, 1, d), gamma=to_dev(gk), pos=to_dev(ring_pos),
                              rope_dim=64, flags=3).view(B, n_tok, d)
    g = np.random.default_rng(3)
    idx = np.stack([np.sort(g.choice(int(l) // 4, k, replace=False)) for l in lens]).astype(np.int32)[:, None]
    out = csa.csa_attend_rope(to_dev(q), d_kv, d_tok, to_dev(idx), to_dev(lens), q_gamma=to_dev(gq))
    csa.check_device_error()
    ref = _oracle_attend_rope(q, kv_r, tok_r, gq, lens, dt, idx=idx)
    assert_close(to_host(out), ref, dt, "1M chain")


def test_bad_arguments_are_errors():
    x = torch.zeros(4, 1, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(csa.CsaError):
        csa.csa_norm_rope(x, rope_dim=63)
    with pytest.raises(csa.CsaError):
        csa.csa_norm_rope(x, rope_dim=130)
    with pytest.raises(csa.CsaError):
        csa.csa_norm_rope(x, flags=csa.NR_INVERSE)
    with pytest.raises(csa.CsaError):
        csa.csa_norm_rope(torch.zeros(4, 1, 32, device="cuda"))
    q = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(1, 8, 128, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(1, 1, 4, dtype=torch.int32, device="cuda")
    lens = torch.tensor([8], dtype=torch.int32, device="cuda")
    with pytest.raises(csa.CsaError):
        csa.csa_attend_rope(q, kv, kv, idx, lens, flags=csa.NR_ROTATE | csa.NR_INVERSE)
