"""Shared helpers for the parity tests: host <-> device marshalling of the
workload arrays and the tolerance checks.

Tolerances (problem statement): fp32 outputs max-abs 1e-5; bf16 outputs
|gpu - ref| <= 2e-2 + 1e-2 |ref|.  Indexer scores are fp32 sums of exact
bf16 x bf16 products (or fp32 products), compared with the fp64 oracle at
1e-5 (1 + |s|) for fp32 inputs and 1e-3 (1 + |s|) for bf16 inputs: 128-term
dot products accumulated in fp32 carry relative errors of order 1e-6, so the
bound leaves two orders of margin for accumulation order.
"""
import numpy as np

try:
    import torch
except Exception:  # pragma: no cover
    torch = None

F32_ATOL = 1e-5
BF16_ATOL, BF16_RTOL = 2e-2, 1e-2
SCORE_EPS = {"f32": 1e-5, "bf16": 1e-3}
# Scores computed from caches that the GPU chain built itself: each bf16 cache
# element may sit one bf16 ulp (2^-8 relative) away from the oracle's rounding
# of the exact value, so the end-to-end score bound is the looser 1e-2 (1+|s|).
CHAIN_EPS = {"f32": 1e-5, "bf16": 1e-2}


def to_dev(a, device="cuda"):
    """numpy float32 / bf16-bits(uint16) / int32 -> torch CUDA tensor."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a).to(device)


def to_host(t):
    """torch tensor -> numpy (bf16 -> uint16 bits)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def values(a):
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def assert_close(got, ref64, dt, what=""):
    """got: numpy output in storage dtype; ref64: oracle fp64 values."""
    g = values(got)
    if dt == "f32":
        err = np.abs(g - ref64)
        assert err.max(initial=0.0) <= F32_ATOL, f"{what}: max-abs {err.max():.3g} > {F32_ATOL}"
    else:
        bound = BF16_ATOL + BF16_RTOL * np.abs(ref64)
        bad = np.abs(g - ref64) > bound
        assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside 2e-2+1e-2|ref|, "
                               f"worst {np.abs(g - ref64).max():.3g}")


def assert_scores_close(gpu_scores, ref64, vis, dt, what="scores", eps=None):
    eps = SCORE_EPS[dt] if eps is None else eps
    for r in range(ref64.shape[0]):
        v = int(vis[r])
        g = gpu_scores[r, :v].astype(np.float64)
        ref = ref64[r, :v]
        bad = np.abs(g - ref) > eps * (1 + np.abs(ref))
        assert not bad.any(), f"{what} row {r}: {int(bad.sum())} of {v} beyond {eps}(1+|s|)"
        assert np.all(np.isneginf(gpu_scores[r, v:])), f"{what} row {r}: invisible entries not -inf"


def topk_set_difference_ok(gpu_idx, ref_idx, ref_scores, k, dt, eps=None):
    """Level (ii): the GPU and oracle index sets may differ only in entries
    whose oracle score lies within eps of the oracle's k-th score.  Returns
    the number of differing entries (asserts the rest)."""
    eps = SCORE_EPS[dt] if eps is None else eps
    diff = 0
    for r in range(gpu_idx.shape[0]):
        a = set(int(i) for i in gpu_idx[r] if i >= 0)
        b = set(int(i) for i in ref_idx[r] if i >= 0)
        if a == b:
            continue
        assert len(a) == len(b), f"row {r}: {len(a)} vs {len(b)} selected"
        kth = min(ref_scores[r, i] for i in b)
        for i in a ^ b:
            assert abs(ref_scores[r, i] - kth) <= eps * (1 + abs(kth)), (
                f"row {r}: entry {i} (score {ref_scores[r, i]}) differs, k-th score {kth}")
        diff += len(a - b)
    return diff
