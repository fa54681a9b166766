"""csa_index_topk_noalloc: the indexer + top-k entry point that allocates
nothing, for callers that may not allocate device memory during a call (an
engine whose memory pool already holds nearly all of the GPU, an allocator
that forbids allocations outside its pool, code where cudaMalloc / cudaFree
would synchronise the device).  Its scores live in a fixed device array of
the library; these tests check that it selects exactly what csa_index_topk
(with a caller workspace) selects, on calls in a row that leave different
contents behind in the shared array, and that oversized calls are refused.

The file name makes pytest collect it last."""
import ctypes

import numpy as np
import pytest

import workloads as W

csa = pytest.importorskip("compressed_sparse_long_03_b200")

CSA_ERR_WORKSPACE = -6
MAX_ELEMS = 2 << 20  # 8 MiB of fp32 scores


def test_noalloc_limit_and_rejection():
    """The stated limit, and a call one score past it fails before touching
    any pointer (no GPU needed: the size check comes first)."""
    L = csa.lib()
    assert csa.index_topk_noalloc_max_elems() == MAX_ELEMS
    B, Tq, HI, dI, k = 8, 1, 64, 128, 1024
    nc = MAX_ELEMS // (B * Tq) + 1
    rc = L.csa_index_topk_noalloc(None, None, None, None, None, B, Tq, HI, dI, nc, k,
                                  csa.BF16, None, None)
    assert rc == CSA_ERR_WORKSPACE
    assert "exceed the fixed scratch" in csa.last_error()
    # exactly at the limit the size check passes (and the NULL check fails)
    rc = L.csa_index_topk_noalloc(None, None, None, None, None, B, Tq, HI, dI, nc - 1, k,
                                  csa.BF16, None, None)
    assert rc == -1


def _inputs(seed, B, Tq, HI, dI, nc, lens):
    qI = W.normal(seed, "qI", (B, Tq, HI, dI), 1.0, "bf16")
    w = W.normal(seed, "w", (B, Tq, HI), 1.0, "bf16")
    kI = W.normal(seed, "kI", (B, nc, dI), 1.0, "bf16")
    return qI, w, kI, np.asarray(lens, np.int32)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point():
    """Three calls in a row through the C ABI, each compared with
    csa_index_topk on the same inputs.  Indices are integers computed by the
    same kernels from the same scores, so they must agree exactly.  The
    second call has shorter rows than the first (the array still holds the
    first call's longer rows), the third repeats the first."""
    import torch
    from tests.helpers import to_dev, to_host

    cases = [
        # seed, B, Tq, HI, dI, nc, lens, k, q_pos
        (101, 2, 1, 64, 128, 70000, [4 * 70000, 4 * 70000 - 4093], 1024, None),
        (202, 3, 2, 16, 64, 30000, [4 * 30000, 50001, 4 * 12000 + 3], 512,
         np.array([[4 * 30000 - 9, 4 * 30000 - 1], [50000, 20], [4 * 12000, 4 * 11000]], np.int32)),
    ]
    cases.append(cases[0])
    prev = None
    for seed, B, Tq, HI, dI, nc, lens, k, q_pos in cases:
        qI, w, kI, ln = _inputs(seed, B, Tq, HI, dI, nc, lens)
        dq, dw, dk, dl = to_dev(qI), to_dev(w), to_dev(kI), to_dev(ln)
        dp = None if q_pos is None else to_dev(q_pos)
        ref = csa.csa_index_topk(dq, dw, dk, dl, k, q_pos=dp)
        out = torch.full((B, Tq, k), -7, dtype=torch.int32, device="cuda")
        csa.csa_index_topk_noalloc(dq, dw, dk, dl, k, out, q_pos=dp)
        torch.cuda.synchronize()
        csa.check_device_error()
        got, want = to_host(out), to_host(ref)
        np.testing.assert_array_equal(got, want)
        assert (got >= -1).all() and (got[..., 0] >= 0).all()
        if prev is not None and seed == cases[0][0]:
            np.testing.assert_array_equal(got, prev)
        if seed == cases[0][0]:
            prev = got


@pytest.mark.gpu
def test_noalloc_oversize_leaves_output_untouched():
    """A call past the limit on the GPU is refused with the workspace status
    and does not write idx_out."""
    import torch
    B, Tq, HI, dI, k = 8, 1, 4, 32, 64
    nc = MAX_ELEMS // B + 1  # 262145 entries: within the indexer's range, past the scratch
    qI = torch.zeros(B, Tq, HI, dI, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(B, Tq, HI, dtype=torch.bfloat16, device="cuda")
    kI = torch.zeros(B, 1, dI, dtype=torch.bfloat16, device="cuda")  # refused before any read
    lens = torch.full((B,), 4, dtype=torch.int32, device="cuda")
    out = torch.full((B, Tq, k), -7, dtype=torch.int32, device="cuda")
    L = csa.lib()
    rc = L.csa_index_topk_noalloc(ctypes.c_void_p(qI.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                                  ctypes.c_void_p(kI.data_ptr()), ctypes.c_void_p(lens.data_ptr()),
                                  None, B, Tq, HI, dI, nc, k, csa.BF16,
                                  ctypes.c_void_p(out.data_ptr()), None)
    assert rc == CSA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert (out == -7).all()
