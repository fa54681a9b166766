"""Pins of the oracle's MXFP4 indexer-key format ("Anatomy of a Frontier
Model": the indexer key is 128 numbers in FP4 with one byte of scale per 32,
68 bytes): exact round trips of values on the grid, the rounding of every
midpoint to the even code, saturation, the all-zero block, the error bound
of the format, and bf16-exact dequantised values."""
import numpy as np
import pytest

import oracle
import workloads as W

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def codes_of(codes, dI):
    """uint8 pairs -> per-element 4-bit codes [..., dI]."""
    lo = codes & 15
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[:-1] + (dI,))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_grid_values_round_trip(seed):
    """Blocks whose values lie on the grid times 2^X, with the block maximum
    at magnitude 4 or 6, quantise to exactly those codes and that scale."""
    g = np.random.default_rng(seed)
    rows, dI = 16, 128
    X = g.integers(-20, 20, (rows, dI // 32))
    c = g.integers(0, 16, (rows, dI))
    c[:, ::32] = g.choice([6, 7, 14, 15], (rows, dI // 32))  # one element of |4| or |6| per block
    mag = GRID[c & 7] * np.exp2(np.repeat(X, 32, axis=1))
    vals = np.where(c & 8, -mag, mag).astype(np.float32)
    codes, scales = oracle.quantize_mxfp4(vals)
    np.testing.assert_array_equal(scales, (X + 127).astype(np.uint8))
    got = codes_of(codes, dI)
    # -0.0 keeps its sign bit: code 8 stays 8
    np.testing.assert_array_equal(got, c)
    np.testing.assert_array_equal(oracle.dequant_mxfp4(codes, scales), vals.astype(np.float64))


def test_midpoints_round_to_even_code():
    """y = 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5 (times the block scale) lie
    halfway between grid neighbours and take the even code; values just off
    the midpoints take the nearer neighbour; values above 6 saturate."""
    ys = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.2501, 0.7499, 5.01, 7.9, 6.0]
    want = [0, 2, 2, 4, 4, 6, 6, 1, 1, 7, 7, 7]
    block = np.zeros(32, np.float32)
    block[0] = 4.0  # fixes X = 0
    block[1:1 + len(ys)] = ys
    codes, scales = oracle.quantize_mxfp4(block[None])
    assert scales[0, 0] == 127
    got = codes_of(codes, 32)[0]
    assert got[0] == 6
    np.testing.assert_array_equal(got[1:1 + len(ys)], want)


def test_saturation_and_zero_block():
    blk = np.zeros((2, 32), np.float32)
    blk[0, 0] = 7.5 * 2.0 ** -3  # floor(log2) = -1 -> X = -3; 7.5 saturates to 6
    blk[0, 1] = -7.5 * 2.0 ** -3
    codes, scales = oracle.quantize_mxfp4(blk)
    assert scales[0, 0] == 124 and scales[1, 0] == 0
    got = codes_of(codes, 32)
    assert got[0, 0] == 7 and got[0, 1] == 15
    assert (got[1] == 0).all()
    np.testing.assert_array_equal(oracle.dequant_mxfp4(codes, scales)[1], 0.0)


def test_error_bound_and_bf16_exact():
    """N(0,1) keys in bf16 (the indexer-key workload): every element is
    within half a grid step of its dequantised value (a full step in the
    saturated range), and every dequantised value is a bf16 number."""
    k = W.normal(7, "kI", (64, 128), 1.0, "bf16")
    x = W.bf16_to_f32(k).astype(np.float64)
    codes, scales = oracle.quantize_mxfp4(k)
    dq = oracle.dequant_mxfp4(codes, scales)
    X = np.repeat(scales.astype(np.int64) - 127, 32, axis=1)
    y = np.abs(x) / np.exp2(X)
    step = np.where(y < 2, 0.5, np.where(y < 4, 1.0, 2.0))
    assert (np.abs(x - dq) <= step / 2 * np.exp2(X) + (y >= 6) * 2.0 * np.exp2(X)).all()
    as_bf16 = W.bf16_to_f32(W.bf16_bits(dq.astype(np.float32))).astype(np.float64)
    np.testing.assert_array_equal(as_bf16, dq)
