"""Pins of the oracle's FP8 cache entries (E4M3 codes with one UE8M0 scale
per 64 elements, the RoPE dims kept as they are): published values of the
format, rounding against PyTorch's float8_e4m3fn conversion (a library
routine) wherever that conversion is defined, ties to the even code,
saturation at 448, the scale rule, the zero block, the sign of -0.0, the
error bound, and the RoPE dims.

Definition: "Anatomy of a Frontier Model: Reading DeepSeek-V4 Through Part
V", "The KV cache, recomputed" (448 FP8 numbers with 7 one-byte UE8M0
scales and 64 BF16 RoPE dims per entry).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W


def block_with(values, X=0, d=128, r=64):
    """One entry whose first block has largest magnitude in [2^(X+8), 2^(X+9))
    (so its scale exponent is X) and holds `values` (times 2^X) after it."""
    x = np.zeros((1, d), np.float32)
    x[0, 0] = 256.0 * 2.0 ** X
    x[0, 1:1 + len(values)] = np.asarray(values, np.float64) * 2.0 ** X
    return x


@pytest.mark.parametrize("value,code", [
    (1.0, 0x38), (448.0, 0x7E), (2.0 ** -6, 0x08), (2.0 ** -9, 0x01), (0.875 * 2.0 ** -6, 0x07),
    (240.0, 0x77), (256.0, 0x78), (1.5, 0x3C), (0.5, 0x30), (-1.0, 0xB8), (-0.0, 0x80)])
def test_published_codes(value, code):
    # values of the E4M3 format (1 sign, 4 exponent bits of bias 7, 3 mantissa bits)
    fp8, sc, _ = oracle.quantize_fp8_entries(block_with([value]))
    assert sc[0, 0] == 127  # X = 0
    assert fp8[0, 1] == code
    assert oracle.dequant_fp8_entries(fp8, sc, np.zeros((1, 64), np.float32))[0, 1] == value


def test_rounding_matches_torch_e4m3fn():
    # below the overflow midpoint 464 PyTorch's conversion rounds to nearest,
    # ties to even: every representable value, every midpoint and random values
    vals = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    mids = (vals[:-1] + vals[1:]) / 2
    rnd = np.random.default_rng(0).uniform(0, 463, 2000)
    tiny = np.random.default_rng(1).uniform(0, 2.0 ** -5, 500)
    for chunk in np.array_split(np.concatenate([vals, mids, rnd, tiny, -rnd[:500]]), 60):
        for X in (0, -20, 37):
            x = block_with(chunk, X)
            fp8, sc, _ = oracle.quantize_fp8_entries(x)
            ref = torch.from_numpy((chunk * 2.0 ** 0).astype(np.float32)).to(torch.float8_e4m3fn)
            assert np.array_equal(fp8[0, 1:1 + len(chunk)], ref.view(torch.uint8).numpy()), X


def test_ties_go_to_the_even_code():
    fp8, sc, _ = oracle.quantize_fp8_entries(block_with([1.0625, 1.1875, 17.0, 2.0 ** -10, 3 * 2.0 ** -10]))
    # 1.0625: 1.0 | 1.125 -> 1.0;  1.1875: 1.125 | 1.25 -> 1.25;  17: 16 | 18 -> 16;
    # 2^-10: 0 | 2^-9 -> 0;  3 * 2^-10: 2^-9 | 2^-8 -> 2^-8 (mantissa 2)
    assert list(fp8[0, 1:6]) == [0x38, 0x3A, 0x58, 0x00, 0x02]


def test_saturation_scale_rule_and_zero_block():
    x = np.zeros((3, 128), np.float32)
    x[0, 0], x[0, 1] = 500.0, -511.0         # amax in [256, 512): X = 0, both saturate
    x[1, :64] = 0.0                           # the zero block
    x[2, 5] = 3.0 * 2.0 ** 100                # amax in [2^101, 2^102): X = 93
    fp8, sc, _ = oracle.quantize_fp8_entries(x)
    assert sc[0, 0] == 127 and fp8[0, 0] == 0x7E and fp8[0, 1] == 0xFE
    assert sc[1, 0] == 0 and not fp8[1].any()
    assert sc[2, 0] == 127 + 93
    assert oracle.dequant_fp8_entries(fp8, sc, np.zeros((3, 64), np.float32))[2, 5] == 3.0 * 2.0 ** 100


def test_error_bound_and_rope_dims():
    x = W.normal(5, "kv", (64, 256), 1.0, "bf16")
    fp8, sc, rope = oracle.quantize_fp8_entries(x, rope_dim=64)
    assert fp8.shape == (64, 192) and sc.shape == (64, 3) and rope.shape == (64, 64)
    assert np.array_equal(rope, x[:, 192:])
    v = oracle.values(x)
    dq = oracle.dequant_fp8_entries(fp8, sc, rope)
    np.testing.assert_array_equal(dq[:, 192:], v[:, 192:])
    # below the block's saturation range a normal value is within half a
    # unit of its 3-bit mantissa (2^-4 relative); subnormals within 2^-10 * 2^X
    X = sc.astype(np.int64).repeat(64, axis=1) - 127
    q = v[:, :192]
    scaled = np.abs(q) / 2.0 ** X
    err = np.abs(dq[:, :192] - q) / 2.0 ** X
    normal = (scaled >= 2.0 ** -6) & (scaled <= 448)
    assert np.all(err[normal] <= scaled[normal] * 2.0 ** -4 + 1e-12)
    assert np.all(err[scaled < 2.0 ** -6] <= 2.0 ** -10)
    assert np.all(dq[:, :192][scaled > 448] == np.sign(q[scaled > 448]) * 448 * 2.0 ** X[scaled > 448])


def test_bad_layout_is_an_error():
    with pytest.raises(oracle.OracleError):
        oracle.quantize_fp8_entries(np.zeros((1, 100), np.float32), rope_dim=64)   # 36 FP8 dims
