"""Seeded synthetic inputs for the CSA / HCA hot path.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic.  The CUDA path and the CPU oracle both take their inputs
from here, so both see the same bits.

Conventions
  * Every tensor is drawn from its own stream,
    ``numpy.random.Generator(PCG64([seed, stream_id]))``, as float32 standard
    normals times a standard deviation; bf16 tensors are those float32 values
    rounded to bf16 (nearest, ties to even) and stored as uint16 bit patterns.
  * The seed of workload ``c`` is ``1234 + c``.
  * Shapes are row-major: tokens ``[B][n][d]``, caches ``[B][nc][d]``, queries
    ``[B][Tq][H][d]``, indexer queries ``[B][Tq][HI][dI]``, indexer head
    weights ``[B][Tq][HI]``; compressor weights ``[d][d]`` indexed [in][out],
    position biases ``[8][d]`` (CSA) or ``[m][d]`` (HCA); the window ring
    ``[B][n_tok][d]`` holds token s at row ``s % n_tok``.

The five workloads (sizes, dtypes and distributions as the problem statement
gives them; where it gives none, the reading is stated):
  1  CSA decode fp32: B=1, n=1024, H=8, d=64, HI=4, dI=32, k=64, window 128.
     Tokens, keys, queries and head weights N(0,1); compressor params (value
     and indexer series) N(0, 0.5^2) ("N(0,0.5)" read as std 0.5).  Both
     caches are built by the compressor from the tokens.
  2  CSA prefill bf16: B=1, n=Tq=8192 causal, H=16, d=128, HI=64, dI=128,
     k=512.  Q / tokens / indexer queries and keys N(0,1); compressor params
     and head weights std 1/sqrt(128) ("N(0,1/sqrt(128))" read as std).
  3  HCA decode bf16: B=32, n=131072, H=64, d=128, m=128: pre-built HCA cache
     [32][1024][128] N(0,1), window ring N(0,1), q N(0,1); the compressor is
     exercised separately on 131072 N(0,1) tokens per sequence with params of
     std 1/sqrt(d).
  4  CSA decode at 1M bf16: B=4, n=1,048,576, nc=262,144, H=64, d=128,
     HI=64, dI=128, k=1024: pre-built indexer-key and KV caches N(0,1),
     window ring N(0,1), q and indexer queries N(0,1), head weights std
     1/sqrt(128); one planted needle row per sequence (see ``needle_rows``).
  5  CSA+HCA layer pair bf16: B=64, n_b ~ U{65536..262144}; CSA caches of
     ceil(n_b/4) rows, HCA cache of ceil(n_b/128) rows, all N(0,1); separate
     queries for the two layers; HCA layer without an indexer.
"""
from __future__ import annotations

import json
import os
from dataclasses import dataclass, field

import numpy as np

F32 = "f32"
BF16 = "bf16"

# stream ids: one independent PCG64 stream per tensor role
_STREAMS = {
    "x": 1, "Wa": 2, "Wb": 3, "beta": 4,
    "kx": 5, "kWa": 6, "kWb": 7, "kbeta": 8,
    "q": 9, "qI": 10, "w": 11,
    "kI": 12, "kv": 13, "win": 14,
    "hca_kv": 15, "hca_W": 16, "hca_beta": 17, "hca_x": 18, "q2": 19,
    "lens": 20, "needle_pos": 21,
    "q_gamma": 22, "kv_gamma": 23,
}

HERE = os.path.dirname(os.path.abspath(__file__))
NEEDLE_FIXTURE = os.path.join(os.path.dirname(HERE), "tests", "golden", "needle_cfg4.json")


def seed_of(config_id: int) -> int:
    return 1234 + int(config_id)


def stream(seed: int, role: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([int(seed), _STREAMS[role]]))


def bf16_bits(a) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + r) >> 16).astype(np.uint16)


def bf16_to_f32(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float32 values."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal(seed: int, role: str, shape, std: float, dt: str) -> np.ndarray:
    """N(0, std^2) draws of the given shape in storage dtype dt."""
    g = stream(seed, role)
    a = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a if dt == F32 else bf16_bits(a)


def storage_dtype(dt: str):
    return np.float32 if dt == F32 else np.uint16


@dataclass
class Workload:
    """A named bundle of host arrays plus the scalar problem sizes."""
    name: str
    dt: str
    sizes: dict
    arrays: dict = field(default_factory=dict)

    def __getitem__(self, k):
        return self.arrays[k]

    def __contains__(self, k):
        return k in self.arrays


# --------------------------------------------------------------------------
# presets
# --------------------------------------------------------------------------
CONFIGS = {
    1: dict(name="csa_decode_fp32_n1024", kind="csa_decode_raw", dt=F32, B=1, n=1024, H=8, d=64,
            HI=4, dI=32, k=64, window=128, std_param=0.5, std_w=1.0),
    2: dict(name="csa_prefill_bf16_n8192", kind="csa_prefill", dt=BF16, B=1, n=8192, H=16, d=128,
            HI=64, dI=128, k=512, window=128, std_param=128 ** -0.5, std_w=128 ** -0.5),
    3: dict(name="hca_decode_bf16_b32_n131072", kind="hca_decode", dt=BF16, B=32, n=131072, H=64,
            d=128, m=128, window=128, std_param=128 ** -0.5),
    4: dict(name="csa_decode_bf16_b4_n1048576", kind="csa_decode_cache", dt=BF16, B=4, n=1048576,
            H=64, d=128, HI=64, dI=128, k=1024, window=128, std_w=128 ** -0.5, needle=True),
    5: dict(name="csa_hca_pair_bf16_b64_ragged", kind="pair_decode", dt=BF16, B=64, n_lo=65536,
            n_hi=262144, H=64, d=128, HI=64, dI=128, k=1024, window=128, m=128,
            std_w=128 ** -0.5),
}


def _ceil(a, b):
    return (a + b - 1) // b


def csa_raw(seed, B, n, H, d, HI, dI, dt, std_param, std_w, Tq=1, lens=None, name="csa_raw"):
    """Raw per-token inputs of a CSA layer (both caches are built by the
    compressor): tokens x, per-token indexer keys kx, both series' params,
    queries q / qI and head weights w."""
    lens = np.full(B, n, np.int32) if lens is None else np.asarray(lens, np.int32)
    a = dict(
        x=normal(seed, "x", (B, n, d), 1.0, dt),
        Wa=normal(seed, "Wa", (d, d), std_param, dt),
        Wb=normal(seed, "Wb", (d, d), std_param, dt),
        beta=normal(seed, "beta", (8, d), std_param, dt),
        kx=normal(seed, "kx", (B, n, dI), 1.0, dt),
        kWa=normal(seed, "kWa", (dI, dI), std_param, dt),
        kWb=normal(seed, "kWb", (dI, dI), std_param, dt),
        kbeta=normal(seed, "kbeta", (8, dI), std_param, dt),
        q=normal(seed, "q", (B, Tq, H, d), 1.0, dt),
        qI=normal(seed, "qI", (B, Tq, HI, dI), 1.0, dt),
        w=normal(seed, "w", (B, Tq, HI), std_w, dt),
        lens=lens,
    )
    return Workload(name, dt, dict(B=B, n=n, Tq=Tq, H=H, d=d, HI=HI, dI=dI, nc=_ceil(n, 4)), a)


def csa_cache(seed, B, n, H, d, HI, dI, dt, std_w, lens=None, n_tok=128, name="csa_cache",
              nc_max=None):
    """Decode inputs of a CSA layer whose caches are already built: indexer
    keys kI and KV entries kv (N(0,1), ceil(n_max/4) rows), the window ring,
    one query per sequence."""
    lens = np.full(B, n, np.int32) if lens is None else np.asarray(lens, np.int32)
    nc = _ceil(int(lens.max()), 4) if nc_max is None else nc_max
    a = dict(
        kI=normal(seed, "kI", (B, nc, dI), 1.0, dt),
        kv=normal(seed, "kv", (B, nc, d), 1.0, dt),
        win=normal(seed, "win", (B, n_tok, d), 1.0, dt),
        q=normal(seed, "q", (B, 1, H, d), 1.0, dt),
        qI=normal(seed, "qI", (B, 1, HI, dI), 1.0, dt),
        w=normal(seed, "w", (B, 1, HI), std_w, dt),
        lens=lens,
    )
    return Workload(name, dt, dict(B=B, n=n, Tq=1, H=H, d=d, HI=HI, dI=dI, nc=nc, n_tok=n_tok), a)


def hca_cache(seed, B, n, H, d, dt, m=128, lens=None, n_tok=128, name="hca_cache", q_role="q"):
    """Decode inputs of an HCA layer with a pre-built cache of ceil(n_max/m)
    N(0,1) rows, the window ring and one query per sequence."""
    lens = np.full(B, n, np.int32) if lens is None else np.asarray(lens, np.int32)
    nc = _ceil(int(lens.max()), m)
    a = dict(
        hkv=normal(seed, "hca_kv", (B, nc, d), 1.0, dt),
        win=normal(seed, "win", (B, n_tok, d), 1.0, dt),
        q=normal(seed, q_role, (B, 1, H, d), 1.0, dt),
        lens=lens,
    )
    return Workload(name, dt, dict(B=B, n=n, Tq=1, H=H, d=d, m=m, nc=nc, n_tok=n_tok), a)


def hca_tokens(seed, B, n, d, dt, m=128, std_param=128 ** -0.5, lens=None, name="hca_tokens"):
    """Raw tokens and HCA compressor params (W [d][d], beta [m][d])."""
    lens = np.full(B, n, np.int32) if lens is None else np.asarray(lens, np.int32)
    a = dict(
        x=normal(seed, "hca_x", (B, n, d), 1.0, dt),
        W=normal(seed, "hca_W", (d, d), std_param, dt),
        beta=normal(seed, "hca_beta", (m, d), std_param, dt),
        lens=lens,
    )
    return Workload(name, dt, dict(B=B, n=n, d=d, m=m, nc=_ceil(n, m)), a)


def ragged_lens(seed, B, lo, hi) -> np.ndarray:
    """Context lengths drawn uniformly from the integers [lo, hi]."""
    return stream(seed, "lens").integers(lo, hi, size=B, endpoint=True).astype(np.int32)


def needle_positions(seed, B, nc) -> np.ndarray:
    return stream(seed, "needle_pos").integers(0, nc, size=B).astype(np.int64)


def load_needles(path=NEEDLE_FIXTURE):
    with open(path) as f:
        return json.load(f)


def plant_needles(wl: Workload, fixture: dict) -> None:
    """Overwrite the planted rows of the indexer-key cache with the stored
    needle rows (bf16 bits).  The rows were written by a committed script that
    calls only the CPU oracle; this function just copies them in."""
    if fixture["seed"] != wl.sizes["seed"] or fixture["nc"] != wl.sizes["nc"]:
        raise ValueError("needle fixture does not match this workload")
    for b, (p, hexrow) in enumerate(zip(fixture["positions"], fixture["rows"])):
        row = np.array([int(hexrow[4 * j:4 * j + 4], 16) for j in range(len(hexrow) // 4)],
                       np.uint16)
        wl.arrays["kI"][b, p, :] = row


def make(config_id: int, needle: bool = True) -> Workload:
    """Full-size inputs of one of the five workloads."""
    c = CONFIGS[config_id]
    seed = seed_of(config_id)
    kind = c["kind"]
    if kind == "csa_decode_raw":
        wl = csa_raw(seed, c["B"], c["n"], c["H"], c["d"], c["HI"], c["dI"], c["dt"],
                     c["std_param"], c["std_w"], name=c["name"])
    elif kind == "csa_prefill":
        wl = csa_raw(seed, c["B"], c["n"], c["H"], c["d"], c["HI"], c["dI"], c["dt"],
                     c["std_param"], c["std_w"], Tq=c["n"], name=c["name"])
    elif kind == "hca_decode":
        wl = hca_cache(seed, c["B"], c["n"], c["H"], c["d"], c["dt"], m=c["m"], name=c["name"])
    elif kind == "csa_decode_cache":
        wl = csa_cache(seed, c["B"], c["n"], c["H"], c["d"], c["HI"], c["dI"], c["dt"],
                       c["std_w"], name=c["name"])
        wl.sizes["seed"] = seed
        wl.arrays["needle_pos"] = needle_positions(seed, c["B"], wl.sizes["nc"])
        if needle and c.get("needle"):
            plant_needles(wl, load_needles())
    elif kind == "pair_decode":
        lens = ragged_lens(seed, c["B"], c["n_lo"], c["n_hi"])
        wl = csa_cache(seed, c["B"], int(lens.max()), c["H"], c["d"], c["HI"], c["dI"], c["dt"],
                       c["std_w"], lens=lens, name=c["name"])
        h = hca_cache(seed, c["B"], int(lens.max()), c["H"], c["d"], c["dt"], m=c["m"], lens=lens,
                      q_role="q2")
        wl.arrays["hkv"] = h["hkv"]
        wl.arrays["q2"] = h["q"]
        wl.sizes["hnc"] = h.sizes["nc"]
        wl.sizes["m"] = c["m"]
    else:
        raise KeyError(kind)
    wl.sizes.setdefault("seed", seed)
    wl.sizes.update({k: v for k, v in c.items() if k in ("k", "window", "m")})
    return wl
