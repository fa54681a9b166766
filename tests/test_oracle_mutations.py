"""Mutation check of the oracle's pins: each plausible mistake below (a
swapped series, a transposed weight, a dropped ReLU or head weight, an
off-by-one in visibility or the window, a wrong tie rule, a wrong scale,
double rounding, a wrong rotation or norm) is planted in a copy of the oracle's C source, compiled,
and the pin tests are run against it.  Every mutant must fail at least one
pin; a mutant that survives means the pins do not determine that part of
the definition."""
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "csa_oracle.c")
PINS = ["tests/test_oracle_compress.py", "tests/test_oracle_index_topk.py",
        "tests/test_oracle_attend.py", "tests/test_oracle_e2e.py",
        "tests/test_oracle_mxfp4.py", "tests/test_oracle_rope.py", "tests/test_oracle_fp8.py"]

MUTANTS = {
    "csa_series_swapped": ("const void *W = (j < 4) ? Wa : Wb;", "const void *W = (j < 4) ? Wb : Wa;"),
    "csa_slot_order_reversed": ("z[j * d + c] = acc + ld(beta, dt, (size_t)j * d + c);\n      }\n    }\n    for (int c = 0; c < d; ++c) {\n      double mx = -INFINITY;\n      for (int j = 0; j < 8; ++j)",
                                "z[j * d + c] = acc + ld(beta, dt, (size_t)(7 - j) * d + c);\n      }\n    }\n    for (int c = 0; c < d; ++c) {\n      double mx = -INFINITY;\n      for (int j = 0; j < 8; ++j)"),
    "csa_no_overlap": ("const long s = 4 * (i - 1) + j;\n      valid[j] = (s >= 0 && s < nb);",
                       "const long s = 4 * (i - 1) + j;\n      valid[j] = (s >= 4 * i && s < nb);"),
    "weight_transposed": ("acc += ld(x, dt, xrow + e) * ld(W, dt, (size_t)e * d + c);\n        z[j * d + c] = acc + ld(beta, dt, (size_t)j * d + c);\n      }\n    }\n    for (int c = 0; c < d; ++c) {\n      double mx = -INFINITY;\n      for (int j = 0; j < 8; ++j)",
                          "acc += ld(x, dt, xrow + e) * ld(W, dt, (size_t)c * d + e);\n        z[j * d + c] = acc + ld(beta, dt, (size_t)j * d + c);\n      }\n    }\n    for (int c = 0; c < d; ++c) {\n      double mx = -INFINITY;\n      for (int j = 0; j < 8; ++j)"),
    "hca_bias_ignored": ("z[j * d + c] = acc + ld(beta, dt, (size_t)j * d + c);\n      }\n    }\n    for (int c = 0; c < d; ++c) {\n      double mx = -INFINITY;\n      for (long j = 0;",
                         "z[j * d + c] = acc;\n      }\n    }\n    for (int c = 0; c < d; ++c) {\n      double mx = -INFINITY;\n      for (long j = 0;"),
    "index_relu_dropped": ("acc += ld(w, dt, (size_t)r * HI + h) * (dot > 0.0 ? dot : 0.0);",
                           "acc += ld(w, dt, (size_t)r * HI + h) * dot;"),
    "index_head_weight_dropped": ("acc += ld(w, dt, (size_t)r * HI + h) * (dot > 0.0 ? dot : 0.0);",
                                  "acc += (dot > 0.0 ? dot : 0.0);"),
    "index_visibility_off_by_one": ("    vis[r] = (t + 1) / 4;\n", "    vis[r] = t / 4;\n"),
    "topk_ties_to_higher_index": ("return (a->i < b->i) ? -1 : (a->i > b->i);",
                                  "return (a->i > b->i) ? -1 : (a->i < b->i);"),
    "topk_output_unsorted": ("qsort(orow, (size_t)take, sizeof(int32_t), cmp_i32);", ""),
    "attend_scale": ("scale = 1.0 / sqrt((double)d);", "scale = 1.0 / (double)d;"),
    "attend_window_off_by_one": ("long w0 = t - window + 1;", "long w0 = t - window + 2;"),
    "attend_visibility": ("long vis = (t + 1) / m;", "long vis = (t + 2) / m;"),
    "attend_invisible_index_used": ("if (i < 0 || i >= vis) continue;", "if (i < 0 || i >= nc_max) continue;"),
    "attend_sink_ignored": ("if (sink) den += exp(sink[h] - mx);", ""),
    "mxfp4_ties_to_odd": ("return (lo % 2 == 0) ? lo : lo + 1;", "return (lo % 2 == 1) ? lo : lo + 1;"),
    "mxfp4_scale_off_by_one": ("X = ex - 1 - 2;", "X = ex - 1 - 1;"),
    "rms_sum_not_mean": ("sqrt(ss / d + eps)", "sqrt(ss + eps)"),
    "norm_gamma_ignored": ("y[c] * inv * (gamma ? ld(gamma, dt, (size_t)c) : 1.0)", "y[c] * inv"),
    "rope_turns_backwards": ("const double cs = cos(ang), sn = sin(ang);", "const double cs = cos(ang), sn = -sin(ang);"),
    "rope_half_split_pairs": ("const int i0 = d - r + 2 * j, i1 = i0 + 1;", "const int i0 = d - r + j, i1 = i0 + r / 2;"),
    "rope_frequency_exponent": ("pow(base, -2.0 * j / r)", "pow(base, -1.0 * j / r)"),
    "rope_inverse_ignored": ("(flags & 4) ? -(double)pos[rr] : (double)pos[rr]", "(double)pos[rr]"),
    "fp8_ties_to_odd": ("if (dd < bd || (dd == bd && (c % 2) == 0)) {", "if (dd < bd || (dd == bd && (c % 2) == 1)) {"),
    "fp8_scale_off_by_one": ("X = ex - 1 - 8;", "X = ex - 1 - 7;"),
    "fp8_rope_dims_misplaced": ("((uint16_t *)rope)[(size_t)row * r + e] = ((const uint16_t *)x)[(size_t)row * d + q + e];",
                                "((uint16_t *)rope)[(size_t)row * r + e] = ((const uint16_t *)x)[(size_t)row * d + e];"),
    "round_double_rounding": ("r = nearbyint(ldexp(a, -q));", "r = nearbyint(ldexp((double)(float)a, -q));"),
}


def _run_mutant(name, tmpdir):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation {name} no longer applies"
    mutated = src.replace(old, new, 1)
    cpath = os.path.join(tmpdir, f"{name}.c")
    lib = os.path.join(tmpdir, f"lib_{name}.so")
    with open(cpath, "w") as f:
        f.write(mutated)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", cpath, "-o", lib, "-lm"],
                   check=True, capture_output=True)
    env = dict(os.environ, CSA_ORACLE_LIB=lib, OMP_NUM_THREADS="1")
    p = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PINS],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, p.returncode


def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
            results = list(ex.map(lambda n: _run_mutant(n, tmp), MUTANTS))
    survivors = [n for n, rc in results if rc == 0]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
