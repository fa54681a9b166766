"""The stored needle rows of the 1M CSA decode workload still match the input
generator, and each planted entry scores mu + 4 sigma under the oracle and is
selected by the oracle's top-k (the workload's planted-needle property)."""
import numpy as np
import pytest

import oracle
import workloads
from tests.golden.make_needles import input_digest


@pytest.fixture(scope="module")
def wl():
    return workloads.make(4)


def test_fixture_matches_generator(wl):
    fx = workloads.load_needles()
    assert fx["seed"] == wl.sizes["seed"] and fx["nc"] == wl.sizes["nc"]
    assert fx["input_sha256"] == input_digest(wl)
    assert list(fx["positions"]) == [int(p) for p in wl["needle_pos"]]


@pytest.mark.parametrize("b", [0, 3])
def test_needle_is_plus_4_sigma_and_selected(wl, b):
    fx = workloads.load_needles()
    p = fx["positions"][b]
    sc = oracle.index_scores(wl["qI"][b:b + 1], wl["w"][b:b + 1], wl["kI"][b:b + 1],
                             wl["lens"][b:b + 1])[0, 0]
    others = np.delete(sc, p)
    mu, sigma = others.mean(), others.std()
    assert abs(sc[p] - (mu + 4 * sigma)) <= 0.02 * abs(mu + 4 * sigma)
    k = wl.sizes["k"]
    idx = oracle.select_topk(sc[None], [sc.size], k)[0]
    assert p in set(idx.tolist())
