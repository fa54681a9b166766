"""Write needle_cfg4.json: one planted indexer-key row per sequence of the 1M
CSA decode workload (B=4, 262,144 entries, 64 x 128 indexer, bf16).

Calls only the CPU oracle.  Reading of "a planted needle entry gets a +4 sigma
indexer score at a random position per sequence": for sequence b, position
p_b is drawn by the input generator; mu and sigma are the mean and standard
deviation of the oracle's scores of all entries for that sequence's query;
the row becomes K[p] + alpha * g with g = sum_h w_h q_h over the heads whose
dot product with K[p] is positive (all heads if none), alpha found by
bisection so that the oracle score of the bf16-rounded row is mu + 4 sigma
within 1%.

    python tests/golden/make_needles.py
"""
import hashlib
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads  # noqa: E402


def input_digest(wl) -> str:
    h = hashlib.sha256()
    for k in ("qI", "w"):
        h.update(np.ascontiguousarray(wl[k]).tobytes())
    return h.hexdigest()


def score_of_row(qI, w, row):
    """Oracle score of a single cache row for one query (qI [1][1][HI][dI])."""
    kI = row.reshape(1, 1, -1)
    return float(oracle.index_scores(qI, w, kI, np.array([4], np.int32))[0, 0, 0])


def needle_row(qI, w, krow, target):
    qv = oracle.values(qI[0, 0])            # [HI][dI]
    wv = oracle.values(w[0, 0])             # [HI]
    kv = oracle.values(krow)                # [dI]
    act = (qv @ kv) > 0
    if not act.any():
        act[:] = True
    g = (wv[act, None] * qv[act]).sum(0)
    make = lambda a: workloads.bf16_bits((kv + a * g).astype(np.float32))
    lo, hi = 0.0, 1.0
    while score_of_row(qI, w, make(hi)) < target:
        hi *= 2.0
        if hi > 1e6:
            raise RuntimeError("needle target unreachable")
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        s = score_of_row(qI, w, make(mid))
        if abs(s - target) <= 0.01 * abs(target):
            return make(mid), s
        if s < target:
            lo = mid
        else:
            hi = mid
    raise RuntimeError("bisection did not reach 1%")


def main(path=workloads.NEEDLE_FIXTURE):
    wl = workloads.make(4, needle=False)
    B, nc = wl.sizes["B"], wl.sizes["nc"]
    pos = wl["needle_pos"]
    out = dict(seed=wl.sizes["seed"], nc=nc, input_sha256=input_digest(wl), positions=[],
               rows=[], mu=[], sigma=[], target=[], score=[],
               reading="K[p] + alpha*g, g = sum over active heads of w_h q_h; "
                       "score(bf16 row) = mu + 4 sigma within 1%")
    for b in range(B):
        sc = oracle.index_scores(wl["qI"][b:b + 1], wl["w"][b:b + 1], wl["kI"][b:b + 1],
                                 wl["lens"][b:b + 1])[0, 0]
        mu, sigma = float(sc.mean()), float(sc.std())
        target = mu + 4.0 * sigma
        p = int(pos[b])
        row, s = needle_row(wl["qI"][b:b + 1], wl["w"][b:b + 1], wl["kI"][b, p], target)
        out["positions"].append(p)
        out["rows"].append("".join(f"{int(v):04x}" for v in row))
        out["mu"].append(mu)
        out["sigma"].append(sigma)
        out["target"].append(target)
        out["score"].append(s)
        print(f"b={b} p={p} mu={mu:.5f} sigma={sigma:.5f} target={target:.5f} score={s:.5f}")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
