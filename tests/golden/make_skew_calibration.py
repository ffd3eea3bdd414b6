"""Writes tests/golden/skew_calibration.json: the hot-set shift of the skewed
workload (T=16384, d=7168, 256 routed experts top-8; Student-t df=3
activations with a common direction m*v; centroids of a 10% hot set shifted
by beta*v).

beta is found by bisection so that, at step 0 (bias 0), the hot set takes
50% of all (token, expert) assignments, measured with the CPU oracle's router
on a seeded sample of tokens. Only the oracle and the input generator run.

usage: python tests/golden/make_skew_calibration.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import workloads  # noqa: E402
from oracle import moe  # noqa: E402

M_SHIFT = 4.0           # length of the common mean direction added to u
TARGET = 0.50
SAMPLE = 2048


def hot_share(cfg, u, beta):
    p = dict(m=M_SHIFT, beta=beta)
    e = workloads.centroids(cfg, skew=p).double().numpy()
    _, _, idx, _ = moe.route(u, e, np.zeros(cfg.N_r), cfg.K_r)
    hot = set(workloads.hot_experts(cfg).tolist())
    return float(np.isin(idx, list(hot)).mean())


def main():
    cfg = workloads.CONFIGS["skew"]
    u_all = workloads.activations(cfg, skew=dict(m=M_SHIFT, beta=0.0))
    rows = np.random.default_rng(0).choice(cfg.T, SAMPLE, replace=False)
    u = u_all[rows].double().numpy()
    lo, hi = 0.0, 4.0
    for _ in range(18):
        mid = 0.5 * (lo + hi)
        if hot_share(cfg, u, mid) < TARGET:
            lo = mid
        else:
            hi = mid
    beta = 0.5 * (lo + hi)
    share = hot_share(cfg, u, beta)
    out = dict(m=M_SHIFT, beta=beta, hot_share_at_step0=share,
               sample_tokens=SAMPLE, target=TARGET,
               made_by="tests/golden/make_skew_calibration.py (CPU oracle router)")
    with open(os.path.join(HERE, "skew_calibration.json"), "w") as f:
        json.dump(out, f, indent=1)
    print(out)


if __name__ == "__main__":
    main()
