"""Calibrate the logit-bias scale beta of the Zipf-skewed workload and store it.

The skewed workload adds b_e = beta * ln(p_e) to every token's router logits, with
p_e proportional to (e+1)^-s.  This script picks beta by bisection so that the share of
top-k assignments that expert 0 receives under the oracle's routing is within 0.5% of
p_0, and writes workloads/zipf_beta.json.  It calls only the oracle and the seeded input
generator; run it from the repository root:

    python -m oracle.calibrate_zipf
"""
from __future__ import annotations

import json
import os

import numpy as np

from oracle import moe_oracle as orc
import workloads


def expert0_share(l_clean, bias_dir, beta, k):
    idx = orc.top_k(l_clean + beta * bias_dir[None, :], k)
    return float(np.sum(idx == 0)) / idx.size


def main():
    w = workloads.WORKLOADS["zipf"]
    inp = workloads.make_inputs(w, beta=0.0)
    l = orc.router_logits(inp["x"], inp["w_gate"])
    p = workloads.zipf_probs(w.E, w.zipf_s).numpy()
    lnp = np.log(p)
    target = float(p[0])
    lo, hi = 0.0, 8.0
    for _ in range(60):
        mid = 0.5 * (lo + hi)
        if expert0_share(l, lnp, mid, w.k) < target:
            lo = mid
        else:
            hi = mid
    beta = 0.5 * (lo + hi)
    share = expert0_share(l, lnp, beta, w.k)
    idx = orc.top_k(l + beta * lnp[None, :], w.k)
    hist = np.bincount(idx.reshape(-1), minlength=w.E)
    assert abs(share - target) <= 0.005 * target, (share, target)
    out = {
        "beta": beta,
        "target_share_expert0": target,
        "realised_share_expert0": share,
        "realised_histogram": hist.tolist(),
        "workload": w.describe(),
        "written_by": "python -m oracle.calibrate_zipf",
    }
    path = os.path.join(os.path.dirname(workloads.__file__), "zipf_beta.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps({k: out[k] for k in ("beta", "target_share_expert0",
                                           "realised_share_expert0", "realised_histogram")}))


if __name__ == "__main__":
    main()
