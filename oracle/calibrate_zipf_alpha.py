"""Calibrate the Zipf logit-bias scale of the skewed-routing workload.

TEST INFRASTRUCTURE.  The workload asks for a per-expert router-logit bias
drawn from Zipf(s=1.2) over the experts such that one hot expert receives
about 30% of the T*k assignments.  Taking bias_e = ln p_(e+1) literally sends
far more than 30% to expert 0, so the bias is scaled: bias_e = alpha * ln
p_(e+1), and alpha is found here by bisection so that expert 0's share of the
oracle's top-k assignments on the workload's seeded tokens and router
weights is 0.30.  The printed value is stored as ``ZIPF_ALPHA`` in
``mixture_experts_layer_45_b200/workloads.py``; a CPU test re-checks it.

Run:  python oracle/calibrate_zipf_alpha.py
"""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from oracle import moe_ref  # noqa: E402
from mixture_experts_layer_45_b200 import workloads  # noqa: E402


def hot_share(logits0, E, k, alpha):
    bias = workloads.zipf_logit_bias(E, alpha).astype(np.float64)
    idx = moe_ref.topk(logits0 + bias[None, :], k)
    return float((idx == 0).sum()) / idx.size


def main():
    w = workloads.workload("skewed-top2")
    r = workloads.draw_router_inputs(w)
    logits0 = moe_ref.router_logits(r["x"], r["w_router"])
    lo, hi = 0.0, 1.0
    for _ in range(24):
        mid = 0.5 * (lo + hi)
        if hot_share(logits0, w.E, w.k, mid) < 0.30:
            lo = mid
        else:
            hi = mid
    alpha = hi
    print(f"ZIPF_ALPHA = {alpha!r}  share = {hot_share(logits0, w.E, w.k, alpha):.5f}")


if __name__ == "__main__":
    main()
