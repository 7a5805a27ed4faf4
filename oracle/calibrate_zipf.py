"""Calibrate the Zipf(1.1) routing skew of the DeepSeek-V3-shaped T=8192 prefill workload.

Test infrastructure: computes, with the oracle's own router and top-k, the
offset strength beta for which the busiest expert receives ~10x the mean load
(max_e count_e / (T*k/E) in [9.5, 10.5]) on the seed-0 tokens, by bisection.
The result is written into fp8_fp4_moe_b200/inputs.py as ZIPF_BETA_T8192 by
hand (the value is a fixture constant; this script is how it was obtained).

    python -m oracle.calibrate_zipf
"""
from __future__ import annotations

import numpy as np
import torch

from fp8_fp4_moe_b200 import inputs as I

from . import moe as M


def max_load_ratio(w, scores, beta):
    bias = I.zipf_offsets(w.E, beta).numpy()
    ids = M.select_experts(scores, bias, w.k)
    counts = np.bincount(ids.ravel(), minlength=w.E)
    return counts.max() / (w.T * w.k / w.E)


def calibrate(seed=0, lo=0.0, hi=1.0, target=(9.5, 10.5), iters=40):
    w = I.WORKLOADS["dsv3_t8192_zipf"]
    x, W_r, _ = I.make_routing_inputs(w, seed, zipf_beta=0.0)
    scores = M.router_scores(x.view(torch.int16).numpy().view(np.uint16), W_r.numpy())
    for _ in range(iters):
        mid = (lo + hi) / 2
        r = max_load_ratio(w, scores, mid)
        if target[0] <= r <= target[1]:
            return mid, r
        if r < target[0]:
            lo = mid
        else:
            hi = mid
    raise RuntimeError("bisection did not reach the target band")


if __name__ == "__main__":
    beta, ratio = calibrate()
    print(f"ZIPF_BETA_T8192 = {beta!r}   # busiest/mean = {ratio:.3f}")
