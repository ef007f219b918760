"""Calibrate beta of the skewed long-prefill workload's router bias with the CPU oracle.

The workload (T=16384 tokens, 288 experts, top-8, seed 4) asks for a router bias drawn
"Zipf(s=1.1) so that the top 10% of experts receive about 50% of the assignments".  A plain
Zipf(1.1) law over 288 ranks gives its top 29 ranks about 70% of the mass, so the bias is
b_e = beta * ln(r_e^-1.1 / sum_r r^-1.1) with beta chosen here by bisection: the oracle's
routing of this workload's own x and W_router must give the 29 most-loaded experts a share
of 0.50 of all T*k assignments.

Only the oracle is called.  The result goes into tests/golden/skew_bias_beta.json; the
constant SKEW_BETA in sparse_mixture_experts_ffn_b200/inputs.py is copied from it.

    python tests/golden/calibrate_skew_bias.py
"""
import json
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from sparse_mixture_experts_ffn_b200 import inputs  # noqa: E402

TARGET = 0.50


def top_share(scores, bias, k, E, top):
    idx, _, _ = oracle.route(scores, k, bias)
    counts = np.bincount(idx.ravel(), minlength=E)
    return float(np.sort(counts)[::-1][:top].sum() / counts.sum())


def main():
    cfg = inputs.CONFIGS["prefill_t16384_skew"]
    x, Wr, _ = inputs.make_routing_inputs(cfg, beta=1.0)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    wb = Wr.view(torch.int16).numpy().view(np.uint16)
    scores = oracle.router_scores(xb, wb)
    top = int(round(0.1 * cfg.E))
    lo, hi = 0.0, 2.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        b = inputs.skew_bias(cfg, beta=mid)
        share = top_share(scores, b.numpy(), cfg.top_k, cfg.E, top)
        if share < TARGET:
            lo = mid
        else:
            hi = mid
    beta = round(0.5 * (lo + hi), 6)
    b = inputs.skew_bias(cfg, beta=beta)
    share = top_share(scores, b.numpy(), cfg.top_k, cfg.E, top)
    out = dict(workload=cfg.name, T=cfg.T, E=cfg.E, top_k=cfg.top_k, seed=cfg.seed,
               zipf_s=inputs.ZIPF_S, top_experts=top, target_share=TARGET, beta=beta,
               measured_share=round(share, 6))
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "skew_bias_beta.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    print(json.dumps(out))


if __name__ == "__main__":
    main()
