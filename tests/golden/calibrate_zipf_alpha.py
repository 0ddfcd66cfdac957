"""Calibrate the temperature of the Zipf-shaped router bias of the prefill workload.

The prefill workload (M=2048, H=7168, E=256, top_k=16, seed 3) draws its
router bias as b_e = -alpha * 1.1 * ln(rank_e), a Zipf(s=1.1)-shaped
popularity.  Zipf shares taken literally are unreachable (an expert can hold
at most one slot per token, i.e. 16x the mean), so alpha is chosen so that
the busiest expert receives about 10x the mean number of slots.  This script
routes the seed-3 inputs with the CPU oracle, bisects alpha, and writes
zipf_alpha.json beside itself.  It calls only the oracle and the input
generator.

Run:  python tests/golden/calibrate_zipf_alpha.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from prefill_sigmoid_top_b200 import inputs  # noqa: E402
from prefill_sigmoid_top_b200.inputs import bf16_bits  # noqa: E402

TARGET = 10.0


def ratio_for(tree, bias, K, E):
    z = (tree + bias[None, :].astype(np.float32)).astype(np.float32)  # fp32 add, as the router does
    ids, _ = oracle.topk(z, K)
    counts = np.bincount(ids.ravel(), minlength=E)
    return counts.max() / counts.mean(), counts


def main():
    cfg = inputs.WORKLOADS[3]
    w_router, _, _, x = inputs.router_inputs(cfg, alpha=1.0)
    tree = oracle.router_logits(bf16_bits(x), bf16_bits(w_router), None)  # bias-free canonical sums
    lo, hi = 0.0, 2.0
    best = None
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        bias = inputs.router_inputs(cfg, alpha=mid)[1].numpy()
        r, counts = ratio_for(tree, bias, cfg.K, cfg.E)
        best = (mid, r, counts)
        if abs(r - TARGET) < 0.05:
            break
        if r < TARGET:
            lo = mid
        else:
            hi = mid
    alpha = round(best[0], 4)
    bias = inputs.router_inputs(cfg, alpha=alpha)[1].numpy()
    r, counts = ratio_for(tree, bias, cfg.K, cfg.E)
    out = dict(alpha=alpha, max_over_mean=float(r), max_count=int(counts.max()), min_count=int(counts.min()),
               mean_count=float(counts.mean()), empty_experts=int((counts == 0).sum()),
               note="prefill workload seed 3, M=2048, E=256, top_k=16; routed with the CPU oracle")
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_alpha.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
