"""The seeded input generator: determinism, shapes, distributions, Zipf calibration."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from prefill_sigmoid_top_b200 import inputs
from tests._util import bf16_bits

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_deterministic_and_shapes():
    cfg = inputs.WORKLOADS[0]
    a = inputs.make_inputs(cfg)
    b = inputs.make_inputs(cfg)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    assert a["x"].shape == (cfg.M, cfg.H) and a["x"].dtype == torch.bfloat16
    assert a["w_router"].shape == (cfg.E, cfg.H)
    assert a["w_gate"].shape == (cfg.E, cfg.I, cfg.H) and a["w_down"].shape == (cfg.E, cfg.H, cfg.I)
    assert a["bias"].dtype == torch.float32 and (a["bias"] == 0).all()


def test_distributions():
    cfg = inputs.WORKLOADS[0].with_(M=256, H=1024, I=512, E=4, bias="normal", seed=5)
    a = inputs.make_inputs(cfg)
    assert abs(a["x"].float().std().item() - 1.0) < 0.02
    assert abs(a["w_router"].float().std().item() * np.sqrt(cfg.H) - 1.0) < 0.03
    assert abs(a["w_gate"].float().std().item() * np.sqrt(cfg.H) - 1.0) < 0.02
    assert abs(a["w_down"].float().std().item() * np.sqrt(cfg.I) - 1.0) < 0.02
    assert abs((a["gamma"].float() - 1).std().item() - 0.1) < 0.01


def test_router_side_independent_of_expert_draws():
    cfg = inputs.WORKLOADS[1]
    w_r, b, g, x = inputs.router_inputs(cfg)
    assert x.shape == (8, 7168) and b.shape == (256,)
    assert 0.2 < b.std().item() < 0.45   # N(0, 0.1): std ~ 0.316


def test_zipf_alpha_matches_calibration():
    with open(os.path.join(GOLDEN, "zipf_alpha.json")) as f:
        cal = json.load(f)
    assert inputs.ZIPF_ALPHA == cal["alpha"]
    assert abs(cal["max_over_mean"] - 10.0) <= 0.5 and cal["empty_experts"] == 0


@pytest.mark.slow
def test_zipf_ratio_reproduced_by_oracle():
    cfg = inputs.WORKLOADS[3]
    w_r, b, g, x = inputs.router_inputs(cfg)
    ids, _ = oracle.route(bf16_bits(x), bf16_bits(w_r), b.numpy(), cfg.K)
    counts = np.bincount(ids.ravel(), minlength=cfg.E)
    assert abs(counts.max() / counts.mean() - 10.0) <= 0.5
