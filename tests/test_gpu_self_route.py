"""Self-routing up projection (align folded into the up kernel) against the oracle's plan and the
two-launch path.

Bars: every plan array bit-exact against oracle.align (the plan is a deterministic function of the
ids); h bit-identical, row by row over the real rows, to moe_grouped_up_swiglu run on the plan from
moe_align_block_size (the same tiles and the same MMA sequence); the layer output bit-identical with
the fold on and off.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import prefill_sigmoid_top_b200 as moe
from prefill_sigmoid_top_b200 import inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"

CASES = [
    # M, H, I, E, K, B
    (16, 256, 128, 8, 2, 16),
    (1, 256, 128, 8, 1, 16),
    (37, 512, 256, 64, 6, 32),
    (100, 256, 128, 4, 2, 16),     # 50 rows per expert: two 32-row token tiles each
    (64, 256, 128, 1024, 16, 16),  # 1024 slots, the limit
    (8, 7168, 2048, 64, 16, 16),   # the decode shape with 64 experts
    (9, 256, 128, 3, 3, 128),      # one 128-row block per expert
]


def _weights(cfg):
    d = inputs.make_inputs(cfg, DEV)
    return d


def _plan_np(p):
    return {k: v.cpu().numpy() for k, v in p.items()}


@pytest.mark.parametrize("M,H,I,E,K,B", CASES)
def test_routed_up_matches_align_plus_up(M, H, I, E, K, B):
    cfg = inputs.WORKLOADS[0].with_(M=M, H=H, I=I, E=E, K=K, B=B, bias="normal", seed=M * 3 + E)
    d = _weights(cfg)
    shape = moe.Shape(M, H, I, E, K, B)
    ids, _ = moe.route(d["x"], d["w_router"], d["bias"], K)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    h_r, plan_r = moe.grouped_up_swiglu_routed(d["x"], d["w_gate"], d["w_up"], ids, shape, err_flag=err)
    plan_a = moe.align_block_size(ids, E, B, err_flag=err)
    h_a = moe.grouped_up_swiglu(d["x"], d["w_gate"], d["w_up"], plan_a, shape, err_flag=err)
    torch.cuda.synchronize()
    assert moe.get_device_error(err) == 0
    o = oracle.align(ids.cpu().numpy(), E, B)
    g = _plan_np(plan_r)
    n = o["ntpp"]
    assert int(g["num_tokens_post_padded"][0]) == n
    assert np.array_equal(g["expert_counts"], o["counts"])
    assert np.array_equal(g["expert_offsets"], o["offsets"])
    assert np.array_equal(g["sorted_ids"][:n], o["sorted_ids"])
    assert np.array_equal(g["block_expert"][: n // B], o["block_expert"])
    real = torch.from_numpy(o["sorted_ids"] < M * K)
    rows = torch.nonzero(real).flatten().to(DEV)
    assert torch.equal(h_r.index_select(0, rows).view(torch.int16), h_a.index_select(0, rows).view(torch.int16))


def test_routed_up_flags_invalid_ids():
    M, H, I, E, K, B = 16, 256, 128, 8, 2, 16
    cfg = inputs.WORKLOADS[0].with_(M=M, H=H, I=I, E=E, K=K, B=B, seed=3)
    d = _weights(cfg)
    ids = torch.randint(0, E, (M, K), dtype=torch.int32, device=DEV)
    ids[3, 1] = E        # out of range: flagged on the device, never read as an expert
    ids[7, 0] = -5
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.grouped_up_swiglu_routed(d["x"], d["w_gate"], d["w_up"], ids, moe.Shape(M, H, I, E, K, B), err_flag=err)
    torch.cuda.synchronize()
    assert moe.get_device_error(err) == 4


@pytest.mark.parametrize("cid", [1])
def test_layer_same_output_with_and_without_fold(cid):
    cfg = inputs.WORKLOADS[cid]
    d = inputs.make_inputs(cfg, DEV)
    args = (d["x"], d["w_router"], d["bias"], d["w_gate"], d["w_up"], d["w_down"], d["gamma"], cfg.eps, cfg.K, cfg.B)
    out_fold = moe.layer(*args).clone()
    old = os.environ.get("MOE_SELF_ROUTE")
    os.environ["MOE_SELF_ROUTE"] = "0"
    try:
        out_two = moe.layer(*args).clone()
    finally:
        if old is None:
            del os.environ["MOE_SELF_ROUTE"]
        else:
            os.environ["MOE_SELF_ROUTE"] = old
    torch.cuda.synchronize()
    assert torch.equal(out_fold.view(torch.int16), out_two.view(torch.int16))
