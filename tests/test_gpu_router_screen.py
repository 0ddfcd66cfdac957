"""The screened router (moe_route from 128 tokens: integer tensor-core logits bound the canonical ones, and
only the experts that can be selected get their canonical fp32 logit) against the plain router
(MOE_ROUTER_SCREEN=0: every canonical logit) and the oracle.

Ids and weights must be the plain router's bit for bit, and the ids the oracle's.  The cases cover token
and expert counts that are not multiples of the 128 x 128 integer tile, one expert, more experts than a
warp's 256, all-equal logits (every expert a candidate), rows that are not finite, and magnitudes far from
1 (scales of the integer digits near the ends of the fp32 range)."""
import numpy as np
import pytest
import torch

import oracle
import prefill_sigmoid_top_b200 as moe
from prefill_sigmoid_top_b200 import inputs
from tests._util import bf16_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"

SHAPES = [
    # M, H, E, K, bias
    (128, 256, 8, 2, "normal"),
    (300, 512, 33, 5, "normal"),     # M and E not multiples of the 128-row tiles
    (256, 1024, 64, 8, "normal"),
    (200, 256, 256, 16, "normal"),
    (130, 768, 1000, 32, "normal"),  # E > 256: 32 experts per lane in the candidate kernel
    (512, 2048, 128, 4, "zipf"),
    (129, 256, 1, 1, "normal"),      # one expert
]


def _both(x, w_r, b, K, monkeypatch):
    ids, w = moe.route(x, w_r, b, K)
    monkeypatch.setenv("MOE_ROUTER_SCREEN", "0")
    ids_p, w_p = moe.route(x, w_r, b, K)
    monkeypatch.delenv("MOE_ROUTER_SCREEN")
    torch.cuda.synchronize()
    return ids, w, ids_p, w_p


def _same_bits(a, b):
    return torch.equal(a.view(torch.int32), b.view(torch.int32))  # NaN weights (a NaN token) compare too


def _check(x, w_r, b, K, monkeypatch, oracle_ids=True):
    ids, w, ids_p, w_p = _both(x.to(DEV), w_r.to(DEV), None if b is None else b.to(DEV), K, monkeypatch)
    assert torch.equal(ids, ids_p)
    assert _same_bits(w, w_p)
    if oracle_ids:
        bn = np.zeros(w_r.shape[0], np.float32) if b is None else b.numpy()
        ids_o, _ = oracle.route(bf16_bits(x), bf16_bits(w_r), bn, K)
        assert np.array_equal(ids.cpu().numpy(), ids_o)


@pytest.mark.parametrize("M,H,E,K,bias", SHAPES)
def test_screened_equals_plain_and_oracle(M, H, E, K, bias, monkeypatch):
    cfg = inputs.WORKLOADS[0].with_(M=M, H=H, E=E, K=K, bias=bias, seed=M + 3 * E)
    w_r, b, _, x = inputs.router_inputs(cfg)
    _check(x, w_r, b, K, monkeypatch)


def test_all_equal_logits_make_every_expert_a_candidate(monkeypatch):
    M, H, E, K = 200, 256, 64, 8
    x = torch.randn(M, H).to(torch.bfloat16)
    w_r = torch.zeros(E, H, dtype=torch.bfloat16)
    b = torch.full((E,), 0.25, dtype=torch.float32)
    ids, w, ids_p, w_p = _both(x.to(DEV), w_r.to(DEV), b.to(DEV), K, monkeypatch)
    assert torch.equal(ids, ids_p) and _same_bits(w, w_p)
    assert (ids.cpu() == torch.arange(K, dtype=torch.int32).expand(M, K)).all()


def test_rows_that_are_not_finite(monkeypatch):
    M, H, E, K = 160, 512, 64, 8
    cfg = inputs.WORKLOADS[0].with_(M=M, H=H, E=E, K=K, bias="normal", seed=77)
    w_r, b, _, x = inputs.router_inputs(cfg)
    w_r[[5, 40]] = float("nan")
    w_r[17, 3] = float("inf")
    x[4] = float("nan")
    x[150, 100] = float("-inf")
    _check(x, w_r, b, K, monkeypatch)


@pytest.mark.parametrize("scale", [2.0 ** -60, 2.0 ** 40, 2.0 ** 125])  # 2^125: canonical fp32 sums overflow
def test_magnitudes_far_from_one(scale, monkeypatch):
    M, H, E, K = 144, 512, 48, 6
    cfg = inputs.WORKLOADS[0].with_(M=M, H=H, E=E, K=K, bias="normal", seed=5)
    w_r, b, _, x = inputs.router_inputs(cfg)
    x = (x.float() * scale).to(torch.bfloat16)
    x[7, 11] = 1.0  # one token whose largest element dwarfs the rest: coarse digits, wide bounds
    _check(x, w_r, b, K, monkeypatch)


@pytest.mark.parametrize("cid", [2, 3, 4])
def test_full_size_screened_equals_plain(cid, monkeypatch):
    cfg = inputs.WORKLOADS[cid]
    w_r, b, _, x = inputs.router_inputs(cfg)
    ids, w, ids_p, w_p = _both(x.to(DEV), w_r.to(DEV), b.to(DEV), cfg.K, monkeypatch)
    assert torch.equal(ids, ids_p)
    assert _same_bits(w, w_p)
