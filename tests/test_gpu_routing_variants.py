"""GPU parity for the routing variants (softmax / sigmoid scores, renormalisation, routed scale,
selection-only bias) against the oracle.

Bars: ids bit-exact (the selection key is the same canonical fp32 logit on both sides); weights
within 2e-6 x routed_scale.  Derivation: the kernel's weights are fp32; a sigmoid score carries
a few ulp (~2^-22 relative), and a softmax denominator is a sum of up to E terms in at most
E/32 + 5 fp32 additions, ~1e-6 relative at E = 1024; every weight is at most routed_scale.
"""
import numpy as np
import pytest
import torch

import oracle
import prefill_sigmoid_top_b200 as moe
from prefill_sigmoid_top_b200 import inputs
from tests._util import bf16_bits

pytestmark = pytest.mark.gpu

DEV = "cuda"

VARIANTS = [
    # scoring, renormalize, routed_scale, bias_in_score
    (moe.SCORE_SIGMOID, True, 1.0, True),
    (moe.SCORE_SIGMOID, False, 1.0, True),
    (moe.SCORE_SIGMOID, True, 2.5, False),
    (moe.SCORE_SOFTMAX, True, 1.0, True),
    (moe.SCORE_SOFTMAX, False, 1.0, True),
    (moe.SCORE_SOFTMAX, False, 2.5, False),
]


def _run(cfg, variant, bias_override=None):
    scoring, renorm, scale, in_score = variant
    w_r, b, g, x = inputs.router_inputs(cfg)
    if bias_override is not None:
        b = bias_override
    ids, w = moe.route_ex(x.to(DEV), w_r.to(DEV), b.to(DEV), cfg.K, scoring, renorm, scale, in_score)
    ids_o, w_o = oracle.route_ex(bf16_bits(x), bf16_bits(w_r), b.numpy(), cfg.K, scoring, renorm, scale, in_score)
    assert np.array_equal(ids.cpu().numpy(), ids_o)
    assert np.abs(w.cpu().numpy() - w_o).max() <= 2e-6 * scale


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("M,E,K", [(37, 64, 6), (19, 256, 16), (9, 1024, 8)])
def test_variants_small(variant, M, E, K):
    cfg = inputs.WORKLOADS[0].with_(M=M, H=512, E=E, K=K, bias="normal", seed=M + E)
    _run(cfg, variant)


@pytest.mark.parametrize("variant", VARIANTS)
def test_selection_only_bias_changes_picks(variant):
    # a strong ramp bias: picks follow the key, weights follow the unbiased logit
    cfg = inputs.WORKLOADS[0].with_(M=33, H=256, E=64, K=8, seed=5)
    ramp = torch.from_numpy((np.arange(cfg.E, dtype=np.float32) - cfg.E / 2) * 0.2)
    _run(cfg, variant, bias_override=ramp)


@pytest.mark.parametrize("cid", [1, 3])
def test_variants_full_size(cid):
    cfg = inputs.WORKLOADS[cid]
    _run(cfg, (moe.SCORE_SOFTMAX, True, 2.5, True))
    _run(cfg, (moe.SCORE_SIGMOID, False, 1.0, False))


def test_default_options_equal_route_bitwise():
    cfg = inputs.WORKLOADS[2]
    w_r, b, g, x = inputs.router_inputs(cfg)
    xd, wd, bd = x.to(DEV), w_r.to(DEV), b.to(DEV)
    ids0, w0 = moe.route(xd, wd, bd, cfg.K)
    ids1, w1 = moe.route_ex(xd, wd, bd, cfg.K)
    assert torch.equal(ids0, ids1)
    assert torch.equal(w0.view(torch.int32), w1.view(torch.int32))
