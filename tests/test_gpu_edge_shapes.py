"""Whole layer at the edges of the accepted shapes, against the oracle.

* E = 1024 experts, top_k = 32, H = 8192, block 256, I = 128 (the largest expert count, top-k,
  hidden size and block the boundary accepts; decode path with the align step in the up kernel);
* H = 8192 with ~150 routed rows per expert (the 2-SM pair kernels, 256-row token tiles);
* E = 1, K = 1 (every token on the one expert).
Bars as the other layer tests: ids bit-exact, weights within 1e-6, out within 2e-2 RMS of the
oracle's fp64 value before its final rounding.  Only the touched experts' weights are copied to the
host.
"""
import numpy as np
import pytest
import torch

import oracle
import prefill_sigmoid_top_b200 as moe
from prefill_sigmoid_top_b200 import inputs
from tests._util import bf16_bits, bits_to_f64, rms
from tests.test_gpu_parity import DEV, expert_lists, host_bits, run_layer, to_dev

pytestmark = pytest.mark.gpu

EDGE = [
    inputs.WORKLOADS[0].with_(name="e1024_k32", M=8, H=8192, I=128, E=1024, K=32, B=256, seed=21, bias="normal"),
    inputs.WORKLOADS[0].with_(name="h8192_pairs", M=300, H=8192, I=512, E=16, K=8, B=16, seed=22, bias="normal"),
    inputs.WORKLOADS[0].with_(name="one_expert", M=33, H=512, I=256, E=1, K=1, B=16, seed=23, bias="normal"),
]


@pytest.mark.parametrize("cfg", EDGE, ids=lambda c: c.name)
def test_layer_edge_shapes(cfg):
    d = to_dev(cfg)
    g = run_layer(d, cfg)
    hb = host_bits(d)
    ids_o, w_o = oracle.route(hb["x"], hb["w_router"], hb["bias"], cfg.K)
    assert np.array_equal(g["ids"], ids_o)
    assert np.abs(g["w"] - w_o).max() <= 1e-6
    wg, wu, wd = expert_lists(d, ids_o.ravel(), cfg.E)
    r = oracle.layer(hb["x"], hb["w_router"], hb["bias"], wg, wu, wd, hb["gamma"], cfg.eps, cfg.K)
    ref = r["out_f64"]
    assert np.abs(bits_to_f64(g["out"]) - ref).max() <= 2e-2 * rms(ref)
    rref = r["residual_f64"]
    assert np.abs(bits_to_f64(g["res"]) - rref).max() <= 2e-2 * rms(rref)
