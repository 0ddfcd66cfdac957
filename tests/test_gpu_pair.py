"""2-SM pair GEMMs (cta_group::2, M = 256 over a cluster of two CTAs) against the oracle.

Same bars as the single-SM grouped projections: h and y elementwise within 2^-7 |ref| + 1e-2 RMS(ref)
against the oracle's bf16-rounded values, padding rows of h never written, canaries intact, no device
error.  The cases cover token tiles narrower than a box (8 rows per CTA), several 256-row tiles per
expert with a ragged tail, empty experts, both token-tile widths, and x rows either pre-gathered into
plan order or gathered by the up kernel itself (tile::gather4).
"""
import numpy as np
import pytest
import torch

import oracle
import prefill_sigmoid_top_b200 as moe
from prefill_sigmoid_top_b200 import inputs
from tests._util import bf16_bits, bits_to_f64
from tests.test_gpu_parity import DEV, canary_ok, close_elementwise, expert_lists, guarded, host_bits, to_dev

pytestmark = pytest.mark.gpu

PAIR_CASES = [
    dict(M=300, H=512, I=256, E=8, K=3, B=64),     # ~112 rows per expert
    dict(M=600, H=512, I=512, E=4, K=2, B=16),     # 300 rows per expert: 256-row tiles plus a ragged tail
    dict(M=40, H=1024, I=256, E=16, K=4, B=16),    # ~10 rows per expert: 8 rows per CTA
    dict(M=5, H=512, I=256, E=64, K=6, B=32),      # most experts empty
    dict(M=600, H=1024, I=512, E=4, K=2, B=16),    # two weight blocks per expert in both projections
    dict(M=64, H=1024, I=1024, E=8, K=4, B=16),    # ~32 rows per expert over four up weight blocks
]


@pytest.mark.parametrize("gather", ["0", "1"])
@pytest.mark.parametrize("pair", ["128", "256"])
@pytest.mark.parametrize("case", PAIR_CASES)
def test_pair_up_down(case, pair, gather, monkeypatch):
    monkeypatch.setenv("MOE_PAIR_GATHER", gather)  # x rows pre-gathered into plan order, or gathered in the GEMM
    monkeypatch.setenv("MOE_GEMM_PERSISTENT", "1")
    monkeypatch.setenv("MOE_UP_GATHER", "pregather")
    monkeypatch.setenv("MOE_GEMM_NMAX", "128")
    monkeypatch.setenv("MOE_GEMM_PAIR", pair)
    cfg = inputs.WORKLOADS[0].with_(bias="normal", seed=case["M"] + 7 * case["E"], **case)
    d = to_dev(cfg)
    hb = host_bits(d)
    ids_o, _ = oracle.route(hb["x"], hb["w_router"], hb["bias"], cfg.K)
    plan_o = oracle.align(ids_o, cfg.E, cfg.B)
    shape = moe.Shape(cfg.M, cfg.H, cfg.I, cfg.E, cfg.K, cfg.B)
    cap = moe.align_capacity(shape)
    sorted_full = np.full(cap, -1, np.int32)
    sorted_full[: plan_o["ntpp"]] = plan_o["sorted_ids"]
    bexp = np.zeros(cap // cfg.B + 1, np.int32)
    bexp[: len(plan_o["block_expert"])] = plan_o["block_expert"]
    plan = dict(sorted_ids=torch.from_numpy(sorted_full).to(DEV), block_expert=torch.from_numpy(bexp).to(DEV),
                expert_counts=torch.from_numpy(plan_o["counts"]).to(DEV),
                expert_offsets=torch.from_numpy(plan_o["offsets"]).to(DEV),
                num_tokens_post_padded=torch.tensor([plan_o["ntpp"]], dtype=torch.int32, device=DEV))
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    raw_h, h = guarded(cap * cfg.I, torch.bfloat16)
    h = h.view(cap, cfg.I)
    moe.grouped_up_swiglu(d["x"], d["w_gate"], d["w_up"], plan, shape, h=h, err_flag=err)
    raw_y, y = guarded(cfg.M * cfg.K * cfg.H, torch.bfloat16)
    y = y.view(cfg.M * cfg.K, cfg.H)
    moe.grouped_down(h, d["w_down"], plan, shape, y=y, err_flag=err)
    torch.cuda.synchronize()
    assert moe.get_device_error(err) == 0
    assert canary_ok(raw_h, cap * cfg.I, torch.bfloat16) and canary_ok(raw_y, cfg.M * cfg.K * cfg.H, torch.bfloat16)
    wg, wu, wd = expert_lists(d, range(cfg.E), cfg.E)
    r = oracle.layer(hb["x"], hb["w_router"], hb["bias"], wg, wu, wd, hb["gamma"], cfg.eps, cfg.K, want_h=True)
    h_np = bits_to_f64(bf16_bits(h))
    real = plan_o["sorted_ids"] < cfg.M * cfg.K
    rows = np.nonzero(real)[0]
    slots = plan_o["sorted_ids"][real]
    h_ref = bits_to_f64(r["h"].reshape(cfg.M * cfg.K, cfg.I))[slots]
    ok, e, nbad = close_elementwise(h_np[rows], h_ref)
    assert ok, ("h", e, nbad)
    pad_rows = np.nonzero(~real)[0]
    if len(pad_rows):
        assert np.isnan(h_np[pad_rows]).all()
    y_ref = bits_to_f64(r["y"].reshape(cfg.M * cfg.K, cfg.H))
    ok, e, nbad = close_elementwise(bits_to_f64(bf16_bits(y)), y_ref)
    assert ok, ("y", e, nbad)
