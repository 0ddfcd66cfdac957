"""The single-launch layer (route, plan, up, down and finalize in one cooperative kernel) on decode shapes.

Bars: every output of moe_layer bit-identical to the separate launches (MOE_FUSED_LAYER=0), which the
other tests pin to the oracle -- out, residual, routing ids and weights, the plan in the workspace, h over
the real plan rows and y over every slot; routing ids and the plan bit-exact against the oracle directly;
out within 2e-2 x RMS of the oracle's fp64 layer; repeated calls on one workspace give the same bits (the
counters of the launch are cleared by every call).
"""
import os

import numpy as np
import pytest
import torch

import oracle
import prefill_sigmoid_top_b200 as moe
from prefill_sigmoid_top_b200 import inputs
from tests._util import bf16_bits, bits_to_f64, rms

pytestmark = pytest.mark.gpu

DEV = "cuda"

CASES = [
    # M, H, I, E, K, B
    (16, 256, 128, 8, 2, 16),
    (1, 256, 128, 8, 1, 16),       # one token, one slot
    (37, 512, 256, 64, 6, 32),     # ragged M
    (48, 256, 128, 4, 2, 16),      # expert 0 made hot (every token): 48 rows = two token tiles
    (64, 512, 256, 256, 16, 16),   # 1024 routed slots (the limit) over 256 experts
    (8, 7168, 2048, 64, 16, 16),   # the decode shape with 64 experts
    (9, 256, 128, 3, 3, 128),      # one 128-row block per expert
    (5, 8192, 256, 32, 8, 16),     # the widest hidden size the finalize slices take
    (200, 512, 256, 64, 4, 16),    # more than 64 tokens: the many-token finalize order
    (1000, 256, 128, 128, 1, 16),  # top-1, 1000 tokens
]
HOT = (48, 256, 128, 4, 2, 16)


def _inputs(case, seed):
    M, H, I, E, K, B = case
    cfg = inputs.WORKLOADS[0].with_(M=M, H=H, I=I, E=E, K=K, B=B, bias="normal", seed=seed)
    d = inputs.make_inputs(cfg, DEV)
    if case == HOT:
        d["bias"][0] += 8.0  # every token selects expert 0
    return cfg, d


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy()


def _run(d, shape, eps):
    M, H, I, E, K, B = shape.M, shape.H, shape.I, shape.E, shape.top_k, shape.block_size
    ws = torch.empty(moe.layer_workspace_size(shape), dtype=torch.uint8, device=DEV)
    ws.fill_(0xAB)
    out = torch.empty(M, H, dtype=torch.bfloat16, device=DEV)
    res = torch.empty(M, H, dtype=torch.bfloat16, device=DEV)
    ids = torch.full((M, K), -1, dtype=torch.int32, device=DEV)
    tw = torch.full((M, K), float("nan"), dtype=torch.float32, device=DEV)
    moe.layer(d["x"], d["w_router"], d["bias"], d["w_gate"], d["w_up"], d["w_down"], d["gamma"], eps, K, B, ws=ws,
              out=out, residual_out=res, topk_ids=ids, topk_w=tw)
    torch.cuda.synchronize()
    lay = moe.layer_workspace_layout(shape)
    err = ws[lay["err_flag"]:lay["err_flag"] + 4].view(torch.int32)
    assert moe.get_device_error(err) == 0

    def i32(name, n):
        return ws[lay[name]:lay[name] + 4 * n].view(torch.int32).cpu().numpy()

    ntpp = int(i32("num_tokens_post_padded", 1)[0])
    plan = dict(ntpp=ntpp, counts=i32("expert_counts", E), offsets=i32("expert_offsets", E + 1),
                sorted_ids=i32("sorted_ids", ntpp), block_expert=i32("block_expert", ntpp // B))
    cap = M * K + E * (B - 1)
    h = ws[lay["h"]:lay["h"] + 2 * cap * I].view(torch.bfloat16).view(cap, I)
    y = ws[lay["y"]:lay["y"] + 2 * M * K * H].view(torch.bfloat16).view(M * K, H)
    real = torch.from_numpy(plan["sorted_ids"] < M * K)
    rows = torch.nonzero(real).flatten().to(DEV)
    return dict(out=_bits(out), res=_bits(res), ids=ids.cpu().numpy(), w=tw.cpu().numpy(), plan=plan,
                h=_bits(h.index_select(0, rows)), y=_bits(y))


def _with_env(key, value, fn):
    old = os.environ.get(key)
    os.environ[key] = value
    try:
        return fn()
    finally:
        if old is None:
            del os.environ[key]
        else:
            os.environ[key] = old


@pytest.mark.parametrize("M,H,I,E,K,B", CASES)
def test_fused_layer_matches_separate_launches(M, H, I, E, K, B):
    cfg, d = _inputs((M, H, I, E, K, B), 7 * M + E)
    shape = moe.Shape(M, H, I, E, K, B)
    assert moe.layer_kernel_count(shape) == 1
    f = _run(d, shape, cfg.eps)
    if (M, H, I, E, K, B) == HOT:
        assert f["plan"]["counts"][0] == M
    s = _with_env("MOE_FUSED_LAYER", "0", lambda: _run(d, shape, cfg.eps))
    assert np.array_equal(f["ids"], s["ids"])
    assert np.array_equal(f["w"].view(np.int32), s["w"].view(np.int32))
    for k in ("ntpp", "counts", "offsets", "sorted_ids", "block_expert"):
        assert np.array_equal(f["plan"][k], s["plan"][k]), k
    assert np.array_equal(f["h"], s["h"])
    assert np.array_equal(f["y"], s["y"])
    assert np.array_equal(f["out"], s["out"])
    assert np.array_equal(f["res"], s["res"])


@pytest.mark.parametrize("case", [CASES[0], CASES[2], CASES[3], CASES[6]])
def test_fused_layer_against_oracle(case):
    M, H, I, E, K, B = case
    cfg, d = _inputs(case, 11 * M + E)
    shape = moe.Shape(M, H, I, E, K, B)
    g = _run(d, shape, cfg.eps)
    wg = [bf16_bits(d["w_gate"][e]) for e in range(E)]
    wu = [bf16_bits(d["w_up"][e]) for e in range(E)]
    wd = [bf16_bits(d["w_down"][e]) for e in range(E)]
    r = oracle.layer(bf16_bits(d["x"]), bf16_bits(d["w_router"]), d["bias"].cpu().numpy(), wg, wu, wd,
                     bf16_bits(d["gamma"]), cfg.eps, K)
    assert np.array_equal(g["ids"], r["ids"])
    assert np.abs(g["w"] - r["w"]).max() <= 1e-6
    o = oracle.align(r["ids"], E, B)
    assert g["plan"]["ntpp"] == o["ntpp"]
    assert np.array_equal(g["plan"]["counts"], o["counts"])
    assert np.array_equal(g["plan"]["offsets"], o["offsets"])
    assert np.array_equal(g["plan"]["sorted_ids"], o["sorted_ids"])
    assert np.array_equal(g["plan"]["block_expert"], o["block_expert"])
    ref = r["out_f64"]
    assert np.abs(bits_to_f64(g["out"].view(np.uint16)) - ref).max() <= 2e-2 * rms(ref)


def test_fused_layer_repeat_on_one_workspace():
    M, H, I, E, K, B = CASES[4]
    cfg, d = _inputs(CASES[4], 5)
    shape = moe.Shape(M, H, I, E, K, B)
    ws = torch.empty(moe.layer_workspace_size(shape), dtype=torch.uint8, device=DEV)
    outs = []
    for _ in range(4):
        out = moe.layer(d["x"], d["w_router"], d["bias"], d["w_gate"], d["w_up"], d["w_down"], d["gamma"], cfg.eps,
                        K, B, ws=ws)
        outs.append(out.clone())
    torch.cuda.synchronize()
    lay = moe.layer_workspace_layout(shape)
    assert moe.get_device_error(ws[lay["err_flag"]:lay["err_flag"] + 4].view(torch.int32)) == 0
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
