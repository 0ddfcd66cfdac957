"""Pins for the oracle's expert MLP, finalize and whole layer.

* E=1, K=1 reduces the layer to one SwiGLU MLP plus RMSNorm: checked against
  torch's own fp64 ops (matmul, silu, rms_norm) on the CPU.
* Sparse routed sum == dense mixture over all experts with unselected weights 0.
* K == E is the dense mixture with every expert selected.
* A hand case small enough to check by eye (2 tokens, 4 experts).
* NVFP4 layer with inputs on the NVFP4 grid reduces to the bf16 layer.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from prefill_sigmoid_top_b200 import inputs
from tests._util import bf16_bits, bf16_nearest_even, bits_to_f64, rms


def _np_inputs(cfg):
    t = inputs.make_inputs(cfg, "cpu")
    E = cfg.E
    return dict(
        x=bf16_bits(t["x"]), w_router=bf16_bits(t["w_router"]), bias=t["bias"].numpy(),
        gamma=bf16_bits(t["gamma"]),
        w_gate=[bf16_bits(t["w_gate"][e]) for e in range(E)],
        w_up=[bf16_bits(t["w_up"][e]) for e in range(E)],
        w_down=[bf16_bits(t["w_down"][e]) for e in range(E)],
    )


def _ulp_diff(a_bits, b_bits):
    """|difference| in units of bf16 spacing (same-sign finite values)."""
    a = a_bits.astype(np.int32)
    b = b_bits.astype(np.int32)
    sa = np.where(a & 0x8000, -(a & 0x7FFF), a & 0x7FFF)
    sb = np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    return np.abs(sa - sb)


def test_single_expert_equals_torch_swiglu_rmsnorm():
    cfg = inputs.WORKLOADS[0].with_(E=1, K=1, M=8, H=256, I=128, seed=21)
    d = _np_inputs(cfg)
    r = oracle.layer(d["x"], d["w_router"], d["bias"], d["w_gate"], d["w_up"], d["w_down"], d["gamma"],
                     cfg.eps, cfg.K, want_h=True)
    assert (r["ids"] == 0).all() and np.allclose(r["w"], 1.0, atol=0)
    x = torch.tensor(bits_to_f64(d["x"]))
    wg, wu, wd = (torch.tensor(bits_to_f64(a[0])) for a in (d["w_gate"], d["w_up"], d["w_down"]))
    gamma = torch.tensor(bits_to_f64(d["gamma"]))
    # h: torch fp64 SwiGLU, rounded to bf16 through fp32 (a double rounding that can
    # differ from a one-step rounding by one bf16 step, rarely)
    h_t = (F.silu(x @ wg.T) * (x @ wu.T)).float().to(torch.bfloat16)
    dh = _ulp_diff(r["h"][:, 0, :], bf16_bits(h_t))
    assert dh.max() <= 1 and (dh > 0).mean() < 1e-2
    # y from the oracle's own h (so one h step cannot cascade)
    h_o = torch.tensor(bits_to_f64(r["h"][:, 0, :]))
    y_t = (h_o @ wd.T).float().to(torch.bfloat16)
    dy = _ulp_diff(r["y"][:, 0, :], bf16_bits(y_t))
    assert dy.max() <= 1 and (dy > 0).mean() < 1e-2
    # out = rms_norm(x + y) * gamma, from the oracle's own y
    s = x + torch.tensor(bits_to_f64(r["y"][:, 0, :]))
    out_t = F.rms_norm(s, (cfg.H,), gamma, eps=cfg.eps).float().to(torch.bfloat16)
    do = _ulp_diff(r["out"], bf16_bits(out_t))
    assert do.max() <= 1 and (do > 0).mean() < 1e-2
    dr = _ulp_diff(r["residual"], bf16_bits(s.float().to(torch.bfloat16)))
    assert dr.max() <= 1


def test_sparse_equals_dense_mixture():
    cfg = inputs.WORKLOADS[0]
    d = _np_inputs(cfg)
    r = oracle.layer(d["x"], d["w_router"], d["bias"], d["w_gate"], d["w_up"], d["w_down"], d["gamma"],
                     cfg.eps, cfg.K)
    wdense = np.zeros((cfg.M, cfg.E))
    for t in range(cfg.M):
        wdense[t, r["ids"][t]] = r["w"][t]
    mix = oracle.dense_mixture(d["x"], d["w_gate"], d["w_up"], d["w_down"], wdense)
    sparse = np.einsum("tk,tkh->th", r["w"], bits_to_f64(r["y"]))
    assert np.allclose(sparse, mix, rtol=0, atol=1e-12 * max(1.0, np.abs(mix).max()))


def test_k_equals_e_is_dense_mixture():
    cfg = inputs.WORKLOADS[0].with_(E=4, K=4, M=6, seed=22, bias="normal")
    d = _np_inputs(cfg)
    r = oracle.layer(d["x"], d["w_router"], d["bias"], d["w_gate"], d["w_up"], d["w_down"], d["gamma"],
                     cfg.eps, cfg.K)
    for t in range(cfg.M):
        assert sorted(r["ids"][t].tolist()) == [0, 1, 2, 3]
    z = oracle.router_logits(d["x"], d["w_router"], d["bias"]).astype(np.float64)
    s = 1 / (1 + np.exp(-z))
    wdense = s / s.sum(axis=1, keepdims=True)
    mix = oracle.dense_mixture(d["x"], d["w_gate"], d["w_up"], d["w_down"], wdense)
    sparse = np.einsum("tk,tkh->th", r["w"], bits_to_f64(r["y"]))
    assert np.allclose(sparse, mix, rtol=0, atol=1e-12 * max(1.0, np.abs(mix).max()))


def _bits_of(vals):
    return np.array([bf16_nearest_even(float(v)) for v in np.ravel(vals)], np.uint16).reshape(np.shape(vals))


def test_hand_case():
    # H=256 with only columns 0,1 in use; I=2; E=4; K=2; M=2.
    H, I, E, K, M = 256, 2, 4, 2, 2
    x = np.zeros((M, H))
    x[0, :2] = [1.0, 2.0]
    x[1, :2] = [-1.0, 0.5]
    wr = np.zeros((E, H))
    wr[:, 0] = [0.0, 1.0, -1.0, 0.5]
    bias = np.array([0.25, 0.0, 0.0, 0.0], np.float32)
    # logits: token0 (0.25, 1, -1, 0.5) -> ids (1, 3); token1 (0.25, -1, 1, -0.5) -> ids (2, 0)
    wg = np.zeros((E, I, H))
    wu = np.zeros((E, I, H))
    wd = np.zeros((E, H, I))
    for e in range(E):
        wg[e, 0, 0] = wg[e, 1, 1] = 1.0          # g_i = x_i
        wu[e, 0, 0] = wu[e, 1, 1] = e + 1.0      # u_i = (e+1) x_i
        wd[e, 0, 0], wd[e, 1, 1] = 1.0, -1.0     # y_0 = h_0, y_1 = -h_1
    gamma = np.ones(H)
    r = oracle.layer(_bits_of(x), _bits_of(wr), bias, [_bits_of(a) for a in wg], [_bits_of(a) for a in wu],
                     [_bits_of(a) for a in wd], _bits_of(gamma), 1e-5, K, want_h=True)
    assert r["ids"].tolist() == [[1, 3], [2, 0]]
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))
    w0 = np.array([sig(1.0), sig(0.5)]) / (sig(1.0) + sig(0.5))
    w1 = np.array([sig(1.0), sig(0.25)]) / (sig(1.0) + sig(0.25))
    assert np.allclose(r["w"], [w0, w1], rtol=0, atol=1e-15)
    for t, (ids, ws) in enumerate([((1, 3), w0), ((2, 0), w1)]):
        s = x[t, :].copy()
        for k, e in enumerate(ids):
            h = [bf16_nearest_even((x[t, i] * sig(x[t, i])) * ((e + 1) * x[t, i])) for i in range(I)]
            assert r["h"][t, k].tolist() == h
            hv = bits_to_f64(np.array(h, np.uint16))
            y = np.zeros(H)
            y[0], y[1] = bits_to_f64(np.array([bf16_nearest_even(hv[0]), bf16_nearest_even(-hv[1])], np.uint16))
            assert np.array_equal(bits_to_f64(r["y"][t, k]), y)
            s += ws[k] * y
        inv = 1.0 / math.sqrt(float(np.sum(s * s)) / H + 1e-5)
        out = [bf16_nearest_even(v * inv) for v in s]
        assert r["out"][t].tolist() == out
        assert r["residual"][t].tolist() == [bf16_nearest_even(v) for v in s]


def test_finalize_matches_torch_rms_norm():
    rng = np.random.default_rng(8)
    M, K, H = 5, 3, 512
    x = bf16_bits(torch.randn(M, H).to(torch.bfloat16))
    y = bf16_bits(torch.randn(M, K, H).to(torch.bfloat16))
    w = rng.dirichlet(np.ones(K), size=M)
    gamma = bf16_bits((1 + 0.1 * torch.randn(H)).to(torch.bfloat16))
    out, res = oracle.finalize(x, y, w, gamma, 1e-5)
    s = torch.tensor(bits_to_f64(x)) + torch.einsum("tk,tkh->th", torch.tensor(w), torch.tensor(bits_to_f64(y)))
    ref = F.rms_norm(s, (H,), torch.tensor(bits_to_f64(gamma)), eps=1e-5)
    d = _ulp_diff(out, bf16_bits(ref.float().to(torch.bfloat16)))
    assert d.max() <= 1 and (d > 0).mean() < 1e-2


def test_nvfp4_layer_on_grid_reduces_to_bf16_layer():
    # Operands drawn from the e2m1 grid with a 6 in every 16-block: NVFP4
    # quantisation then reproduces them up to the fp32 rounding of the global
    # scale, so h equals the bf16 layer's h (to within one bf16 step).
    rng = np.random.default_rng(9)
    M, H, I, E, K = 4, 256, 64, 4, 2
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])

    def on_grid(rows, cols):
        v = rng.choice(grid, size=(rows, cols)) * rng.choice([-1, 1], size=(rows, cols))
        v[:, ::16] = 6.0
        return v

    x = on_grid(M, H)
    wr = rng.standard_normal((E, H)) * 0.0625
    bias = np.zeros(E, np.float32)
    wg = [on_grid(I, H) for _ in range(E)]
    wu = [on_grid(I, H) for _ in range(E)]
    wd = [on_grid(H, I) * 0.125 for _ in range(E)]
    gamma = np.ones(H)
    xb, wrb, gb = _bits_of(x), _bits_of(wr), _bits_of(gamma)
    wgb, wub, wdb = [_bits_of(a) for a in wg], [_bits_of(a) for a in wu], [_bits_of(a) for a in wd]
    ref = oracle.layer(xb, wrb, bias, wgb, wub, wdb, gb, 1e-5, K, want_h=True)
    q = lambda mats: [oracle.nvfp4_quantize_bf16(m) for m in mats]
    gq, uq, dq = q(wgb), q(wub), q(wdb)
    for (codes, scales, gs), wb in zip(gq, wgb):
        # near-identity: the dequantised weights are the inputs up to fp32 scale rounding
        assert np.allclose(oracle.nvfp4_dequantize(codes, scales, gs), bits_to_f64(wb), rtol=2.0 ** -21, atol=0)
    r = oracle.layer_nvfp4(xb, wrb, bias, gq, uq, dq, gb, 1e-5, K)
    assert np.array_equal(r["ids_all"], ref["ids"])
    h_ref = ref["h"].reshape(M * K, I)
    dh = _ulp_diff(r["h_all"], h_ref)
    assert dh.max() <= 1 and (dh > 0).mean() < 0.02
    # down projection: quantise the oracle's own h with the call-wide global
    # scale, dequantise, and multiply with numpy (library matmul) in fp64
    hf = bits_to_f64(r["h_all"]).astype(np.float32)
    hgs = oracle.nvfp4_global_scale(float(np.abs(hf).max()))
    hc, hs = oracle.nvfp4_quantize(hf, hgs)
    hdeq = oracle.nvfp4_dequantize(hc, hs, hgs)
    for slot in range(M * K):
        e = r["ids_all"].ravel()[slot]
        wdq = oracle.nvfp4_dequantize(*dq[e])
        y_np = hdeq[slot] @ wdq.T
        y_bits = np.array([bf16_nearest_even(v) for v in y_np], np.uint16)
        assert _ulp_diff(r["y"].reshape(M * K, H)[slot], y_bits).max() <= 1
