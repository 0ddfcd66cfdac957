"""Pins for the oracle's tensor-parallel layer (the expert intermediate dimension split over G ranks, the
finalize fused with the reduction across ranks and the RMSNorm; flashinfer PR #5701 analysis, intro).

* One rank is the unsharded layer, bit for bit (the residual enters on rank 0, so s is the finalize's).
* A hand case on two ranks whose partial rows are exact: every value written out and rounded by the
  brute-force bf16 search.
* On random inputs the ranks' partial rows add up to the unsharded rows within their bf16 roundings
  (linearity of the down projection over I), and so does s.
"""
import math

import numpy as np
import pytest

import oracle
from prefill_sigmoid_top_b200 import inputs
from tests._util import bf16_bits, bf16_nearest_even, bits_to_f64, rms


def _np_inputs(cfg):
    t = inputs.make_inputs(cfg, "cpu")
    E = cfg.E
    return dict(x=bf16_bits(t["x"]), wr=bf16_bits(t["w_router"]), b=t["bias"].numpy(), g=bf16_bits(t["gamma"]),
                wg=[bf16_bits(t["w_gate"][e]) for e in range(E)], wu=[bf16_bits(t["w_up"][e]) for e in range(E)],
                wd=[bf16_bits(t["w_down"][e]) for e in range(E)])


def _bits_of(vals):
    return np.array([bf16_nearest_even(float(v)) for v in np.ravel(vals)], np.uint16).reshape(np.shape(vals))


def test_one_rank_is_the_unsharded_layer():
    cfg = inputs.WORKLOADS[0].with_(M=6, H=256, I=256, E=8, K=3, bias="normal", seed=31)
    d = _np_inputs(cfg)
    r1 = oracle.layer(d["x"], d["wr"], d["b"], d["wg"], d["wu"], d["wd"], d["g"], cfg.eps, cfg.K)
    rt = oracle.layer_tp(d["x"], d["wr"], d["b"], d["wg"], d["wu"], d["wd"], d["g"], cfg.eps, cfg.K, 1,
                         want_y_parts=True)
    assert np.array_equal(rt["ids"], r1["ids"]) and np.array_equal(rt["w"], r1["w"])
    assert np.array_equal(rt["y_parts"][0], r1["y"])
    for k in ("out", "residual", "out_f64", "residual_f64"):
        assert np.array_equal(rt[k], r1[k]), k


def test_two_rank_hand_case():
    # the hand case of the unsharded layer (2 tokens, 4 experts, I = 2) on two ranks: rank 0 holds column 0
    # of h (y_0 = [h_0, 0, ...]), rank 1 column 1 (y_1 = [0, -h_1, ...]); both partial rows are exact.
    H, I, E, K, M = 256, 2, 4, 2, 2
    x = np.zeros((M, H))
    x[0, :2] = [1.0, 2.0]
    x[1, :2] = [-1.0, 0.5]
    wr = np.zeros((E, H))
    wr[:, 0] = [0.0, 1.0, -1.0, 0.5]
    bias = np.array([0.25, 0.0, 0.0, 0.0], np.float32)
    wg, wu, wd = np.zeros((E, I, H)), np.zeros((E, I, H)), np.zeros((E, H, I))
    for e in range(E):
        wg[e, 0, 0] = wg[e, 1, 1] = 1.0
        wu[e, 0, 0] = wu[e, 1, 1] = e + 1.0
        wd[e, 0, 0], wd[e, 1, 1] = 1.0, -1.0
    gamma = np.ones(H)
    r = oracle.layer_tp(_bits_of(x), _bits_of(wr), bias, [_bits_of(a) for a in wg], [_bits_of(a) for a in wu],
                        [_bits_of(a) for a in wd], _bits_of(gamma), 1e-5, K, 2, want_y_parts=True)
    assert r["ids"].tolist() == [[1, 3], [2, 0]]
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))
    w = [np.array([sig(1.0), sig(0.5)]) / (sig(1.0) + sig(0.5)), np.array([sig(1.0), sig(0.25)]) / (sig(1.0) + sig(0.25))]
    for t, ids in enumerate([(1, 3), (2, 0)]):
        p0 = x[t].copy()
        p1 = np.zeros(H)
        for k, e in enumerate(ids):
            h = [bits_to_f64(np.array([bf16_nearest_even(x[t, i] * sig(x[t, i]) * (e + 1) * x[t, i])], np.uint16))[0]
                 for i in range(I)]
            y0, y1 = np.zeros(H), np.zeros(H)
            y0[0] = h[0]
            y1[1] = -h[1]
            assert np.array_equal(bits_to_f64(r["y_parts"][0, t, k]), y0)
            assert np.array_equal(bits_to_f64(r["y_parts"][1, t, k]), y1)
            p0 += w[t][k] * y0
            p1 += w[t][k] * y1
        s = p0 + p1
        inv = 1.0 / math.sqrt(float(np.sum(s * s)) / H + 1e-5)
        assert r["out"][t].tolist() == [bf16_nearest_even(v * inv) for v in s]
        assert r["residual"][t].tolist() == [bf16_nearest_even(v) for v in s]


@pytest.mark.parametrize("G", [2, 4])
def test_partials_add_up_to_the_unsharded_layer(G):
    cfg = inputs.WORKLOADS[0].with_(M=6, H=256, I=256, E=8, K=4, bias="normal", seed=40 + G)
    d = _np_inputs(cfg)
    r1 = oracle.layer(d["x"], d["wr"], d["b"], d["wg"], d["wu"], d["wd"], d["g"], cfg.eps, cfg.K)
    rt = oracle.layer_tp(d["x"], d["wr"], d["b"], d["wg"], d["wu"], d["wd"], d["g"], cfg.eps, cfg.K, G,
                         want_y_parts=True)
    assert np.array_equal(rt["ids"], r1["ids"])
    # linearity over I: sum_r y_r = y up to the G + 1 bf16 roundings (at most half a step each, i.e.
    # 2^-8 of the rounded value's magnitude: bf16 keeps 8 significant bits)
    yp = bits_to_f64(rt["y_parts"])
    y = bits_to_f64(r1["y"])
    bound = 2.0 ** -8 * (np.abs(yp).sum(axis=0) + np.abs(y)) * (1 + 1e-9) + 1e-300
    assert (np.abs(yp.sum(axis=0) - y) <= bound).all()
    # s = x + sum_k w_k sum_r y_r, so |s_tp - s| is at most the weighted sum of those bounds
    sb = np.einsum("tk,tkh->th", r1["w"], bound) + 1e-12 * np.abs(r1["residual_f64"])
    assert (np.abs(rt["residual_f64"] - r1["residual_f64"]) <= sb).all()
    assert np.abs(rt["out_f64"] - r1["out_f64"]).max() <= 2e-2 * rms(r1["out_f64"])
    # the per-rank parts, added in rank order, are the layer's s exactly
    s = None
    for rank in range(G):
        p = oracle.tp_partial(d["x"], d["wr"], d["b"], d["wg"], d["wu"], d["wd"], cfg.K, G, rank)["p"]
        s = p if s is None else s + p
    assert np.array_equal(s, rt["residual_f64"])


def test_split_must_divide_the_intermediate_dimension():
    cfg = inputs.WORKLOADS[0].with_(M=2, H=256, I=128, E=4, K=2, seed=3)
    d = _np_inputs(cfg)
    with pytest.raises(RuntimeError):
        oracle.tp_partial(d["x"], d["wr"], d["b"], d["wg"], d["wu"], d["wd"], cfg.K, 3, 0)
