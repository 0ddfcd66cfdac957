"""Pins for the oracle's router: canonical fp32 logit order, top-k selection, weights."""
import itertools

import numpy as np
import pytest
import scipy.special

import oracle
from prefill_sigmoid_top_b200 import inputs
from tests._util import bf16_bits, bits_to_f64, f32_to_bf16_bits


def _bits(vals):
    return f32_to_bf16_bits(np.asarray(vals, np.float32))


def _single_logit(xv, wv, bias=0.0):
    x = _bits(xv)[None, :]
    w = _bits(wv)[None, :]
    return float(oracle.router_logits(x, w, np.array([bias], np.float32))[0, 0])


# ------------------------------------------------------------------ canonical order
def test_tree_order_hand_case():
    # H=256: lane l owns h = 8l..8l+7.  Partials: p0 = 2^24, p16 = 1, p8 = 1, p24 = 1.
    # Tree: p0+p16 = 2^24+1 -> 2^24 (tie, even); p8+p24 = 2; then 2^24 + 2 exactly.
    # (A left-to-right sum would give 2^24; the exact sum is 2^24 + 3.)
    H = 256
    x = np.zeros(H)
    w = np.zeros(H)
    x[0], w[0] = 4096.0, 4096.0       # lane 0 -> 2^24
    x[8 * 16], w[8 * 16] = 1.0, 1.0   # lane 16
    x[8 * 8], w[8 * 8] = 1.0, 1.0     # lane 8
    x[8 * 24], w[8 * 24] = 1.0, 1.0   # lane 24
    assert _single_logit(x, w) == 2.0 ** 24 + 2.0


def test_lane_accumulates_sequentially_across_chunks():
    # Lane 0 owns h = 0..7 and 256..263 (H=512).  Products 2^24, 1 (h=1), 1 (h=256),
    # 1 (h=257): sequential fma in increasing h gives 2^24 at every step; summing each
    # chunk first would give 2^24 + 2.
    H = 512
    x = np.zeros(H)
    w = np.zeros(H)
    x[0], w[0] = 4096.0, 4096.0
    for h in (1, 256, 257):
        x[h], w[h] = 1.0, 1.0
    assert _single_logit(x, w) == 2.0 ** 24


def test_fma_within_lane_and_bias_last():
    # Lane 0: products 1, 2^-24 (h=1), then bias 2^-24.  Sequential: 1 + 2^-24 -> 1
    # (tie, even).  Bias added after the tree: 1 + 2^-24 -> 1.  Exact would be 1 + 2^-23.
    H = 256
    x = np.zeros(H)
    w = np.zeros(H)
    x[0], w[0] = 1.0, 1.0
    x[1], w[1] = 2.0 ** -12, 2.0 ** -12
    assert _single_logit(x, w, bias=2.0 ** -24) == 1.0
    # a bias large enough to register is added exactly once, at the end
    assert _single_logit(x, w, bias=0.5) == 1.5


def test_logit_error_bound_random():
    cfg = inputs.WORKLOADS[0].with_(M=32, H=1024, E=16)
    w_router, bias, gamma, x = inputs.router_inputs(cfg)
    z32, z64 = oracle.router_logits(bf16_bits(x), bf16_bits(w_router), bias.numpy(), want_f64=True)
    xd, wd = bits_to_f64(bf16_bits(x)), bits_to_f64(bf16_bits(w_router))
    absdot = np.abs(xd) @ np.abs(wd).T
    bound = 2 * cfg.H * 2.0 ** -24 * absdot + np.abs(z64) * 2.0 ** -24
    assert (np.abs(z32.astype(np.float64) - z64) <= bound).all()
    # and the fp64 value is the plain dot product (numpy matmul as the library check)
    assert np.allclose(z64, xd @ wd.T + bias.numpy().astype(np.float64), rtol=0, atol=1e-12)


# ------------------------------------------------------------------ top-k
def _valid_topk_set(z, S, K):
    """S is the top-k set: every selected key beats every unselected one (ties -> lower id)."""
    if len(set(S)) != K:
        return False
    rest = [j for j in range(len(z)) if j not in S]
    for i in S:
        for j in rest:
            if not (z[i] > z[j] or (z[i] == z[j] and i < j)):
                return False
    return True


def test_topk_exhaustive_tiny():
    cfg = inputs.WORKLOADS[0]
    w_router, bias, gamma, x = inputs.router_inputs(cfg)
    z = oracle.router_logits(bf16_bits(x), bf16_bits(w_router), bias.numpy())
    ids, w = oracle.topk(z, cfg.K)
    for t in range(cfg.M):
        valid = [S for S in itertools.combinations(range(cfg.E), cfg.K) if _valid_topk_set(z[t], S, cfg.K)]
        assert len(valid) == 1
        assert sorted(ids[t].tolist()) == sorted(valid[0])
        # slot order: descending key, ties to lower id
        for a, b in zip(ids[t][:-1], ids[t][1:]):
            assert z[t, a] > z[t, b] or (z[t, a] == z[t, b] and a < b)


def test_topk_ties_and_signed_zero():
    z = np.array([[0.0, -0.0, 1.0, 1.0, -0.0, 0.0, 2.0, -1.0],
                  [-0.0, 0.0, 0.0, -0.0, -0.0, 0.0, 0.0, 0.0]], np.float32)
    ids, w = oracle.topk(z, 5)
    assert ids[0].tolist() == [6, 2, 3, 0, 1]
    assert ids[1].tolist() == [0, 1, 2, 3, 4]
    assert np.allclose(w[1], 0.2, rtol=0, atol=1e-15)


def test_topk_nan_logit_ranks_last():
    # A NaN logit (outside the workloads) is read as -inf: the selection is numpy's stable
    # lexicographic order on (key descending, id ascending) with NaN keys replaced by -inf,
    # and a NaN expert gets sigmoid weight 0; every id stays inside [0, E).
    rng = np.random.default_rng(17)
    z = rng.standard_normal((6, 40)).astype(np.float32)
    z[0, [3, 9, 30]] = np.nan
    z[1, :] = np.nan                  # a whole token of NaN: every key -inf, ids 0..K-1
    z[2, 5] = -np.inf
    z[2, 6] = np.nan                  # ties with the -inf at 5; 5 < 6 wins
    z[3, :37] = np.nan                # only 3 finite keys for K = 8
    K = 8
    ids, w = oracle.topk(z, K)
    key = np.where(np.isnan(z), -np.inf, z)
    for t in range(z.shape[0]):
        order = np.lexsort((np.arange(z.shape[1]), -key[t].astype(np.float64)))
        assert ids[t].tolist() == order[:K].tolist()
    assert ((ids >= 0) & (ids < z.shape[1])).all()
    assert not (ids[0][:, None] == np.array([3, 9, 30])[None, :]).any()
    assert ids[1].tolist() == list(range(K))
    assert np.isnan(w[1]).all()       # 0 / 0: every selected score is 0
    assert set(ids[3][:3].tolist()) == {37, 38, 39}
    assert (w[3][3:] == 0).all() and np.allclose(w[3][:3].sum(), 1.0, rtol=0, atol=1e-12)
    ids_ex, w_ex = oracle.topk_ex(z, K, oracle.SCORING_SIGMOID)
    assert np.array_equal(ids_ex, ids)


def test_weights_sum_order_and_ratio():
    rng = np.random.default_rng(5)
    z = (rng.standard_normal((64, 256)) * 2).astype(np.float32)
    K = 16
    ids, w = oracle.topk(z, K)
    assert np.allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert (np.diff(w, axis=1) <= 0).all()
    sel = np.take_along_axis(z, ids, axis=1).astype(np.float64)
    s = scipy.special.expit(sel)   # library sigmoid
    assert np.allclose(w, s / s.sum(axis=1, keepdims=True), rtol=1e-13, atol=0)


def test_route_all_configs_shapes_small():
    # the canonical order needs H % 256 == 0; every workload satisfies it
    for cfg in inputs.WORKLOADS.values():
        assert cfg.H % 256 == 0 and cfg.K <= cfg.E


# ------------------------------------------------------------------ routing variants
@pytest.mark.parametrize("renormalize", [True, False])
@pytest.mark.parametrize("scale", [1.0, 2.5])
def test_softmax_scoring_matches_scipy(renormalize, scale):
    rng = np.random.default_rng(31)
    z = (rng.standard_normal((40, 64)) * 3).astype(np.float32)
    ids, w = oracle.topk_ex(z, 6, oracle.SCORING_SOFTMAX, renormalize, scale)
    ids_s, _ = oracle.topk(z, 6)
    assert np.array_equal(ids, ids_s)                 # selection is the same
    p = scipy.special.softmax(z.astype(np.float64), axis=1)  # library softmax over all experts
    sel = np.take_along_axis(p, ids, axis=1)
    ref = (sel / sel.sum(axis=1, keepdims=True) if renormalize else sel) * scale
    assert np.allclose(w, ref, rtol=1e-12, atol=0)


def test_sigmoid_without_renormalisation_is_the_score():
    rng = np.random.default_rng(32)
    z = rng.standard_normal((20, 32)).astype(np.float32)
    ids, w = oracle.topk_ex(z, 4, oracle.SCORING_SIGMOID, False, 1.0)
    assert np.allclose(w, scipy.special.expit(np.take_along_axis(z, ids, axis=1).astype(np.float64)),
                       rtol=1e-13, atol=0)
    ids2, w2 = oracle.topk_ex(z, 4, oracle.SCORING_SIGMOID, True, 1.0)
    ids3, w3 = oracle.topk(z, 4)
    assert np.array_equal(ids2, ids3) and np.allclose(w2, w3, rtol=1e-15, atol=0)


def test_selection_only_bias():
    # The bias shifts which experts are picked but not their weights: the picked set is the one the
    # biased logit picks, and the weights are the renormalised sigmoid of the unbiased logit.
    cfg = inputs.WORKLOADS[0].with_(M=24, H=512, E=32, K=4)
    w_router, bias, gamma, x = inputs.router_inputs(cfg)
    b = (np.arange(cfg.E, dtype=np.float32) - cfg.E / 2) * 0.25   # large enough to change the picks
    ids, w = oracle.route_ex(bf16_bits(x), bf16_bits(w_router), b, cfg.K, bias_in_score=False)
    ids_biased, _ = oracle.route(bf16_bits(x), bf16_bits(w_router), b, cfg.K)
    assert np.array_equal(ids, ids_biased)
    z = oracle.router_logits(bf16_bits(x), bf16_bits(w_router), None).astype(np.float64)
    s = scipy.special.expit(np.take_along_axis(z, ids, axis=1))
    assert np.allclose(w, s / s.sum(axis=1, keepdims=True), rtol=1e-13, atol=0)
    # and the picks differ from the unbiased ones somewhere, so the bias did act
    ids_plain, _ = oracle.route(bf16_bits(x), bf16_bits(w_router), None, cfg.K)
    assert not np.array_equal(ids, ids_plain)
