"""Pins for the oracle's expert-major block plan (moe_align_block_size)."""
import numpy as np
import pytest

import oracle


def _check_plan(ids, E, B):
    M, K = ids.shape
    p = oracle.align(ids, E, B)
    assert p["status"] == 0
    flat = ids.ravel()
    n = M * K
    counts = np.bincount(flat, minlength=E)                      # library histogram
    assert np.array_equal(p["counts"], counts)
    padded = (counts + B - 1) // B * B
    assert np.array_equal(p["offsets"], np.concatenate([[0], np.cumsum(padded)]))
    assert p["ntpp"] == int(padded.sum())
    assert (p["offsets"] % B == 0).all()
    s = p["sorted_ids"]
    # real entries: exactly the stable sort of slots by expert (library stable sort)
    order = np.argsort(flat, kind="stable")
    real = s[s != n]
    assert np.array_equal(real, order)
    # each expert's entries sit at the start of its segment, then padding
    for e in range(E):
        seg = s[p["offsets"][e]:p["offsets"][e + 1]]
        assert (seg[:counts[e]] < n).all() and (flat[seg[:counts[e]]] == e).all()
        assert (seg[counts[e]:] == n).all()
    # block -> expert equals a linear scan of the padded prefix (library searchsorted)
    nb = p["ntpp"] // B
    expect = np.searchsorted(p["offsets"], np.arange(nb) * B, side="right") - 1
    assert np.array_equal(p["block_expert"], expect)
    # blocks of empty experts never appear
    assert all(counts[e] > 0 for e in p["block_expert"])
    return p


@pytest.mark.parametrize("M,K,E,B", [(16, 2, 8, 16), (8, 16, 256, 16), (37, 5, 64, 32), (1, 1, 1, 16),
                                     (512, 16, 256, 64), (300, 8, 1024, 256), (5, 3, 3, 128)])
def test_plan_invariants_random(M, K, E, B):
    rng = np.random.default_rng(M * 131 + E)
    # distinct experts per token, as routing produces
    ids = np.stack([rng.choice(E, size=K, replace=False) for _ in range(M)]).astype(np.int32)
    _check_plan(ids, E, B)


def test_plan_skewed_and_empty_experts():
    rng = np.random.default_rng(3)
    E, K, M, B = 64, 4, 200, 16
    p_e = np.zeros(E)
    p_e[:10] = 1.0
    ids = np.stack([rng.choice(E, size=K, replace=False, p=p_e / p_e.sum()) for _ in range(M)]).astype(np.int32)
    p = _check_plan(ids, E, B)
    assert (p["counts"][10:] == 0).all()
    assert np.array_equal(p["offsets"][11:], np.full(E - 10, p["offsets"][10]))


def test_plan_hand_case():
    # 3 tokens, top-2, 3 experts, block 4:  slots f = 0..5 -> experts [2,0, 0,2, 2,1]
    ids = np.array([[2, 0], [0, 2], [2, 1]], np.int32)
    p = oracle.align(ids, 3, 4)
    assert p["counts"].tolist() == [2, 1, 3]
    assert p["offsets"].tolist() == [0, 4, 8, 12]
    assert p["sorted_ids"].tolist() == [1, 2, 6, 6, 5, 6, 6, 6, 0, 3, 4, 6]
    assert p["block_expert"].tolist() == [0, 1, 2]


@pytest.mark.parametrize("bad", [-1, 8, 1 << 20])
def test_out_of_range_id_rejected(bad):
    ids = np.array([[0, 1], [2, bad]], np.int32)
    assert oracle.align(ids, 8, 16)["status"] == 4
