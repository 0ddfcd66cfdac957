"""Pins for the oracle's number formats: bf16 rounding, e2m1 and e4m3 codecs.

The oracle's codecs are checked against the formats' published definitions
(written out here as value tables), against torch's own conversions where
torch has them, and against brute-force nearest-even searches.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests._util import bf16_nearest_even, f32_to_bf16_bits

pytestmark = pytest.mark.filterwarnings("ignore")


# ------------------------------------------------------------------ bf16
def test_bf16_value_all_patterns_match_torch():
    bits = np.arange(0, 1 << 16, 97, dtype=np.uint32).astype(np.uint16)
    ref = torch.as_tensor(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16_value(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def test_bf16_round_floats_match_torch():
    # For inputs that are already fp32, a one-step double->bf16 RNE equals
    # torch's fp32->bf16 RNE conversion (a library routine).
    rng = np.random.default_rng(11)
    vals = np.concatenate([
        rng.standard_normal(3000).astype(np.float32),
        (rng.standard_normal(500) * 1e-38).astype(np.float32),   # subnormal range
        (rng.standard_normal(500) * 1e37).astype(np.float32),    # near overflow
        np.array([0.0, -0.0, 1.0, -1.0, 3.3895314e38, 3.39e38, -3.39e38], np.float32),
    ])
    # exact ties: bf16 value + half a spacing
    base = rng.standard_normal(500).astype(np.float32)
    tb = (base.view(np.uint32) & 0xFFFF0000) | 0x8000
    vals = np.concatenate([vals, tb.view(np.float32)])
    ref = f32_to_bf16_bits(vals)
    got = np.array([oracle.bf16_round(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_round_doubles_brute_force():
    # Doubles with bits below fp32 precision: the one-step rounding must equal
    # an exact nearest-even search over the whole bf16 grid.
    rng = np.random.default_rng(12)
    vals = list(rng.standard_normal(400) * 10.0 ** rng.integers(-40, 38, 400))
    # values just above / below bf16 midpoints by less than one fp32 ulp:
    # a two-step double->float->bf16 rounding gets these wrong.
    for _ in range(200):
        b = int(rng.integers(0x0080, 0x7F00))
        lo = float(np.array([b << 16], np.uint32).view(np.float32)[0])
        hi = float(np.array([(b + 1) << 16], np.uint32).view(np.float32)[0])
        mid = (lo + hi) / 2
        vals += [mid, math.nextafter(mid, math.inf), math.nextafter(mid, -math.inf), -mid]
    vals += [0.0, -0.0, 1e-300, -1e-300, 3.3961e38, 3.3895e38, 1e39]
    for v in vals:
        assert oracle.bf16_round(v) == bf16_nearest_even(v), v


# ------------------------------------------------------------------ e2m1
# OCP Microscaling spec, FP4 E2M1: magnitudes by code 0..7.
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decode_table():
    for c in range(16):
        mag = E2M1_TABLE[c & 7]
        expect = -mag if c & 8 else mag
        got = oracle.e2m1_value(c)
        assert got == expect and math.copysign(1, got) == math.copysign(1, expect if c != 8 else -0.0)


def _nearest_even_grid(a, table):
    best = None
    for code, v in enumerate(table):
        d = abs(a - v)
        if best is None or d < best[0] or (d == best[0] and code % 2 == 0):
            best = (d, code)
    return best[1]


def test_e2m1_encode_brute_force_and_saturation():
    pts = set()
    for i in range(len(E2M1_TABLE) - 1):
        lo, hi = E2M1_TABLE[i], E2M1_TABLE[i + 1]
        mid = (lo + hi) / 2
        pts.update([lo, hi, mid, np.nextafter(np.float32(mid), np.float32(0)),
                    np.nextafter(np.float32(mid), np.float32(10))])
    pts.update(np.linspace(0, 6, 97).tolist())
    for a in sorted(float(p) for p in pts):
        expect = _nearest_even_grid(a, E2M1_TABLE)
        assert oracle.e2m1_encode(a) == expect, a
        assert oracle.e2m1_encode(-a) == (expect | 8), -a
    for big in [6.0, 6.5, 7.0, 8.0, 1e30]:
        assert oracle.e2m1_encode(big) == 7
        assert oracle.e2m1_encode(-big) == 15


# ------------------------------------------------------------------ e4m3
def _torch_e4m3_values():
    codes = torch.arange(256, dtype=torch.uint8)
    return codes.view(torch.float8_e4m3fn).double().numpy()


def test_e4m3_decode_matches_torch_and_definition():
    tv = _torch_e4m3_values()
    for c in range(256):
        got = oracle.e4m3_value(c)
        if np.isnan(tv[c]):
            assert math.isnan(got)
        else:
            assert got == tv[c], c
    # the definition: largest finite 448, smallest subnormal 2^-9
    assert oracle.e4m3_value(0x7E) == 448.0 and oracle.e4m3_value(0x01) == 2.0 ** -9
    assert oracle.e4m3_value(0x08) == 2.0 ** -6


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(13)
    vals = np.concatenate([
        rng.uniform(-464, 464, 4000), rng.standard_normal(2000) * 1e-2, rng.standard_normal(1000) * 1e-3,
    ]).astype(np.float32)
    tv = _torch_e4m3_values()
    mids = []
    pos = sorted(set(float(v) for v in tv if np.isfinite(v) and v >= 0))
    for lo, hi in zip(pos[:-1], pos[1:]):
        mids.append((lo + hi) / 2)
    vals = np.concatenate([vals, np.array(mids, np.float32), -np.array(mids, np.float32)])
    ref = torch.as_tensor(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in vals], np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_saturates():
    for big in [449.0, 464.0, 480.0, 1000.0, 1e30]:
        assert oracle.e4m3_encode(big) == 0x7E
        assert oracle.e4m3_encode(-big) == 0xFE


# ------------------------------------------------------------------ NVFP4 recipe
def test_nvfp4_global_scale():
    assert oracle.nvfp4_global_scale(0.0) == 1.0
    assert oracle.nvfp4_global_scale(2688.0) == 1.0
    assert oracle.nvfp4_global_scale(6.0) == np.float32(6.0) / np.float32(2688.0)


def test_nvfp4_zero_block_and_exact_block():
    # all-zero block -> scale 0 and codes 0
    v = np.zeros((1, 32), np.float32)
    v[0, 16:] = np.array(E2M1_TABLE + [-t for t in E2M1_TABLE], np.float32) * 4.0
    codes, scales = oracle.nvfp4_quantize(v, 1.0)
    assert scales[0, 0] == 0 and (codes[0, :16] == 0).all()
    # second block: amax 24 -> scale e4m3(24/6/1) = 4 exactly; codes are the e2m1 grid
    assert oracle.e4m3_value(int(scales[0, 1])) == 4.0
    expect = list(range(8)) + [c | 8 for c in range(8)]
    expect[8] = 8  # -0 encodes with the sign bit
    assert codes[0, 16:].tolist() == expect


def test_nvfp4_error_bound_random():
    # Dequantised value within half an e2m1 spacing (times the block scale),
    # plus the block scale's own rounding, of the input.
    rng = np.random.default_rng(14)
    v = (rng.standard_normal((64, 256)) * rng.uniform(0.01, 10, (64, 1))).astype(np.float32)
    amax = float(np.abs(v).max())
    gs = oracle.nvfp4_global_scale(amax)
    codes, scales = oracle.nvfp4_quantize(v, gs)
    deq = oracle.nvfp4_dequantize(codes, scales, gs)
    assert np.abs(deq).max() <= amax * (1 + 1 / 16) + 1e-12
    sb = np.vectorize(oracle.e4m3_value)(scales).astype(np.float64)
    step = np.repeat(sb * gs, 16, axis=1)  # one unit of the e2m1 grid
    # e2m1 spacing is <= 2 units at the top of the grid (4 -> 6)
    err = np.abs(deq - v.astype(np.float64))
    assert (err <= step * 1.0 + 1e-30).all()
    # block amax maps near the top of the grid: |q| max is 4 or 6 in each nonzero block
    q = np.vectorize(oracle.e2m1_value)(codes)
    blk = np.abs(q).reshape(64, 16, 16).max(axis=2)
    assert ((blk >= 4) | (blk == 0)).all()
