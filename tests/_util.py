"""Helpers shared by the tests (independent of both the oracle and the CUDA library)."""
from __future__ import annotations

import bisect
from fractions import Fraction

import numpy as np
import torch

# ------------------------------------------------------------------ bf16 grid
# All finite non-negative bf16 values, exactly, sorted (the bit patterns
# 0x0000..0x7F7F are monotone in value).
_BF16_POS_BITS = np.arange(0, 0x7F80, dtype=np.uint32)
_BF16_POS_VALS = (_BF16_POS_BITS << 16).view(np.float32).astype(np.float64)
_BF16_MAX = float(_BF16_POS_VALS[-1])


def bf16_nearest_even(v: float) -> int:
    """Brute-force round-to-nearest-even of a double onto the bf16 grid.

    Searches the sorted list of all finite bf16 magnitudes and compares the
    two neighbours with exact rational arithmetic.  Beyond the largest finite
    value plus half a spacing the result is infinity.
    """
    if v != v:
        return 0x7FC0
    sign = 0x8000 if np.signbit(v) else 0
    a = abs(v)
    if a == float("inf"):
        return sign | 0x7F80
    half_top = Fraction(_BF16_MAX) + (Fraction(_BF16_MAX) - Fraction(float(_BF16_POS_VALS[-2]))) / 2
    if Fraction(a) >= half_top:
        return sign | 0x7F80
    i = bisect.bisect_left(_BF16_POS_VALS, a)
    if i < len(_BF16_POS_VALS) and _BF16_POS_VALS[i] == a:
        return sign | int(_BF16_POS_BITS[i])
    lo_i, hi_i = i - 1, i
    if hi_i >= len(_BF16_POS_VALS):
        return sign | int(_BF16_POS_BITS[lo_i])
    fa, flo, fhi = Fraction(a), Fraction(float(_BF16_POS_VALS[lo_i])), Fraction(float(_BF16_POS_VALS[hi_i]))
    dlo, dhi = fa - flo, fhi - fa
    if dlo < dhi:
        pick = lo_i
    elif dhi < dlo:
        pick = hi_i
    else:
        pick = lo_i if (_BF16_POS_BITS[lo_i] & 1) == 0 else hi_i
    return sign | int(_BF16_POS_BITS[pick])


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 values."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f32_to_bf16_bits(v) -> np.ndarray:
    """float32 values -> bf16 bits via torch's own conversion (round-to-nearest-even)."""
    t = torch.as_tensor(np.asarray(v, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_tensor_from_f64(v) -> torch.Tensor:
    """Exactly representable values -> torch bf16 tensor (asserts exactness)."""
    a = np.asarray(v, dtype=np.float64)
    t = torch.as_tensor(a.astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(t.double().numpy(), a), "value not representable in bf16"
    return t


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def rms(a) -> float:
    a = np.asarray(a, dtype=np.float64)
    return float(np.sqrt(np.mean(a * a)))


def sample_tokens(ids_o, n_total, seed, tile):
    """Tokens checked at full size: every token routed to the coldest touched expert; the first two and
    all of the last (ragged) `tile`-row token tile of the hottest expert (its slots in ascending slot id,
    the plan order); then random tokens up to n_total."""
    M, K = ids_o.shape
    flat = ids_o.ravel()
    counts = np.bincount(flat)
    hot = int(np.argmax(counts))
    cold = int(np.argmin(np.where(counts > 0, counts, np.iinfo(np.int64).max)))
    hot_slots = np.nonzero(flat == hot)[0]
    last_tile = hot_slots[(len(hot_slots) - 1) // tile * tile:]
    pick = set(int(s) // K for s in hot_slots[:2]) | set(int(s) // K for s in last_tile)
    pick |= set(int(s) // K for s in np.nonzero(flat == cold)[0])
    rng = np.random.default_rng(seed)
    for t in rng.permutation(M):
        if len(pick) >= n_total:
            break
        pick.add(int(t))
    return np.array(sorted(pick), np.int32)


def token_tile(cfg):
    """Token-tile width of the workload's grouped kernels (2-SM pairs: 256 rows from 96 routed rows per
    expert on average, else 128; NVFP4: 128; decode shapes: 32)."""
    per_expert = cfg.M * cfg.K / cfg.E
    if cfg.wdtype == "nvfp4":
        return 128
    return 32 if per_expert <= 24 else (256 if per_expert >= 96 else 128)
