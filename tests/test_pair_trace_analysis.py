"""The pair-GEMM timeline tool's arithmetic on a hand-made trace (CPU): spans, per-N means, gaps between a
pair's tiles and the pairs' end times, from stamps whose values are written out here."""
import numpy as np
import pytest

from prefill_sigmoid_top_b200 import pair_trace


def _stamp(buf, kind, tile, e, w, t, N, start, ready, mma_end, epi_start, released):
    meta = e | (w << 12) | (t << 20) | (N << 28)
    buf[kind, tile, :6] = [meta, start, ready, mma_end, epi_start, released]


def test_analysis_of_a_two_pair_trace():
    buf = np.zeros((2, 8192, 8), np.uint64)
    us = 1000  # stamps are nanoseconds
    # two pairs; tiles 0, 2 on pair 0 and 1, 3 on pair 1 (round-robin)
    _stamp(buf, 0, 0, 0, 0, 0, 256, 1 * us, 2 * us, 81 * us, 81 * us, 87 * us)
    _stamp(buf, 0, 1, 0, 1, 0, 32, 1 * us, 2 * us, 81 * us, 81 * us, 83 * us)
    _stamp(buf, 0, 2, 1, 0, 0, 32, 87 * us, 88 * us, 167 * us, 167 * us, 169 * us)
    _stamp(buf, 0, 3, 1, 1, 0, 256, 83 * us, 84 * us, 163 * us, 163 * us, 169 * us)
    r = pair_trace.analyze(buf, 2)
    up = r["up"]
    assert up["tiles"] == 4 and "down" not in r
    assert up["span"] == pytest.approx(168.0)          # from the first start (1 us) to the last stamp (169 us)
    assert up["by_N"][256]["mainloop"] == pytest.approx(80.0)
    assert up["by_N"][256]["drain"] == pytest.approx(6.0)
    assert up["by_N"][32]["drain"] == pytest.approx(2.0)
    assert up["gap_mean"] == pytest.approx(((87 - 81) + (83 - 81)) / 2)  # next start - previous last MMA
    assert up["gap_per_pair"] == pytest.approx(8.0 / 2)
    assert up["pair_end"]["min"] == pytest.approx(168.0) and up["pair_end"]["max"] == pytest.approx(168.0)
