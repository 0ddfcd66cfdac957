"""The single-launch timeline tool's arithmetic on a hand-made trace (CPU): phase times from the first CTA's
start, producer waits per CTA, tile counts and the projection rate, from stamps written out here."""
import numpy as np
import pytest

from prefill_sigmoid_top_b200 import layer_trace as lt


def test_analysis_of_a_three_cta_trace():
    buf = np.zeros((lt.CTAS, lt.SLOTS), np.uint64)
    us = 1000  # stamps are nanoseconds
    base = 5_000_000
    for c, (start, barrier, plan, down, up_pub, down_pub, fs, fe, wr, ws, nu, nd) in enumerate([
            (0, 8, 18, 760, 840, 1160, 1170, 1180, 5, 300, 9, 4),
            (1, 8, 19, 770, 846, 1170, 1171, 1182, 7, 310, 8, 5),
            (2, 9, 19, 0, 830, 1165, 1172, 1183, 9, 320, 10, 3)]):
        row = buf[c]
        row[lt.START] = base + start * us
        row[lt.BARRIER] = base + barrier * us
        row[lt.PLAN] = base + plan * us
        row[lt.FIRST_DOWN] = 0 if down == 0 else base + down * us  # CTA 2 never claimed a down tile
        row[lt.LAST_UP_PUB] = base + up_pub * us
        row[lt.LAST_DOWN_PUB] = base + down_pub * us
        row[lt.FIN_START] = base + fs * us
        row[lt.FIN_END] = base + fe * us
        row[lt.WAIT_ROWS] = wr * us
        row[lt.WAIT_SLOT] = ws * us
        row[lt.UP_TILES] = nu
        row[lt.DOWN_TILES] = nd
        row[lt.END] = base + (fe + 1) * us
    r = lt.analyze(buf, weight_bytes=7.0e9)
    assert r["ctas"] == 3
    assert r["barrier"] == {"min": 8.0, "median": 8.0, "max": 9.0}
    assert r["first_down_claimed"]["min"] == pytest.approx(760.0)   # the CTA without a stamp is left out
    assert r["first_down_claimed"]["max"] == pytest.approx(770.0)
    assert r["last_up_published"]["max"] == pytest.approx(846.0)
    assert r["finalize_end"]["max"] == pytest.approx(1183.0)
    assert r["wait_rows_us_per_cta"] == pytest.approx(7.0)
    assert r["wait_slot_us_per_cta"] == pytest.approx(310.0)
    assert (r["up_tiles"], r["down_tiles"]) == (27, 12)
    assert r["projection_us"] == pytest.approx(1170.0 - 19.0)         # median plan -> last down published
    assert r["projection_TBps"] == pytest.approx(7.0e9 / (1151.0e-6) / 1e12)


def test_empty_trace():
    assert lt.analyze(np.zeros((lt.CTAS, lt.SLOTS), np.uint64)) == {}
