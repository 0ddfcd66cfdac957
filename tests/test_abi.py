"""The C-ABI library: loads, exports every symbol the header declares, validates on the host.

No compute call is made here: every call below fails host validation before
any CUDA work, so these tests run without a GPU (and launch nothing with one).
"""
import ctypes
import os
import re

import pytest

import prefill_sigmoid_top_b200 as moe
from prefill_sigmoid_top_b200 import _Plan, _Shape, _Weights, _Layout, _RouteOpts

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")
HEADERS = sorted(os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
                 if f.endswith(".h"))

FAKE = ctypes.c_void_p(0x10000)       # aligned non-null address, never dereferenced
FAKE_MIS = ctypes.c_void_p(0x10008)   # 8-byte aligned only


def declared_functions():
    """Every function that a header under include/ declares."""
    text = "".join(open(h).read() for h in HEADERS)
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text, re.M)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 15
    L = moe.library()
    for n in names:
        assert hasattr(L, n), n


def test_status_strings():
    for code, name in moe.STATUS.items():
        assert moe.status_string(code).startswith(name)


C0 = moe.Shape(M=16, H=256, I=128, E=8, top_k=2, block_size=16)
C1 = moe.Shape(M=8, H=7168, I=2048, E=256, top_k=16, block_size=16)


def test_sizes():
    assert moe.align_capacity(C0) == 16 * 2 + 8 * 15
    assert moe.align_capacity(C1) == 8 * 16 + 256 * 15
    assert moe.route_workspace_size(C1) >= 8 * 256 * 4
    lay = moe.layer_workspace_layout(C1)
    assert lay["total"] == moe.layer_workspace_size(C1)
    offs = [lay[k] for k in ["err_flag", "logits", "topk_ids", "topk_w", "sorted_ids", "block_expert",
                             "expert_counts", "expert_offsets", "num_tokens_post_padded", "h", "y"]]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert lay["y"] - lay["h"] >= moe.align_capacity(C1) * 2048 * 2
    assert lay["total"] - lay["y"] >= 8 * 16 * 7168 * 2


@pytest.mark.parametrize("shape", [C0, C1, moe.Shape(M=64, H=512, I=256, E=256, top_k=16, block_size=16),
                                   moe.Shape(M=200, H=512, I=256, E=64, top_k=4, block_size=16)],
                         ids=["C0", "C1", "M64_E256", "M200"])
def test_single_launch_counters_in_the_cleared_region(shape):
    """The single-launch layer's counters (grid barrier, work counter, finalize count, one up count per
    expert, and per token a slice count and 8 partial sums when M <= 64) sit after the error word and
    before the logits: the region moe_layer clears with one memset before every call."""
    lay = moe.layer_workspace_layout(shape)
    words = 3 + shape.E + (9 * shape.M if shape.M <= 64 else 0)
    assert lay["err_flag"] == 0
    assert lay["err_flag"] + 4 <= lay["sync"]
    assert lay["sync"] % 16 == 0
    assert lay["sync"] + 4 * words <= lay["logits"]


@pytest.mark.parametrize("bad", [
    dict(H=255), dict(H=8448), dict(I=64), dict(E=0), dict(E=1025), dict(top_k=0), dict(top_k=9),
    dict(block_size=24), dict(block_size=8), dict(block_size=512), dict(M=0),
])
def test_unsupported_shapes(bad):
    kw = dict(M=16, H=256, I=128, E=8, top_k=2, block_size=16)
    kw.update(bad)
    s = moe.Shape(**kw)
    assert moe.align_capacity(s) == 0
    L = moe.library()
    st = L.moe_route(FAKE, FAKE, None, s.c(), FAKE, FAKE, FAKE, 1 << 20, None)
    assert st == 2


def test_null_and_misaligned_pointers():
    L = moe.library()
    s = C0.c()
    assert L.moe_route(None, FAKE, None, s, FAKE, FAKE, FAKE, 1 << 20, None) == 1
    assert L.moe_route(FAKE_MIS, FAKE, None, s, FAKE, FAKE, FAKE, 1 << 20, None) == 1
    assert L.moe_route(FAKE, FAKE, None, s, FAKE, FAKE, None, 0, None) == 3   # no workspace
    assert L.moe_route(FAKE, FAKE, None, s, FAKE, FAKE, FAKE, 4, None) == 3   # too small
    assert L.moe_align_block_size(FAKE, s, None, FAKE, FAKE, FAKE, FAKE, None, None) == 1
    assert L.moe_finalize_rmsnorm(FAKE, FAKE, FAKE, FAKE, ctypes.c_float(1e-5), s, None, None, None) == 1
    assert L.moe_finalize_rmsnorm(FAKE, FAKE, FAKE, FAKE, ctypes.c_float(-1.0), s, FAKE, None, None) == 1
    w = _Weights(0, 0x10000, 0x10000, 0x10000, None, None, None)
    p = _Plan(0x10000, 0x10000, 0x10000, 0x10000, 0x10000)
    assert L.moe_grouped_up_swiglu(None, ctypes.byref(w), ctypes.byref(p), s, FAKE, None, 0, None, None) == 1
    assert L.moe_grouped_up_swiglu(FAKE, None, ctypes.byref(p), s, FAKE, None, 0, None, None) == 1
    assert L.moe_grouped_up_swiglu(FAKE, ctypes.byref(w), None, s, FAKE, None, 0, None, None) == 1
    assert L.moe_grouped_down(FAKE, ctypes.byref(w), ctypes.byref(p), s, FAKE_MIS, None, 0, None, None) == 1
    w_nv = _Weights(7, 0x10000, 0x10000, 0x10000, None, None, None)
    assert L.moe_grouped_down(FAKE, ctypes.byref(w_nv), ctypes.byref(p), s, FAKE, None, 0, None, None) == 2


def test_layer_workspace_checks():
    L = moe.library()
    s = C0.c()
    w = _Weights(0, 0x10000, 0x10000, 0x10000, None, None, None)
    need = moe.layer_workspace_size(C0)
    args = [FAKE, FAKE, None, ctypes.byref(w), FAKE, ctypes.c_float(1e-5), s, FAKE, None, None, None]
    assert L.moe_layer(*args, None, need, None) == 3
    assert L.moe_layer(*args, FAKE, need - 1, None) == 3
    assert L.moe_layer(FAKE, FAKE, None, None, FAKE, ctypes.c_float(1e-5), s, FAKE, None, None, None, FAKE, need,
                       None) == 1
    lay = _Layout()
    assert L.moe_layer_workspace_layout(s, 0, None) == 1
    assert L.moe_layer_workspace_layout(s, 0, ctypes.byref(lay)) == 0 and lay.total == need


def test_device_error_rejects_null():
    code = ctypes.c_int32(0)
    assert moe.library().moe_get_device_error(None, None, ctypes.byref(code)) == 1


def test_measure_calls_reject_bad_arguments():
    L = moe.library()
    panel = 128 * 7168 * 2  # one 128-row panel of the stream's [rows, 7168] bf16 view
    moved = ctypes.c_size_t(0)

    def tma(buf, nbytes, boxes, stages, steps, warps=1):
        return L.moe_measure_tma_stream(buf, nbytes, boxes, stages, 0, warps, steps, None, ctypes.byref(moved),
                                        None)

    assert tma(None, panel, 2, 5, 10) == 1
    assert tma(FAKE_MIS, panel, 2, 5, 10) == 1
    assert tma(FAKE, panel - 1, 2, 5, 10) == 1      # under one panel
    assert tma(FAKE, panel, 0, 5, 10) == 1          # boxes outside 1..3
    assert tma(FAKE, panel, 4, 2, 10) == 1
    assert tma(FAKE, panel, 1, 1, 10) == 1          # stages outside 2..16
    assert tma(FAKE, panel, 1, 17, 10) == 1
    assert tma(FAKE, panel, 3, 5, 10) == 1          # 240 KB ring: above 192 KB
    assert tma(FAKE, panel, 2, 5, 0) == 1           # no steps
    assert tma(FAKE, panel, 2, 4, 10, warps=0) == 1  # warps outside 1..4
    assert tma(FAKE, panel, 1, 8, 10, warps=5) == 1
    assert tma(FAKE, panel, 2, 5, 10, warps=2) == 1  # stages not a multiple of warps

    def mix(buf, nbytes, m, stages, steps):
        return L.moe_measure_tma_mix(buf, nbytes, m, stages, steps, None, ctypes.byref(moved), None)

    big = 256 << 20
    assert mix(None, big, 2, 4, 100) == 1
    assert mix(FAKE_MIS, big, 2, 4, 100) == 1
    assert mix(FAKE, big - 16, 2, 4, 100) == 1     # under 256 MB
    assert mix(FAKE, big, -1, 4, 100) == 1         # mix outside 0..4
    assert mix(FAKE, big, 5, 4, 100) == 1
    assert mix(FAKE, big, 2, 1, 100) == 1          # stages outside 2..4
    assert mix(FAKE, big, 2, 5, 100) == 1
    assert mix(FAKE, big, 2, 4, 7) == 1            # fewer than 8 steps
    assert moved.value == 0
    assert L.moe_measure_hbm_read(None, 1024, None, None) == 1
    assert L.moe_measure_hbm_read(FAKE, 1000, None, None) == 1


def test_selftest_rejects_bad_arguments():
    L = moe.library()
    assert L.moe_selftest_wait_timeout(None, 1000, None) == 1
    assert L.moe_selftest_wait_timeout(FAKE, 0, None) == 1
    assert L.moe_selftest_wait_timeout(FAKE, 2_000_000, None) == 1


def test_route_ex_rejects_bad_options():
    L = moe.library()
    s = C0.c()
    ok = _RouteOpts(moe.SCORE_SOFTMAX, 1, 1, 1.0)
    args = lambda o: (FAKE, FAKE, None, s, o, FAKE, FAKE, FAKE, 1 << 20, None)
    assert L.moe_route_ex(*args(None)) == 1
    assert L.moe_route_ex(*args(ctypes.byref(_RouteOpts(2, 1, 1, 1.0)))) == 1
    assert L.moe_route_ex(*args(ctypes.byref(_RouteOpts(1, 1, 1, 0.0)))) == 1
    assert L.moe_route_ex(*args(ctypes.byref(_RouteOpts(1, 1, 1, float("inf"))))) == 1
    assert L.moe_route_ex(*args(ctypes.byref(_RouteOpts(1, 1, 1, float("nan"))))) == 1
    assert L.moe_route_ex(FAKE, FAKE, None, s, ctypes.byref(ok), FAKE, FAKE, FAKE, 4, None) == 3
    assert L.moe_route_ex(FAKE_MIS, FAKE, None, s, ctypes.byref(ok), FAKE, FAKE, FAKE, 1 << 20, None) == 1


def test_routed_up_rejects_bad_arguments():
    L = moe.library()
    w = _Weights(0, 0x10000, 0x10000, 0x10000, None, None, None)
    args = lambda shape, wp: (FAKE, wp, FAKE, shape.c(), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None)
    big = moe.Shape(M=129, H=256, I=128, E=8, top_k=8, block_size=16)  # 1032 slots > 1024
    assert L.moe_grouped_up_swiglu_routed(*args(big, ctypes.byref(w))) == 2
    w_nv = _Weights(1, 0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 0x10000)
    assert L.moe_grouped_up_swiglu_routed(*args(C0, ctypes.byref(w_nv))) == 2
    assert L.moe_grouped_up_swiglu_routed(*args(C0, None)) == 1
    a = list(args(C0, ctypes.byref(w)))
    a[0] = FAKE_MIS
    assert L.moe_grouped_up_swiglu_routed(*a) == 1
    a = list(args(C0, ctypes.byref(w)))
    a[4] = None
    assert L.moe_grouped_up_swiglu_routed(*a) == 1


def test_layer_kernel_count(monkeypatch):
    assert moe.layer_kernel_count(C1) == 1            # decode: the whole layer in one launch
    monkeypatch.setenv("MOE_FUSED_LAYER", "0")
    assert moe.layer_kernel_count(C1) == 5            # decode, separate launches: align folded into up
    monkeypatch.delenv("MOE_FUSED_LAYER")
    many_experts = moe.Shape(M=2, H=7168, I=2048, E=512, top_k=8, block_size=16)
    assert moe.layer_kernel_count(many_experts) == 5  # the single launch takes E <= 256
    # from 128 tokens the routing is screened: digits, integer partial logits, then one kernel for the
    # candidates, their exact logits and the top-k
    batch = moe.Shape(M=512, H=7168, I=2048, E=256, top_k=16, block_size=64)
    assert moe.layer_kernel_count(batch) == 7         # routing 3, align; the up kernel gathers x rows itself
    prefill = moe.Shape(M=2048, H=7168, I=2048, E=256, top_k=16, block_size=128)
    assert moe.layer_kernel_count(prefill) == 8       # routing 3, align and a gather pass of x (256-row tiles)
    monkeypatch.setenv("MOE_PAIR_GATHER", "0")
    assert moe.layer_kernel_count(batch) == 8
    monkeypatch.delenv("MOE_PAIR_GATHER")
    assert moe.layer_kernel_count(batch, moe.MOE_W_NVFP4) == 11
    monkeypatch.setenv("MOE_ROUTER_SCREEN", "0")      # logits of every expert + top-k
    assert moe.layer_kernel_count(batch) == 6
    assert moe.layer_kernel_count(prefill) == 7
    assert moe.layer_kernel_count(batch, moe.MOE_W_NVFP4) == 10
    monkeypatch.delenv("MOE_ROUTER_SCREEN")
    assert moe.layer_kernel_count(moe.Shape(M=16, H=255, I=128, E=8, top_k=2, block_size=16)) == -1
