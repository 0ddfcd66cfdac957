"""moe_route_noalloc: routing for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc (for example a plugin inside a host
framework that owns every device allocation, or code with a fixed, pre-budgeted
footprint), so they cannot hand moe_route its logits scratch buffer.
moe_route_noalloc keeps that scratch in a fixed array inside the library.
This test calls it through the C ABI and checks it against moe_route on two
calls in a row with different shapes.  Both run the same kernels, so ids, slot
order and weights must be the same bits (stricter than the 1e-6 weight
tolerance the oracle comparisons use).  It lives in a file of its
own that pytest collects last.
"""
import ctypes

import numpy as np
import pytest
import torch

import prefill_sigmoid_top_b200 as moe
from prefill_sigmoid_top_b200 import inputs

pytestmark = pytest.mark.gpu

MAX_LOGITS = 1 << 20  # MOE_ROUTE_NOALLOC_MAX_LOGITS in include/moe_b200.h


def _noalloc(x, w_router, bias, K):
    M, H = x.shape
    E = w_router.shape[0]
    ids = torch.full((M, K), -1, dtype=torch.int32, device=x.device)
    w = torch.full((M, K), float("nan"), dtype=torch.float32, device=x.device)
    shape = moe.Shape(M, H, 128, E, K, 16).c()
    st = moe.library().moe_route_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(w_router.data_ptr()),
                                         ctypes.c_void_p(bias.data_ptr()), shape, ctypes.c_void_p(ids.data_ptr()),
                                         ctypes.c_void_p(w.data_ptr()),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, ids, w


def test_route_noalloc_matches_route_on_two_calls():
    cases = [inputs.WORKLOADS[1], inputs.WORKLOADS[0].with_(M=37, H=1024, E=64, K=8, bias="normal", seed=9)]
    for cfg in cases:  # two calls in a row; the second reuses the array the first wrote
        w_r, b, _, x = inputs.router_inputs(cfg)
        x, w_r, b = x.cuda(), w_r.cuda(), b.cuda()
        ids_ref, w_ref = moe.route(x, w_r, b, cfg.K)
        st, ids, w = _noalloc(x, w_r, b, cfg.K)
        assert st == 0, moe.status_string(st)
        torch.cuda.synchronize()
        assert torch.equal(ids, ids_ref)
        assert torch.equal(w, w_ref)


def test_route_noalloc_rejects_more_logits_than_the_array_holds():
    E = 256
    M = MAX_LOGITS // E + 1
    x = torch.zeros(M, 256, dtype=torch.bfloat16, device="cuda")
    w_r = torch.zeros(E, 256, dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(E, dtype=torch.float32, device="cuda")
    st, ids, _ = _noalloc(x, w_r, b, 4)
    assert st == 2  # MOE_ERR_UNSUPPORTED, nothing launched
    torch.cuda.synchronize()
    assert (ids == -1).all()
