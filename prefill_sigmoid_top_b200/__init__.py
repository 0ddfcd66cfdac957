"""Python binding of libmoe_b200.so, the B200 (sm_100a) routed-MoE layer library.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels (see include/moe_b200.h for the operations and their definitions).
Tensors are torch CUDA tensors; the library is called on
``torch.cuda.current_stream()``.  There is no CPU fallback: if the library
cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

import torch

__all__ = [
    "MoEError", "Shape", "library", "route", "align_block_size", "grouped_up_swiglu", "grouped_down",
    "finalize_rmsnorm", "layer", "layer_workspace_size", "up_workspace_size", "layer_workspace_layout", "align_capacity",
    "route_workspace_size", "get_device_error", "status_string", "STATUS", "NVFP4Weights", "quantize_nvfp4",
    "prepare_nvfp4_weights", "nvfp4_weights", "nvfp4_blob_bytes", "grouped_up_swiglu_nvfp4", "grouped_down_nvfp4",
    "layer_nvfp4", "down_workspace_size",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libmoe_b200.so")
_lock = threading.Lock()
_lib = None

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_INVALID_INPUT", 5: "MOE_ERR_TIMEOUT", 6: "MOE_ERR_CUDA"}
MOE_W_BF16, MOE_W_NVFP4 = 0, 1


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}" if what else status_string(status))


class _Shape(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32), ("E", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("block_size", ctypes.c_int32)]


class _Weights(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("gate", ctypes.c_void_p), ("up", ctypes.c_void_p),
                ("down", ctypes.c_void_p), ("gate_gs", ctypes.c_void_p), ("up_gs", ctypes.c_void_p),
                ("down_gs", ctypes.c_void_p)]


class _Plan(ctypes.Structure):
    _fields_ = [("sorted_ids", ctypes.c_void_p), ("block_expert", ctypes.c_void_p),
                ("expert_counts", ctypes.c_void_p), ("expert_offsets", ctypes.c_void_p),
                ("num_tokens_post_padded", ctypes.c_void_p)]


class _RouteOpts(ctypes.Structure):
    _fields_ = [("scoring", ctypes.c_int32), ("renormalize", ctypes.c_int32), ("bias_in_score", ctypes.c_int32),
                ("routed_scale", ctypes.c_float)]


SCORE_SOFTMAX, SCORE_SIGMOID = 0, 1

_LAYOUT_FIELDS = ["err_flag", "logits", "topk_ids", "topk_w", "sorted_ids", "block_expert", "expert_counts",
                  "expert_offsets", "num_tokens_post_padded", "h", "y", "act_scratch", "sync", "total"]


class _Layout(ctypes.Structure):
    _fields_ = [(f, ctypes.c_size_t) for f in _LAYOUT_FIELDS]


@dataclass(frozen=True)
class Shape:
    M: int
    H: int
    I: int
    E: int
    top_k: int
    block_size: int

    def c(self) -> _Shape:
        return _Shape(self.M, self.H, self.I, self.E, self.top_k, self.block_size)


def _declare(L):
    vp, sz, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    sig = {
        "moe_status_string": (ctypes.c_char_p, [st]),
        "moe_route": (st, [vp, vp, vp, _Shape, vp, vp, vp, sz, vp]),
        "moe_route_workspace_size": (sz, [_Shape]),
        "moe_route_ex": (st, [vp, vp, vp, _Shape, ctypes.POINTER(_RouteOpts), vp, vp, vp, sz, vp]),
        "moe_align_block_size": (st, [vp, _Shape, vp, vp, vp, vp, vp, vp, vp]),
        "moe_align_capacity": (sz, [_Shape]),
        "moe_grouped_up_swiglu": (st, [vp, ctypes.POINTER(_Weights), ctypes.POINTER(_Plan), _Shape, vp, vp, sz,
                                       vp, vp]),
        "moe_up_workspace_size": (sz, [_Shape, ctypes.c_int]),
        "moe_grouped_down": (st, [vp, ctypes.POINTER(_Weights), ctypes.POINTER(_Plan), _Shape, vp, vp, sz, vp,
                                  vp]),
        "moe_down_workspace_size": (sz, [_Shape, ctypes.c_int]),
        "moe_grouped_up_swiglu_routed": (st, [vp, ctypes.POINTER(_Weights), vp, _Shape, vp, vp, vp, vp, vp, vp, vp,
                                              vp]),
        "moe_finalize_rmsnorm": (st, [vp, vp, vp, vp, ctypes.c_float, _Shape, vp, vp, vp]),
        "moe_layer": (st, [vp, vp, vp, ctypes.POINTER(_Weights), vp, ctypes.c_float, _Shape, vp, vp, vp, vp, vp,
                           sz, vp]),
        "moe_layer_workspace_size": (sz, [_Shape, ctypes.c_int]),
        "moe_layer_kernel_count": (ctypes.c_int, [_Shape, ctypes.c_int]),
        "moe_layer_workspace_layout": (st, [_Shape, ctypes.c_int, ctypes.POINTER(_Layout)]),
        "moe_quantize_nvfp4": (st, [vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, vp, vp, vp, vp, sz, vp]),
        "moe_nvfp4_quantize_workspace_size": (sz, [ctypes.c_int64]),
        "moe_prepare_nvfp4_weights": (st, [vp, vp, _Shape, ctypes.c_int, vp, sz, vp]),
        "moe_nvfp4_blob_bytes": (sz, [_Shape, ctypes.c_int]),
        "moe_get_device_error": (st, [vp, vp, ctypes.POINTER(ctypes.c_int32)]),
        "moe_route_noalloc": (st, [vp, vp, vp, _Shape, vp, vp, vp]),
        "moe_selftest_wait_timeout": (st, [vp, ctypes.c_uint32, vp]),
        "moe_measure_hbm_read": (st, [vp, sz, vp, vp]),
        "moe_measure_tma_stream": (st, [vp, sz, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, vp, ctypes.POINTER(ctypes.c_size_t), vp]),
        "moe_measure_tma_mix": (st, [vp, sz, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp,
                                     ctypes.POINTER(ctypes.c_size_t), vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args


def library():
    """The loaded libmoe_b200.so (built in-tree on first use if it is missing)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                from . import build as _build
                _build.build()
            L = ctypes.CDLL(_LIB_PATH)
            _declare(L)
            _lib = L
    return _lib


def status_string(status: int) -> str:
    return library().moe_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != 0:
        raise MoEError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("moe_b200 operates on CUDA tensors only")


def _bf16(t):
    if t.dtype != torch.bfloat16 or not t.is_contiguous():
        raise ValueError("expected a contiguous bf16 tensor")
    return t


def _weights_struct(w_gate, w_up, w_down):
    return _Weights(MOE_W_BF16, w_gate.data_ptr(), w_up.data_ptr(), w_down.data_ptr(), None, None, None)


# ------------------------------------------------------------------ sizes
def align_capacity(shape: Shape) -> int:
    return int(library().moe_align_capacity(shape.c()))


def route_workspace_size(shape: Shape) -> int:
    return int(library().moe_route_workspace_size(shape.c()))


def layer_workspace_size(shape: Shape, wdtype: int = MOE_W_BF16) -> int:
    return int(library().moe_layer_workspace_size(shape.c(), wdtype))


def layer_workspace_layout(shape: Shape, wdtype: int = MOE_W_BF16) -> dict:
    lay = _Layout()
    _check(library().moe_layer_workspace_layout(shape.c(), wdtype, ctypes.byref(lay)), "moe_layer_workspace_layout")
    return {f: int(getattr(lay, f)) for f in _LAYOUT_FIELDS}


# ------------------------------------------------------------------ steps
def route(x, w_router, bias, top_k, topk_ids=None, topk_w=None, ws=None):
    """Sigmoid top-k routing -> (topk_ids int32 [M,K], topk_w fp32 [M,K])."""
    _need_cuda(x, w_router, bias)
    M, H = x.shape
    E = w_router.shape[0]
    shape = Shape(M, H, 128, E, top_k, 16)
    if topk_ids is None:
        topk_ids = torch.empty(M, top_k, dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty(M, top_k, dtype=torch.float32, device=x.device)
    need = route_workspace_size(shape)
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _check(library().moe_route(_ptr(_bf16(x)), _ptr(_bf16(w_router)), _ptr(bias), shape.c(), _ptr(topk_ids),
                               _ptr(topk_w), _ptr(ws), ws.numel(), _stream()), "moe_route")
    return topk_ids, topk_w


def route_ex(x, w_router, bias, top_k, scoring=SCORE_SIGMOID, renormalize=True, routed_scale=1.0,
             bias_in_score=True, topk_ids=None, topk_w=None, ws=None):
    """Routing variants: softmax or sigmoid scores, optional renormalisation, a routed scale, and a bias
    that is part of the logit or only shifts the selection key -> (topk_ids, topk_w)."""
    _need_cuda(x, w_router, bias)
    M, H = x.shape
    E = w_router.shape[0]
    shape = Shape(M, H, 128, E, top_k, 16)
    if topk_ids is None:
        topk_ids = torch.empty(M, top_k, dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty(M, top_k, dtype=torch.float32, device=x.device)
    need = route_workspace_size(shape)
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    opts = _RouteOpts(int(scoring), int(bool(renormalize)), int(bool(bias_in_score)), float(routed_scale))
    _check(library().moe_route_ex(_ptr(_bf16(x)), _ptr(_bf16(w_router)), _ptr(bias), shape.c(), ctypes.byref(opts),
                                  _ptr(topk_ids), _ptr(topk_w), _ptr(ws), ws.numel(), _stream()), "moe_route_ex")
    return topk_ids, topk_w


def align_block_size(topk_ids, E, block_size, err_flag=None, out=None):
    """Expert-major plan -> dict of device tensors (sorted_ids, block_expert, expert_counts,
    expert_offsets, num_tokens_post_padded)."""
    _need_cuda(topk_ids)
    M, K = topk_ids.shape
    shape = Shape(M, 256, 128, E, K, block_size)
    cap = align_capacity(shape)
    if cap == 0:
        raise MoEError(2, "moe_align_capacity")
    dev = topk_ids.device
    if out is None:
        out = dict(sorted_ids=torch.empty(cap, dtype=torch.int32, device=dev),
                   block_expert=torch.empty(cap // block_size + 1, dtype=torch.int32, device=dev),
                   expert_counts=torch.empty(E, dtype=torch.int32, device=dev),
                   expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
                   num_tokens_post_padded=torch.empty(1, dtype=torch.int32, device=dev))
    _check(library().moe_align_block_size(_ptr(topk_ids), shape.c(), _ptr(out["sorted_ids"]),
                                          _ptr(out["block_expert"]), _ptr(out["expert_counts"]),
                                          _ptr(out["expert_offsets"]), _ptr(out["num_tokens_post_padded"]),
                                          _ptr(err_flag), _stream()), "moe_align_block_size")
    return out


def _plan_struct(plan):
    return _Plan(plan["sorted_ids"].data_ptr(), plan["block_expert"].data_ptr(), plan["expert_counts"].data_ptr(),
                 plan["expert_offsets"].data_ptr(), plan["num_tokens_post_padded"].data_ptr())


def layer_kernel_count(shape: Shape, wdtype: int = MOE_W_BF16) -> int:
    """Kernels one moe_layer call launches for this shape (host-side count)."""
    return int(library().moe_layer_kernel_count(shape.c(), wdtype))


def up_workspace_size(shape: Shape, wdtype: int = MOE_W_BF16) -> int:
    return int(library().moe_up_workspace_size(shape.c(), wdtype))


def grouped_up_swiglu(x, w_gate, w_up, plan, shape: Shape, h=None, err_flag=None, ws=None):
    """h[cap, I] = bf16(silu(x W_gate^T) * (x W_up^T)) in plan order."""
    _need_cuda(x, w_gate, w_up)
    if h is None:
        h = torch.empty(align_capacity(shape), shape.I, dtype=torch.bfloat16, device=x.device)
    if ws is None:
        need = up_workspace_size(shape)
        ws = torch.empty(need, dtype=torch.uint8, device=x.device) if need else None
    w = _weights_struct(w_gate, w_up, w_up)
    p = _plan_struct(plan)
    _check(library().moe_grouped_up_swiglu(_ptr(_bf16(x)), ctypes.byref(w), ctypes.byref(p), shape.c(), _ptr(h),
                                           _ptr(ws), 0 if ws is None else ws.numel(), _ptr(err_flag), _stream()),
           "moe_grouped_up_swiglu")
    return h


def grouped_up_swiglu_routed(x, w_gate, w_up, topk_ids, shape: Shape, h=None, plan=None, err_flag=None):
    """Align + up projection in one launch: returns (h [cap, I] in plan order, plan dict of device tensors)."""
    _need_cuda(x, w_gate, w_up, topk_ids)
    cap = align_capacity(shape)
    if cap == 0:
        raise MoEError(2, "moe_align_capacity")
    dev = x.device
    if h is None:
        h = torch.empty(cap, shape.I, dtype=torch.bfloat16, device=dev)
    if plan is None:
        plan = dict(sorted_ids=torch.empty(cap, dtype=torch.int32, device=dev),
                    block_expert=torch.empty(cap // shape.block_size + 1, dtype=torch.int32, device=dev),
                    expert_counts=torch.empty(shape.E, dtype=torch.int32, device=dev),
                    expert_offsets=torch.empty(shape.E + 1, dtype=torch.int32, device=dev),
                    num_tokens_post_padded=torch.empty(1, dtype=torch.int32, device=dev))
    w = _weights_struct(w_gate, w_up, w_up)
    _check(library().moe_grouped_up_swiglu_routed(
        _ptr(_bf16(x)), ctypes.byref(w), _ptr(topk_ids), shape.c(), _ptr(plan["sorted_ids"]),
        _ptr(plan["block_expert"]), _ptr(plan["expert_counts"]), _ptr(plan["expert_offsets"]),
        _ptr(plan["num_tokens_post_padded"]), _ptr(h), _ptr(err_flag), _stream()), "moe_grouped_up_swiglu_routed")
    return h, plan


def grouped_down(h, w_down, plan, shape: Shape, y=None, err_flag=None):
    """y[M*K, H] = bf16(h W_down^T), scattered to slot order."""
    _need_cuda(h, w_down)
    if y is None:
        y = torch.empty(shape.M * shape.top_k, shape.H, dtype=torch.bfloat16, device=h.device)
    w = _weights_struct(w_down, w_down, w_down)
    p = _plan_struct(plan)
    _check(library().moe_grouped_down(_ptr(_bf16(h)), ctypes.byref(w), ctypes.byref(p), shape.c(), _ptr(y), None, 0,
                                      _ptr(err_flag), _stream()), "moe_grouped_down")
    return y


def finalize_rmsnorm(x, y, topk_w, gamma, eps, out=None, residual_out=None, want_residual=False):
    """out = RMSNorm(x + sum_k w_k y_k) * gamma (and bf16(x + sum) if asked)."""
    _need_cuda(x, y, topk_w, gamma)
    M, H = x.shape
    K = topk_w.shape[1]
    shape = Shape(M, H, 128, max(K, 1), K, 16)
    if out is None:
        out = torch.empty_like(x)
    if want_residual and residual_out is None:
        residual_out = torch.empty_like(x)
    _check(library().moe_finalize_rmsnorm(_ptr(_bf16(x)), _ptr(_bf16(y)), _ptr(topk_w), _ptr(_bf16(gamma)),
                                          float(eps), shape.c(), _ptr(out), _ptr(residual_out), _stream()),
           "moe_finalize_rmsnorm")
    return (out, residual_out) if want_residual else out


def layer(x, w_router, bias, w_gate, w_up, w_down, gamma, eps, top_k, block_size, ws=None, out=None,
          residual_out=None, topk_ids=None, topk_w=None):
    """The whole routed-MoE layer; returns out [M,H] bf16."""
    _need_cuda(x, w_router, w_gate, w_up, w_down, gamma)
    M, H = x.shape
    E, I = w_gate.shape[0], w_gate.shape[1]
    shape = Shape(M, H, I, E, top_k, block_size)
    if ws is None:
        ws = torch.empty(layer_workspace_size(shape), dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty_like(x)
    w = _weights_struct(w_gate, w_up, w_down)
    _check(library().moe_layer(_ptr(_bf16(x)), _ptr(_bf16(w_router)), _ptr(bias), ctypes.byref(w),
                               _ptr(_bf16(gamma)), float(eps), shape.c(), _ptr(out), _ptr(residual_out),
                               _ptr(topk_ids), _ptr(topk_w), _ptr(ws), ws.numel(), _stream()), "moe_layer")
    return out


# ------------------------------------------------------------------ NVFP4
@dataclass
class NVFP4Weights:
    """Prepared NVFP4 expert weights: one blob (uint8) per projection and the
    per-expert fp32 global scales."""
    gate: torch.Tensor
    up: torch.Tensor
    down: torch.Tensor
    gate_gs: torch.Tensor
    up_gs: torch.Tensor
    down_gs: torch.Tensor

    def c(self) -> _Weights:
        return _Weights(MOE_W_NVFP4, self.gate.data_ptr(), self.up.data_ptr(), self.down.data_ptr(),
                        self.gate_gs.data_ptr(), self.up_gs.data_ptr(), self.down_gs.data_ptr())


def quantize_nvfp4(w):
    """w bf16 [n_mats, rows, cols] -> (codes uint8 [n,rows,cols/2], scales uint8 [n,rows,cols/16], gs fp32 [n])."""
    _need_cuda(w)
    n, rows, cols = w.shape
    codes = torch.empty(n, rows, cols // 2, dtype=torch.uint8, device=w.device)
    scales = torch.empty(n, rows, cols // 16, dtype=torch.uint8, device=w.device)
    gs = torch.empty(n, dtype=torch.float32, device=w.device)
    ws = torch.empty(int(library().moe_nvfp4_quantize_workspace_size(n)), dtype=torch.uint8, device=w.device)
    _check(library().moe_quantize_nvfp4(_ptr(_bf16(w)), n, rows, cols, _ptr(codes), _ptr(scales), _ptr(gs), _ptr(ws),
                                        ws.numel(), _stream()), "moe_quantize_nvfp4")
    return codes, scales, gs


def nvfp4_blob_bytes(shape: Shape, which: int) -> int:
    return int(library().moe_nvfp4_blob_bytes(shape.c(), which))


def prepare_nvfp4_weights(codes, scales, shape: Shape, which: int):
    blob = torch.empty(nvfp4_blob_bytes(shape, which), dtype=torch.uint8, device=codes.device)
    _check(library().moe_prepare_nvfp4_weights(_ptr(codes), _ptr(scales), shape.c(), which, _ptr(blob), blob.numel(),
                                               _stream()), "moe_prepare_nvfp4_weights")
    return blob


def nvfp4_weights(w_gate, w_up, w_down, shape: Shape) -> NVFP4Weights:
    """Quantise bf16 expert weights and prepare the blobs the NVFP4 kernels read."""
    blobs, gss = [], []
    for which, w in enumerate((w_gate, w_up, w_down)):
        codes, scales, gs = quantize_nvfp4(w)
        blobs.append(prepare_nvfp4_weights(codes, scales, shape, which))
        gss.append(gs)
        del codes, scales
    return NVFP4Weights(blobs[0], blobs[1], blobs[2], gss[0], gss[1], gss[2])


def down_workspace_size(shape: Shape, wdtype: int = MOE_W_BF16) -> int:
    return int(library().moe_down_workspace_size(shape.c(), wdtype))


def grouped_up_swiglu_nvfp4(x, nw: NVFP4Weights, plan, shape: Shape, h=None, err_flag=None, ws=None):
    """NVFP4 form of grouped_up_swiglu (x quantised on the fly into ws)."""
    _need_cuda(x)
    if h is None:
        h = torch.empty(align_capacity(shape), shape.I, dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = torch.empty(up_workspace_size(shape, MOE_W_NVFP4), dtype=torch.uint8, device=x.device)
    w = nw.c()
    p = _plan_struct(plan)
    _check(library().moe_grouped_up_swiglu(_ptr(_bf16(x)), ctypes.byref(w), ctypes.byref(p), shape.c(), _ptr(h),
                                           _ptr(ws), ws.numel(), _ptr(err_flag), _stream()), "moe_grouped_up_swiglu")
    return h


def grouped_down_nvfp4(h, nw: NVFP4Weights, plan, shape: Shape, y=None, err_flag=None, ws=None):
    """NVFP4 form of grouped_down (h quantised on the fly into ws)."""
    _need_cuda(h)
    if y is None:
        y = torch.empty(shape.M * shape.top_k, shape.H, dtype=torch.bfloat16, device=h.device)
    if ws is None:
        ws = torch.empty(down_workspace_size(shape, MOE_W_NVFP4), dtype=torch.uint8, device=h.device)
    w = nw.c()
    p = _plan_struct(plan)
    _check(library().moe_grouped_down(_ptr(_bf16(h)), ctypes.byref(w), ctypes.byref(p), shape.c(), _ptr(y), _ptr(ws),
                                      ws.numel(), _ptr(err_flag), _stream()), "moe_grouped_down")
    return y


def layer_nvfp4(x, w_router, bias, nw: NVFP4Weights, gamma, eps, top_k, block_size, I, ws=None, out=None,
                residual_out=None, topk_ids=None, topk_w=None):
    """The whole layer with NVFP4 expert weights; returns out [M,H] bf16."""
    _need_cuda(x, w_router, gamma)
    M, H = x.shape
    E = w_router.shape[0]
    shape = Shape(M, H, I, E, top_k, block_size)
    if ws is None:
        ws = torch.empty(layer_workspace_size(shape, MOE_W_NVFP4), dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty_like(x)
    w = nw.c()
    _check(library().moe_layer(_ptr(_bf16(x)), _ptr(_bf16(w_router)), _ptr(bias), ctypes.byref(w),
                               _ptr(_bf16(gamma)), float(eps), shape.c(), _ptr(out), _ptr(residual_out),
                               _ptr(topk_ids), _ptr(topk_w), _ptr(ws), ws.numel(), _stream()), "moe_layer")
    return out


def selftest_wait_timeout(err_flag, limit_us: int = 1000):
    """Run the kernel whose bounded wait always expires (see moe_selftest_wait_timeout)."""
    _check(library().moe_selftest_wait_timeout(_ptr(err_flag), int(limit_us), _stream()), "moe_selftest_wait_timeout")


def measure_hbm_read(buf, sink):
    """Enqueue one streaming read of the whole tensor ``buf`` (the HBM read-ceiling kernel of
    moe_measure_hbm_read); ``sink`` is a device int32/uint32 word."""
    _need_cuda(buf, sink)
    _check(library().moe_measure_hbm_read(_ptr(buf), buf.numel() * buf.element_size(), _ptr(sink), _stream()),
           "moe_measure_hbm_read")


def measure_tma_stream(buf, boxes: int, stages: int, contiguous: bool, steps: int, err_flag=None,
                       warps: int = 1) -> int:
    """Enqueue one TMA weight-panel stream over the tensor ``buf`` (moe_measure_tma_stream: ``boxes``
    16 KB boxes per stage, ``stages`` stages in flight, 2-D tensor boxes or ``contiguous`` bulk copies,
    ``warps`` issuing threads per CTA, ``steps`` stages per CTA); returns the bytes the call copies into
    shared memory."""
    _need_cuda(buf)
    moved = ctypes.c_size_t(0)
    _check(library().moe_measure_tma_stream(_ptr(buf), buf.numel() * buf.element_size(), int(boxes), int(stages),
                                            1 if contiguous else 0, int(warps), int(steps),
                                            _ptr(err_flag) if err_flag is not None else None,
                                            ctypes.byref(moved), _stream()), "moe_measure_tma_stream")
    return int(moved.value)


def measure_tma_mix(buf, mix: int, stages: int, steps: int, err_flag=None) -> int:
    """Enqueue one stream of the NVFP4 GEMMs' stage copy mix ``mix`` over the tensor ``buf``
    (moe_measure_tma_mix: ``stages`` slots in flight, ``steps`` k-steps per CTA); returns the bytes the call
    copies into shared memory."""
    _need_cuda(buf)
    moved = ctypes.c_size_t(0)
    _check(library().moe_measure_tma_mix(_ptr(buf), buf.numel() * buf.element_size(), int(mix), int(stages),
                                         int(steps), _ptr(err_flag) if err_flag is not None else None,
                                         ctypes.byref(moved), _stream()), "moe_measure_tma_mix")
    return int(moved.value)


def get_device_error(err_flag) -> int:
    """Synchronise the current stream and return the device-detected status (0 = none)."""
    code = ctypes.c_int32(0)
    _check(library().moe_get_device_error(_ptr(err_flag), _stream(), ctypes.byref(code)), "moe_get_device_error")
    return int(code.value)
