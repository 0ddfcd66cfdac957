"""Tensor-parallel form of the layer (include/moe_b200_tp.h): the expert intermediate dimension split over
the G GPUs of one node, the finalize fused with the reduction across them and the RMSNorm.

Argument marshalling and host plumbing only: the weight slices (views of the caller's tensors made
contiguous), the group buffer and the exchange of its IPC handle over ``torch.distributed`` (any backend:
the handles are host bytes).  Every step of the layer runs in the library's CUDA kernels.
"""
from __future__ import annotations

import ctypes

import torch

from . import MoEError, Shape, _Shape, _Weights, _bf16, _check, _need_cuda, _ptr, _stream, library

MAX_RANKS = 8
HANDLE_BYTES = 72


class _TPGroup(ctypes.Structure):
    _fields_ = [("rank", ctypes.c_int32), ("world", ctypes.c_int32), ("max_tokens", ctypes.c_int32),
                ("hidden", ctypes.c_int32), ("bufs", ctypes.c_void_p * MAX_RANKS)]


_declared = False


def _lib():
    global _declared
    L = library()
    if not _declared:
        vp, sz, st, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_int32
        pp = ctypes.POINTER(ctypes.c_void_p)
        sig = {
            "moe_tp_buffer_bytes": (sz, [i32, i32, i32]),
            "moe_tp_protocol": (ctypes.c_int, [i32, i32, i32]),
            "moe_tp_finalize_allreduce_rmsnorm": (st, [vp, vp, vp, vp, ctypes.c_float, _Shape,
                                                       ctypes.POINTER(_TPGroup), vp, vp, vp, vp]),
            "moe_tp_layer": (st, [vp, vp, vp, ctypes.POINTER(_Weights), vp, ctypes.c_float, _Shape,
                                  ctypes.POINTER(_TPGroup), vp, vp, vp, vp, vp, sz, vp]),
            "moe_tp_layer_workspace_size": (sz, [_Shape]),
            "moe_tp_finalize_emulated": (st, [vp, pp, vp, vp, ctypes.c_float, _Shape, i32, i32, pp, pp, pp, vp,
                                              vp]),
            "moe_tp_ipc_handle": (st, [vp, vp]),
            "moe_tp_ipc_open": (st, [vp, pp]),
            "moe_tp_ipc_close": (st, [vp]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _declared = True
    return L


def buffer_bytes(world: int, max_tokens: int, hidden: int) -> int:
    return int(_lib().moe_tp_buffer_bytes(world, max_tokens, hidden))


def protocol(M: int, world: int, max_tokens: int) -> str:
    """'oneshot' or 'twoshot': the exchange a call with M tokens takes."""
    return {0: "oneshot", 1: "twoshot"}[int(_lib().moe_tp_protocol(M, world, max_tokens))]


def shard_weights(w_gate, w_up, w_down, rank: int, world: int):
    """Rank `rank`'s slice of the expert weights: rows [r*I/G, (r+1)*I/G) of W_gate[e] and W_up[e]
    ([E, I, H]) and the same columns of W_down[e] ([E, H, I]), each made contiguous."""
    E, I, H = w_gate.shape
    if world < 1 or I % world != 0:
        raise ValueError(f"I={I} does not split over {world} ranks")
    Ir = I // world
    sl = slice(rank * Ir, (rank + 1) * Ir)
    return w_gate[:, sl, :].contiguous(), w_up[:, sl, :].contiguous(), w_down[:, :, sl].contiguous()


def exchange_handles(handle: bytes, group=None) -> list:
    """Every rank's IPC handle, in rank order (an all-gather of host bytes over torch.distributed)."""
    import torch.distributed as dist
    out = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, bytes(handle), group=group)
    return out


def ipc_handle(buf: torch.Tensor) -> bytes:
    h = ctypes.create_string_buffer(HANDLE_BYTES)
    _check(_lib().moe_tp_ipc_handle(_ptr(buf), h), "moe_tp_ipc_handle")
    return h.raw


def ipc_open(handle: bytes) -> int:
    p = ctypes.c_void_p()
    _check(_lib().moe_tp_ipc_open(ctypes.create_string_buffer(bytes(handle), HANDLE_BYTES), ctypes.byref(p)),
           "moe_tp_ipc_open")
    return int(p.value)


class TPGroup:
    """One rank's group buffer, zeroed, and the peers' buffers mapped into this process.

    world == 1 needs no buffer.  For world > 1 every rank must construct its TPGroup collectively (the
    handles are exchanged with ``exchange_handles`` over ``group``) with the same max_tokens and hidden."""

    def __init__(self, rank: int, world: int, max_tokens: int, hidden: int, device=None, group=None):
        if not 1 <= world <= MAX_RANKS or not 0 <= rank < world:
            raise ValueError("rank / world outside the supported range")
        self.rank, self.world, self.max_tokens, self.hidden = rank, world, max_tokens, hidden
        self.buf = None
        self._opened = []
        ptrs = [None] * MAX_RANKS
        if world > 1:
            nbytes = buffer_bytes(world, max_tokens, hidden)
            if nbytes == 0:
                raise MoEError(2, "moe_tp_buffer_bytes")
            self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=device)
            torch.cuda.synchronize(self.buf.device)
            handles = exchange_handles(ipc_handle(self.buf), group)
            for r, h in enumerate(handles):
                if r == rank:
                    ptrs[r] = self.buf.data_ptr()
                else:
                    ptrs[r] = ipc_open(h)
                    self._opened.append(ptrs[r])
        self._c = _TPGroup(rank, world, max_tokens, hidden, (ctypes.c_void_p * MAX_RANKS)(*ptrs))

    def c(self):
        return self._c

    def close(self):
        for p in self._opened:
            _lib().moe_tp_ipc_close(ctypes.c_void_p(p))
        self._opened = []


def layer_workspace_size_tp(shape: Shape) -> int:
    return int(_lib().moe_tp_layer_workspace_size(shape.c()))


def tp_layer(x, w_router, bias, gate_r, up_r, down_r, gamma, eps, top_k, block_size, group: TPGroup, ws=None,
             out=None, residual_out=None, topk_ids=None, topk_w=None):
    """This rank's call of the tensor-parallel layer (gate_r/up_r [E, I/G, H], down_r [E, H, I/G]);
    returns out [M,H] bf16, the same bits on every rank."""
    _need_cuda(x, w_router, gate_r, up_r, down_r, gamma)
    M, H = x.shape
    E, Ir = gate_r.shape[0], gate_r.shape[1]
    shape = Shape(M, H, Ir, E, top_k, block_size)
    if ws is None:
        ws = torch.empty(layer_workspace_size_tp(shape), dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty_like(x)
    w = _Weights(0, gate_r.data_ptr(), up_r.data_ptr(), down_r.data_ptr(), None, None, None)
    _check(_lib().moe_tp_layer(_ptr(_bf16(x)), _ptr(_bf16(w_router)), _ptr(bias), ctypes.byref(w), _ptr(_bf16(gamma)),
                               float(eps), shape.c(), ctypes.byref(group.c()), _ptr(out), _ptr(residual_out),
                               _ptr(topk_ids), _ptr(topk_w), _ptr(ws), ws.numel(), _stream()), "moe_tp_layer")
    return out


def tp_finalize(x, y_partial, topk_w, gamma, eps, group: TPGroup, out=None, residual_out=None, err_flag=None):
    """The fused finalize on this rank: y_partial [M*K, H] (or [M,K,H]) this rank's partial rows."""
    _need_cuda(x, y_partial, topk_w, gamma)
    M, H = x.shape
    K = topk_w.shape[1]
    shape = Shape(M, H, 128, max(K, 1), K, 16)
    if out is None:
        out = torch.empty_like(x)
    _check(_lib().moe_tp_finalize_allreduce_rmsnorm(_ptr(_bf16(x)), _ptr(_bf16(y_partial)), _ptr(topk_w),
                                                    _ptr(_bf16(gamma)), float(eps), shape.c(), ctypes.byref(group.c()),
                                                    _ptr(out), _ptr(residual_out), _ptr(err_flag), _stream()),
           "moe_tp_finalize_allreduce_rmsnorm")
    return out


def _ptr_array(ts):
    return (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])


def tp_finalize_emulated(x, y_partials, topk_w, gamma, eps, max_tokens, bufs, outs, residual_outs=None,
                         err_flag=None):
    """All G ranks of a group in one cooperative launch on this GPU (see moe_tp_finalize_emulated):
    y_partials, bufs, outs (and residual_outs) are lists of G device tensors."""
    G = len(y_partials)
    M, H = x.shape
    K = topk_w.shape[1]
    shape = Shape(M, H, 128, max(K, 1), K, 16)
    ys, bs, os_ = _ptr_array(y_partials), _ptr_array(bufs), _ptr_array(outs)
    rs = _ptr_array(residual_outs) if residual_outs is not None else None
    _check(_lib().moe_tp_finalize_emulated(_ptr(_bf16(x)), ys, _ptr(topk_w), _ptr(_bf16(gamma)), float(eps),
                                           shape.c(), G, max_tokens, bs, os_, rs, _ptr(err_flag), _stream()),
           "moe_tp_finalize_emulated")
