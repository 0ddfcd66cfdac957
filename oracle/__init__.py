"""CPU oracle for the routed-MoE layer -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``moe_oracle.cpp`` (plain
C++17, fp64, OpenMP) through ctypes and shares no code with the CUDA library
in ``prefill_sigmoid_top_b200``; neither imports the other.

Every function here is a thin numpy <-> C marshalling layer; the arithmetic
and the page citations are in ``moe_oracle.cpp``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

CXXFLAGS = ["-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/libmoe_oracle.so (g++, no BLAS)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", *CXXFLAGS, _SRC, "-o", tmp])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB_PATH)
            vp, i32, i64, f32, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double
            sig = {
                "oracle_bf16_value": (f64, [ctypes.c_uint16]),
                "oracle_bf16_round": (ctypes.c_uint16, [f64]),
                "oracle_e2m1_value": (f64, [ctypes.c_uint8]),
                "oracle_e4m3_value": (f64, [ctypes.c_uint8]),
                "oracle_e2m1_encode": (ctypes.c_uint8, [f32]),
                "oracle_e4m3_encode": (ctypes.c_uint8, [f32]),
                "oracle_router_logits": (None, [vp, vp, vp, i32, i32, i32, vp, vp]),
                "oracle_topk": (None, [vp, i32, i32, i32, vp, vp]),
                "oracle_topk_ex": (None, [vp, vp, i32, i32, i32, i32, i32, f64, vp, vp]),
                "oracle_align": (i32, [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp]),
                "oracle_expert": (None, [vp, vp, vp, vp, i32, i32, vp, vp]),
                "oracle_finalize": (None, [vp, vp, vp, vp, f64, i32, i32, i32, vp, vp, vp, vp]),
                "oracle_layer": (i32, [vp, vp, vp, vp, vp, vp, vp, f32, i32, i32, i32, i32, i32, vp, i32,
                                       vp, vp, vp, vp, vp, vp, vp, vp]),
                "oracle_dense_mixture": (None, [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp]),
                "oracle_nvfp4_global_scale": (f32, [f32]),
                "oracle_nvfp4_quantize": (None, [vp, i64, i64, f32, vp, vp]),
                "oracle_nvfp4_quantize_bf16": (f32, [vp, i64, i64, vp, vp]),
                "oracle_nvfp4_dequantize": (None, [vp, vp, i64, i64, f32, vp]),
                "oracle_layer_nvfp4": (i32, [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, f32,
                                             i32, i32, i32, i32, i32, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp]),
                "oracle_num_threads": (i32, []),
                "oracle_tp_partial": (i32, [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, i32, vp, vp,
                                            vp, vp]),
                "oracle_rmsnorm_rows": (None, [vp, vp, f64, i32, i32, vp, vp, vp]),
                "oracle_layer_tp": (i32, [vp, vp, vp, vp, vp, vp, vp, f32, i32, i32, i32, i32, i32, vp, i32, vp, vp,
                                          vp, vp, vp, vp, vp]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def _u16(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected raw bf16 bits as uint16, got {a.dtype}")
    return a


def _ptr_table(mats):
    """ctypes array of pointers from a list of numpy arrays (None -> null)."""
    arr = (ctypes.c_void_p * len(mats))()
    for i, m in enumerate(mats):
        arr[i] = m.ctypes.data if m is not None else None
    return arr


# ------------------------------------------------------------------ scalars
def bf16_value(bits: int) -> float:
    return lib().oracle_bf16_value(int(bits))


def bf16_round(v: float) -> int:
    return int(lib().oracle_bf16_round(float(v)))


def e2m1_value(code: int) -> float:
    return lib().oracle_e2m1_value(int(code))


def e4m3_value(code: int) -> float:
    return lib().oracle_e4m3_value(int(code))


def e2m1_encode(v: float) -> int:
    return int(lib().oracle_e2m1_encode(float(v)))


def e4m3_encode(v: float) -> int:
    return int(lib().oracle_e4m3_encode(float(v)))


def num_threads() -> int:
    return int(lib().oracle_num_threads())


# ------------------------------------------------------------------ router
def router_logits(x, w_router, bias=None, want_f64=False):
    """Canonical fp32 logits z32 [M,E] (and the exact fp64 sum if asked)."""
    x, w_router = _u16(x), _u16(w_router)
    M, H = x.shape
    E = w_router.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    z32 = np.empty((M, E), np.float32)
    z64 = np.empty((M, E), np.float64) if want_f64 else None
    lib().oracle_router_logits(_p(x), _p(w_router), _p(b), M, H, E, _p(z32), _p(z64))
    return (z32, z64) if want_f64 else z32


def topk(z32, K):
    z32 = np.ascontiguousarray(z32, dtype=np.float32)
    M, E = z32.shape
    ids = np.empty((M, K), np.int32)
    w = np.empty((M, K), np.float64)
    lib().oracle_topk(_p(z32), M, E, K, _p(ids), _p(w))
    return ids, w


def route(x, w_router, bias, K):
    return topk(router_logits(x, w_router, bias), K)


SCORING_SOFTMAX, SCORING_SIGMOID = 0, 1


def topk_ex(z32, K, scoring=SCORING_SIGMOID, renormalize=True, scale=1.0, sel_bias=None):
    """Selection on fp32(z32 + sel_bias) (sel_bias None -> on z32), as topk(); weights from the sigmoid
    or softmax score of z32, optionally renormalised over the K selected, times scale."""
    z32 = np.ascontiguousarray(z32, dtype=np.float32)
    M, E = z32.shape
    b = None if sel_bias is None else np.ascontiguousarray(sel_bias, dtype=np.float32)
    ids = np.empty((M, K), np.int32)
    w = np.empty((M, K), np.float64)
    lib().oracle_topk_ex(_p(z32), _p(b), M, E, K, int(scoring), int(bool(renormalize)), float(scale), _p(ids),
                         _p(w))
    return ids, w


def route_ex(x, w_router, bias, K, scoring=SCORING_SIGMOID, renormalize=True, scale=1.0, bias_in_score=True):
    """Routing variants.  bias_in_score: the bias is part of the logit (as route()); otherwise it only
    shifts the selection key and the score is taken from the logit without it."""
    if bias_in_score or bias is None:
        return topk_ex(router_logits(x, w_router, bias), K, scoring, renormalize, scale)
    return topk_ex(router_logits(x, w_router, None), K, scoring, renormalize, scale, sel_bias=bias)


# ------------------------------------------------------------------ align
def align(topk_ids, E, B):
    """Returns dict(status, sorted_ids, block_expert, counts, offsets, ntpp).

    Arrays are cut to their defined extent: sorted_ids[:ntpp], block_expert[:ntpp//B].
    """
    ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    M, K = ids.shape
    cap = M * K + E * (B - 1)
    sorted_ids = np.full(cap, -7, np.int32)
    block_expert = np.full(max(cap // B, 1), -7, np.int32)
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    ntpp = np.zeros(1, np.int32)
    st = lib().oracle_align(_p(ids), M, K, E, B, _p(sorted_ids), _p(block_expert), _p(counts), _p(offsets), _p(ntpp))
    n = int(ntpp[0])
    return dict(status=int(st), sorted_ids=sorted_ids[:n].copy(), block_expert=block_expert[: n // B].copy(),
                counts=counts, offsets=offsets, ntpp=n)


def capacity(M, K, E, B):
    return M * K + E * (B - 1)


# ------------------------------------------------------------------ experts
def expert(x_row, w_gate_e, w_up_e, w_down_e):
    """One slot: returns (h bf16 bits [I], y bf16 bits [H])."""
    x_row, wg, wu, wd = _u16(x_row), _u16(w_gate_e), _u16(w_up_e), _u16(w_down_e)
    I, H = wg.shape
    h = np.empty(I, np.uint16)
    y = np.empty(H, np.uint16)
    lib().oracle_expert(_p(x_row), _p(wg), _p(wu), _p(wd), H, I, _p(h), _p(y))
    return h, y


def finalize(x, y, w, gamma, eps, want_residual=True, want_f64=False):
    """x [M,H] bf16 bits, y [M,K,H] bf16 bits, w [M,K] float -> (out, residual) bf16 bits
    (and, if asked, the same two before their final bf16 rounding, as float64)."""
    x, y, gamma = _u16(x), _u16(y), _u16(gamma)
    w = np.ascontiguousarray(w, dtype=np.float64)
    M, K, H = y.shape
    out = np.empty((M, H), np.uint16)
    res = np.empty((M, H), np.uint16) if want_residual else None
    o64 = np.empty((M, H), np.float64) if want_f64 else None
    s64 = np.empty((M, H), np.float64) if want_f64 else None
    lib().oracle_finalize(_p(x), _p(y), _p(w), _p(gamma), float(eps), M, K, H, _p(out), _p(res), _p(o64), _p(s64))
    return (out, res, o64, s64) if want_f64 else (out, res)


def layer(x, w_router, bias, w_gate, w_up, w_down, gamma, eps, K, tokens=None, want_h=False):
    """Whole layer for the chosen tokens (default: all).

    w_gate / w_up / w_down are lists of length E of per-expert arrays (or None
    for experts the chosen tokens do not need).  Returns a dict with ids, w,
    y [n,K,H], out [n,H], residual [n,H] (bf16 bits) and h [n,K,I] if asked.
    """
    x, w_router, gamma = _u16(x), _u16(w_router), _u16(gamma)
    M, H = x.shape
    E = w_router.shape[0]
    wg = [None if a is None else _u16(a) for a in w_gate]
    wu = [None if a is None else _u16(a) for a in w_up]
    wd = [None if a is None else _u16(a) for a in w_down]
    I = next(a for a in wg if a is not None).shape[0]
    tok = np.arange(M, dtype=np.int32) if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    n = len(tok)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    ids = np.empty((n, K), np.int32)
    w = np.empty((n, K), np.float64)
    h = np.empty((n, K, I), np.uint16) if want_h else None
    y = np.empty((n, K, H), np.uint16)
    out = np.empty((n, H), np.uint16)
    res = np.empty((n, H), np.uint16)
    o64 = np.empty((n, H), np.float64)
    s64 = np.empty((n, H), np.float64)
    st = lib().oracle_layer(_p(x), _p(w_router), _p(b), _ptr_table(wg), _ptr_table(wu), _ptr_table(wd), _p(gamma),
                            float(eps), M, H, I, E, K, _p(tok), n, _p(ids), _p(w), _p(h), _p(y), _p(out), _p(res),
                            _p(o64), _p(s64))
    if st != 0:
        raise RuntimeError(f"oracle_layer status {st}")
    return dict(ids=ids, w=w, h=h, y=y, out=out, residual=res, out_f64=o64, residual_f64=s64, tokens=tok)


def dense_mixture(x, w_gate, w_up, w_down, wdense):
    x = _u16(x)
    M, H = x.shape
    E = len(w_gate)
    I = w_gate[0].shape[0]
    wdense = np.ascontiguousarray(wdense, dtype=np.float64)
    mix = np.empty((M, H), np.float64)
    lib().oracle_dense_mixture(_p(x), _ptr_table([_u16(a) for a in w_gate]), _ptr_table([_u16(a) for a in w_up]),
                               _ptr_table([_u16(a) for a in w_down]), _p(wdense), M, H, I, E, _p(mix))
    return mix


# ------------------------------------------------------------------ NVFP4
def nvfp4_global_scale(amax: float) -> float:
    return float(lib().oracle_nvfp4_global_scale(float(amax)))


def nvfp4_quantize(v, gs):
    """v float32 [rows, cols] -> (codes uint8 [rows, cols], scales uint8 [rows, cols//16])."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    rows, cols = v.shape
    codes = np.empty((rows, cols), np.uint8)
    scales = np.empty((rows, cols // 16), np.uint8)
    lib().oracle_nvfp4_quantize(_p(v), rows, cols, float(gs), _p(codes), _p(scales))
    return codes, scales


def nvfp4_quantize_bf16(w):
    """bf16 bits [rows, cols] -> (codes, scales, gs) with the per-matrix global scale."""
    w = _u16(w)
    rows, cols = w.shape
    codes = np.empty((rows, cols), np.uint8)
    scales = np.empty((rows, cols // 16), np.uint8)
    gs = lib().oracle_nvfp4_quantize_bf16(_p(w), rows, cols, _p(codes), _p(scales))
    return codes, scales, float(gs)


def nvfp4_dequantize(codes, scales, gs):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, cols = codes.shape
    out = np.empty((rows, cols), np.float64)
    lib().oracle_nvfp4_dequantize(_p(codes), _p(scales), rows, cols, float(gs), _p(out))
    return out


def layer_nvfp4(x, w_router, bias, gate_q, up_q, down_q, gamma, eps, K, tokens=None):
    """NVFP4 layer.  gate_q/up_q/down_q: lists (length E) of (codes, scales, gs) or None.

    Returns dict(ids_all, w_all, h_all [M*K, I], y [n,K,H], out, residual).
    """
    x, w_router, gamma = _u16(x), _u16(w_router), _u16(gamma)
    M, H = x.shape
    E = w_router.shape[0]
    I = next(q for q in gate_q if q is not None)[0].shape[0]
    tok = np.arange(M, dtype=np.int32) if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    n = len(tok)

    def tables(qs):
        codes = _ptr_table([None if q is None else q[0] for q in qs])
        scales = _ptr_table([None if q is None else q[1] for q in qs])
        gs = np.array([0.0 if q is None else q[2] for q in qs], np.float32)
        return codes, scales, gs

    gc, gsc, ggs = tables(gate_q)
    uc, usc, ugs = tables(up_q)
    dc, dsc, dgs = tables(down_q)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    ids = np.empty((M, K), np.int32)
    w = np.empty((M, K), np.float64)
    h = np.empty((M * K, I), np.uint16)
    y = np.empty((n, K, H), np.uint16)
    out = np.empty((n, H), np.uint16)
    res = np.empty((n, H), np.uint16)
    o64 = np.empty((n, H), np.float64)
    s64 = np.empty((n, H), np.float64)
    st = lib().oracle_layer_nvfp4(_p(x), _p(w_router), _p(b), gc, gsc, _p(ggs), uc, usc, _p(ugs), dc, dsc, _p(dgs),
                                  _p(gamma), float(eps), M, H, I, E, K, _p(tok), n, _p(ids), _p(w), _p(h), _p(y),
                                  _p(out), _p(res), _p(o64), _p(s64))
    if st != 0:
        raise RuntimeError(f"oracle_layer_nvfp4 status {st}")
    return dict(ids_all=ids, w_all=w, h_all=h, y=y, out=out, residual=res, out_f64=o64, residual_f64=s64,
                tokens=tok)


# ------------------------------------------------------------------ tensor parallel
def _tp_common(x, w_router, gamma, w_gate, w_up, w_down, tokens):
    x, w_router = _u16(x), _u16(w_router)
    M, H = x.shape
    E = w_router.shape[0]
    wg = [None if a is None else _u16(a) for a in w_gate]
    wu = [None if a is None else _u16(a) for a in w_up]
    wd = [None if a is None else _u16(a) for a in w_down]
    I = next(a for a in wg if a is not None).shape[0]
    tok = np.arange(M, dtype=np.int32) if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    return x, w_router, wg, wu, wd, M, H, E, I, tok


def tp_partial(x, w_router, bias, w_gate, w_up, w_down, K, G, rank, tokens=None, want_y=False):
    """One rank's part of the tensor-parallel layer (I split over G ranks): returns dict(ids, w,
    p [n,H] fp64 = (rank 0: x) + sum_k w_k y_r[k], y [n,K,H] bf16 bits of the rank's partial rows if asked)."""
    x, w_router, wg, wu, wd, M, H, E, I, tok = _tp_common(x, w_router, None, w_gate, w_up, w_down, tokens)
    n = len(tok)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    ids = np.empty((n, K), np.int32)
    w = np.empty((n, K), np.float64)
    p = np.empty((n, H), np.float64)
    y = np.empty((n, K, H), np.uint16) if want_y else None
    st = lib().oracle_tp_partial(_p(x), _p(w_router), _p(b), _ptr_table(wg), _ptr_table(wu), _ptr_table(wd), H, I, E,
                                 K, G, rank, _p(tok), n, _p(ids), _p(w), _p(p), _p(y))
    if st != 0:
        raise RuntimeError(f"oracle_tp_partial status {st}")
    return dict(ids=ids, w=w, p=p, y=y, tokens=tok)


def rmsnorm_rows(s, gamma, eps):
    """s [n,H] fp64 -> (out bf16 bits, residual bf16 bits, out before rounding fp64)."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    n, H = s.shape
    out = np.empty((n, H), np.uint16)
    res = np.empty((n, H), np.uint16)
    o64 = np.empty((n, H), np.float64)
    lib().oracle_rmsnorm_rows(_p(s), _p(_u16(gamma)), float(eps), n, H, _p(out), _p(res), _p(o64))
    return out, res, o64


def layer_tp(x, w_router, bias, w_gate, w_up, w_down, gamma, eps, K, G, tokens=None, want_y_parts=False):
    """The tensor-parallel layer on G ranks (every rank's part computed here): dict(ids, w, out, residual,
    out_f64, residual_f64, y_parts [G,n,K,H] bf16 bits if asked)."""
    x, w_router, wg, wu, wd, M, H, E, I, tok = _tp_common(x, w_router, gamma, w_gate, w_up, w_down, tokens)
    gamma = _u16(gamma)
    n = len(tok)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    ids = np.empty((n, K), np.int32)
    w = np.empty((n, K), np.float64)
    yp = np.empty((G, n, K, H), np.uint16) if want_y_parts else None
    out = np.empty((n, H), np.uint16)
    res = np.empty((n, H), np.uint16)
    o64 = np.empty((n, H), np.float64)
    s64 = np.empty((n, H), np.float64)
    st = lib().oracle_layer_tp(_p(x), _p(w_router), _p(b), _ptr_table(wg), _ptr_table(wu), _ptr_table(wd), _p(gamma),
                               float(eps), H, I, E, K, G, _p(tok), n, _p(ids), _p(w), _p(yp), _p(out), _p(res), _p(o64),
                               _p(s64))
    if st != 0:
        raise RuntimeError(f"oracle_layer_tp status {st}")
    return dict(ids=ids, w=w, out=out, residual=res, out_f64=o64, residual_f64=s64, y_parts=yp, tokens=tok)

