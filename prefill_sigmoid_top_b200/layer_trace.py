"""Phase timeline of the single-launch layer (decode shapes): a measurement tool, not part of the layer.

Runs ``moe_layer`` on one workload through the timeline build of the library
(``python -m prefill_sigmoid_top_b200.build --trace`` -> libmoe_b200_trace.so, compiled with
-DMOE_LAYER_TRACE, which stamps the global timer at fixed points of every CTA) and prints when, from the
first CTA's start, the CTAs passed the grid barrier after the router logits, finished the top-k and plan,
claimed their first down tile, published their last up and down tiles and ran the finalize; how long the
producers waited for an expert's h rows and for a free ring slot; and the rate of the projection phase.
The stamps cost a few global stores per tile.

  python -m prefill_sigmoid_top_b200.layer_trace [--config 1] [--json out.json]

Must start in a fresh process: it points the package at the timeline library before loading it.
"""
from __future__ import annotations

import argparse
import ctypes
import json

import numpy as np

SLOTS = 16
CTAS = 1024
START, BARRIER, PLAN, FIRST_DOWN, LAST_UP_PUB, LAST_DOWN_PUB, FIN_START, FIN_END, WAIT_ROWS, WAIT_SLOT, \
    UP_TILES, DOWN_TILES, END = range(13)


def trace_workload(cid: int):
    import torch

    import prefill_sigmoid_top_b200 as moe
    from prefill_sigmoid_top_b200 import build, inputs

    if moe._lib is not None:
        raise RuntimeError("layer_trace must run before the package loads its library (use a fresh process)")
    moe._LIB_PATH = build.build(trace=True)
    L = moe.library()
    L.moe_layer_trace_read.argtypes = [ctypes.c_void_p, ctypes.c_size_t]
    cfg = inputs.WORKLOADS[cid]
    d = inputs.make_inputs(cfg, "cuda")
    shape = moe.Shape(cfg.M, cfg.H, cfg.I, cfg.E, cfg.K, cfg.B)
    if moe.layer_kernel_count(shape) != 1:
        raise RuntimeError(f"{cfg.name}: moe_layer is not a single launch at this shape")
    ws = torch.empty(moe.layer_workspace_size(shape), dtype=torch.uint8, device="cuda")
    out = torch.empty(cfg.M, cfg.H, dtype=torch.bfloat16, device="cuda")

    def call():
        moe.layer(d["x"], d["w_router"], d["bias"], d["w_gate"], d["w_up"], d["w_down"], d["gamma"], cfg.eps,
                  top_k=cfg.K, block_size=cfg.B, out=out, ws=ws)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    if L.moe_layer_trace_clear() != 0:
        raise RuntimeError("moe_layer_trace_clear failed")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    call()
    e1.record()
    torch.cuda.synchronize()
    buf = np.zeros((CTAS, SLOTS), np.uint64)
    if L.moe_layer_trace_read(buf.ctypes.data, buf.nbytes) != 0:
        raise RuntimeError("moe_layer_trace_read failed")
    ids, _ = moe.route(d["x"], d["w_router"], d["bias"], cfg.K)
    touched = int(torch.unique(ids).numel())
    weight_bytes = touched * 3 * cfg.I * cfg.H * 2
    return cfg, buf, e0.elapsed_time(e1) * 1e3, weight_bytes


def analyze(buf, weight_bytes: float | None = None) -> dict:
    """Phase times (µs from the first CTA's start) over the CTAs that ran, waits per CTA, tile counts."""
    t = buf.astype(np.int64)
    t = t[t[:, START] > 0]
    if len(t) == 0:
        return {}
    t0 = t[:, START].min()

    def rel(col, mask=None):
        v = t[:, col] if mask is None else t[mask, col]
        v = v[v > 0]
        return (v - t0) / 1e3

    def span(col):
        v = rel(col)
        return None if len(v) == 0 else {"min": float(v.min()), "median": float(np.median(v)), "max": float(v.max())}

    out = {"ctas": int(len(t))}
    for name, col in (("barrier", BARRIER), ("plan", PLAN), ("first_down_claimed", FIRST_DOWN),
                      ("last_up_published", LAST_UP_PUB), ("last_down_published", LAST_DOWN_PUB),
                      ("finalize_start", FIN_START), ("finalize_end", FIN_END), ("end", END)):
        out[name] = span(col)
    out["wait_rows_us_per_cta"] = float(t[:, WAIT_ROWS].mean() / 1e3)
    out["wait_slot_us_per_cta"] = float(t[:, WAIT_SLOT].mean() / 1e3)
    out["up_tiles"] = int(t[:, UP_TILES].sum())
    out["down_tiles"] = int(t[:, DOWN_TILES].sum())
    if weight_bytes and out["plan"] and out["last_down_published"]:
        dur = out["last_down_published"]["max"] - out["plan"]["median"]
        out["projection_us"] = dur
        out["projection_TBps"] = weight_bytes / (dur * 1e-6) / 1e12
    return out


def main(argv=None):
    p = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    p.add_argument("--config", type=int, default=1)
    p.add_argument("--json", default=None)
    a = p.parse_args(argv)
    cfg, buf, ev_us, weight_bytes = trace_workload(a.config)
    res = analyze(buf, weight_bytes)
    res.update(workload=cfg.name, events_us=ev_us, weight_bytes=weight_bytes)
    for k in ("barrier", "plan", "first_down_claimed", "last_up_published", "last_down_published",
              "finalize_start", "finalize_end", "end"):
        v = res.get(k)
        if v:
            print(f"{k:>22}: {v['min']:9.1f} {v['median']:9.1f} {v['max']:9.1f} us (min / median / max over CTAs)")
    print(f"producer waits per CTA: h rows {res['wait_rows_us_per_cta']:.1f} us, ring slot "
          f"{res['wait_slot_us_per_cta']:.1f} us; tiles up {res['up_tiles']}, down {res['down_tiles']}; "
          f"launch {ev_us:.1f} us (events)")
    if "projection_TBps" in res:
        print(f"projection phase (plan done -> last down tile published): {res['projection_us']:.1f} us, "
              f"{weight_bytes / 1e9:.2f} GB of weights, {res['projection_TBps']:.2f} TB/s")
    if a.json:
        with open(a.json, "w") as f:
            json.dump(res, f, indent=1)


if __name__ == "__main__":
    main()
