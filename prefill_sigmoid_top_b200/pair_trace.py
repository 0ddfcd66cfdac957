"""Timeline of the 2-SM pair GEMMs (up and down) on one workload: a measurement tool, not part of the layer.

Runs the workload's grouped projections once through the timeline build of the library
(``python -m prefill_sigmoid_top_b200.build --trace`` -> libmoe_b200_trace.so, the kernels compiled with
-DMOE_PAIR_TRACE, which stamps the global timer at fixed points of every tile) and prints, per kernel:
the span, the mean mainloop and drain (epilogue) time by token-tile width N, the gaps between one tile's
last MMA and the next tile's first on each pair, and when the pairs finish.  The stamps cost a few
global stores per tile, so absolute times run ~1% above the plain build's.

  python -m prefill_sigmoid_top_b200.pair_trace [--config 3] [--json out.json]

Must start in a fresh process: it points the package at the timeline library before loading it.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import sys

import numpy as np


def trace_workload(cid: int):
    import torch

    import prefill_sigmoid_top_b200 as moe
    from prefill_sigmoid_top_b200 import build, inputs

    if moe._lib is not None:
        raise RuntimeError("pair_trace must run before the package loads its library (use a fresh process)")
    moe._LIB_PATH = build.build(trace=True)
    L = moe.library()
    L.moe_pair_trace_read.argtypes = [ctypes.c_void_p, ctypes.c_size_t]
    cfg = inputs.WORKLOADS[cid]
    d = inputs.make_inputs(cfg, "cuda")
    shape = moe.Shape(cfg.M, cfg.H, cfg.I, cfg.E, cfg.K, cfg.B)
    ids, _ = moe.route(d["x"], d["w_router"], d["bias"], cfg.K)
    plan = moe.align_block_size(ids, cfg.E, cfg.B)
    up_ws = torch.empty(moe.up_workspace_size(shape), dtype=torch.uint8, device="cuda")
    h = torch.empty(moe.align_capacity(shape), cfg.I, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(cfg.M * cfg.K, cfg.H, dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        moe.grouped_up_swiglu(d["x"], d["w_gate"], d["w_up"], plan, shape, h=h, ws=up_ws)
        moe.grouped_down(h, d["w_down"], plan, shape, y=y)
    torch.cuda.synchronize()
    if L.moe_pair_trace_clear() != 0:
        raise RuntimeError("moe_pair_trace_clear failed")
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record()
    moe.grouped_up_swiglu(d["x"], d["w_gate"], d["w_up"], plan, shape, h=h, ws=up_ws)
    ev[1].record()
    moe.grouped_down(h, d["w_down"], plan, shape, y=y)
    ev[2].record()
    torch.cuda.synchronize()
    buf = np.zeros((2, 8192, 8), np.uint64)
    if L.moe_pair_trace_read(buf.ctypes.data, buf.nbytes) != 0:
        raise RuntimeError("moe_pair_trace_read failed")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return cfg, buf, dict(up_us=ev[0].elapsed_time(ev[1]) * 1e3, down_us=ev[1].elapsed_time(ev[2]) * 1e3), sms // 2


def analyze(buf, npairs: int) -> dict:
    """Per kernel: span, mainloop and drain by N, gaps between tiles on a pair, pair end times (all in µs)."""
    out = {}
    for kind, name in ((0, "up"), (1, "down")):
        t = buf[kind].astype(np.int64)
        idx = np.nonzero(t[:, 1] > 0)[0]
        t = t[idx]
        if len(t) == 0:
            continue
        N = (t[:, 0] >> 28) & 0xFFF
        t0 = t[:, 1].min()
        start, mend, estart, erel = [(t[:, i] - t0) / 1e3 for i in (1, 3, 4, 5)]
        pair = idx % npairs  # the static round-robin: tile i runs on pair i % npairs
        main = mend - start
        drain = erel - estart
        gaps, busy, end = [], np.zeros(npairs), np.zeros(npairs)
        order = np.lexsort((start, pair))
        for a, b in zip(order[:-1], order[1:]):
            if pair[a] == pair[b]:
                gaps.append(start[b] - mend[a])
        for i in range(len(t)):
            busy[pair[i]] += main[i]
            end[pair[i]] = max(end[pair[i]], erel[i], mend[i])
        span = float(max(erel.max(), mend.max()))
        by_n = {int(v): {"tiles": int((N == v).sum()), "mainloop": float(main[N == v].mean()),
                         "drain": float(drain[N == v].mean())} for v in sorted(set(N.tolist()))}
        out[name] = {"tiles": int(len(t)), "span": span, "mainloop_mean": float(main.mean()),
                     "gap_mean": float(np.mean(gaps)) if gaps else 0.0,
                     "gap_per_pair": float(np.sum(gaps) / npairs) if gaps else 0.0,
                     "busy_frac": float(np.mean(busy / np.maximum(end, 1e-9))),
                     "pair_end": {"min": float(end.min()), "median": float(np.median(end)), "max": float(end.max())},
                     "by_N": by_n}
    return out


def main(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--config", type=int, default=3)
    p.add_argument("--json", default=None)
    a = p.parse_args(argv)
    cfg, buf, ev, npairs = trace_workload(a.config)
    res = {"workload": cfg.name, "events_us": ev, "pairs": npairs, "kernels": analyze(buf, npairs)}
    if a.json:
        with open(a.json, "w") as f:
            json.dump(res, f, indent=1)
    for name, k in res["kernels"].items():
        print(f"{cfg.name} {name}: {k['tiles']} tiles, span {k['span']:.0f} us (events {ev[name + '_us']:.0f} us), "
              f"mainloop {k['mainloop_mean']:.1f} us/tile, gap {k['gap_mean']:.2f} us/tile "
              f"({k['gap_per_pair']:.0f} us/pair), pairs end {k['pair_end']['min']:.0f}-{k['pair_end']['max']:.0f} us")
        print("   N: " + ", ".join(f"{n}: {v['mainloop']:.1f}/{v['drain']:.1f} ({v['tiles']})" for n, v in k["by_N"].items()))
    return res


if __name__ == "__main__":
    ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    main()
