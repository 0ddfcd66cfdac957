#!/usr/bin/env python3
"""Benchmark of the routed-MoE layer on B200 (one JSON line on rank 0).

The metric is the layer's µs and tokens/s at the decode, batch and prefill
token counts, as a fraction of the roofline that bounds each.  The default run
measures four workloads back to back (H=7168, I=2048, E=256, top_k=16):

  decode_m8           M=8,    block 16, seed 1   (the headline: ``value`` and the top-level keys)
  batch_m512          M=512,  block 64, seed 2
  prefill_m2048_zipf  M=2048, block 128, seed 3, Zipf-skewed expert popularity
  nvfp4_m1000         M=1000, block 16, seed 4, NVFP4 expert weights

and reports every one of them under ``workloads``.  One step = one pass of the
whole layer (route -> align -> up+SwiGLU -> down -> finalize+RMSNorm) through
``moe_layer``, inputs resident in HBM.  Each step streams GBs of expert weights,
far more than the 126 MB L2, so no L2 flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--workloads all|C,C,..]
                  [--impl ours|reference]

Multi-GPU: the layer is run as independent replicas, one per rank (no
collective on the data path); rank 0 prints the max-over-ranks time.
--impl reference times the CPU oracle (fp64 C++) on the host cores instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s (decode/batch/prefill routed-MoE layer, H=7168 I=2048 E=256 top_k=16)"
DEFAULT_WORKLOADS = (1, 2, 3, 4)

# ncu DRAM traffic of a workload's dominant kernel, per launch, from a capture
# on a smaller copy of the workload scaled to the full one.  Valid only while
# the kernel sources hash to the recorded value; otherwise "traffic" is null.
NCU_TRAFFIC = {
    # (workload, kernel): (DRAM bytes per launch, hash of the kernel's sources)
    # decode M=8, the single-launch layer, captured at full size, one pass (8.3777 GB read + 4.4 MB
    # written, 1.0013 x its 8.3715 GB of algorithmic bytes)
    (1, "layer_fused"): (8_382_036_224, "9c39ca834ce5fa81"),
    # batch M=512 and prefill M=2048: the up projection (2-SM pair kernel) captured at full size, one pass
    # (dram__bytes_read.sum + dram__bytes_write.sum of one launch)
    (2, "pair_up"): (15_296_836_864, "f133d19d41b4abbf"),
    (3, "pair_up"): (16_907_707_648, "f133d19d41b4abbf"),
    # NVFP4 M=1000: the block-scaled up projection captured at full size, one pass: on 2-SM pairs (the
    # default) and on single SMs (MOE_NVFP4_PAIR=0)
    (4, "nvfp4_pair_up"): (4_565_486_080, "c09c4a0689ec51c0"),
    (4, "nvfp4_up"): (4_656_227_584, "cc73a5d8c3d56c67"),
}
KERNEL_SOURCES = {
    "up": ["prefill_sigmoid_top_b200/csrc/gemm_bf16.cu", "prefill_sigmoid_top_b200/csrc/common.cuh"],
    "layer_fused": ["prefill_sigmoid_top_b200/csrc/layer_fused.cu", "prefill_sigmoid_top_b200/csrc/common.cuh",
                    "prefill_sigmoid_top_b200/csrc/router_dot.cuh"],
    "pair_up": ["prefill_sigmoid_top_b200/csrc/gemm_pair.cu", "prefill_sigmoid_top_b200/csrc/pair_ptx.cuh",
                "prefill_sigmoid_top_b200/csrc/common.cuh", "prefill_sigmoid_top_b200/csrc/tile_list.cuh"],
    "nvfp4_up": ["prefill_sigmoid_top_b200/csrc/nvfp4.cu", "prefill_sigmoid_top_b200/csrc/common.cuh",
                 "prefill_sigmoid_top_b200/csrc/tile_list.cuh"],
    "nvfp4_pair_up": ["prefill_sigmoid_top_b200/csrc/nvfp4_pair.cu", "prefill_sigmoid_top_b200/csrc/pair_ptx.cuh",
                      "prefill_sigmoid_top_b200/csrc/common.cuh", "prefill_sigmoid_top_b200/csrc/tile_list.cuh"],
}


def kernel_hash(kernel: str = "up") -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--config", type=int, default=1, help="the headline workload (value, top-level keys)")
    p.add_argument("--workloads", default="default",
                   help="workloads measured after the headline: 'default' (all four when the headline is the "
                        "decode workload and no size is overridden, else none), 'all', 'none' or a list like 2,3")
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="oracle time per workload's CPU baseline")
    p.add_argument("--experts", type=int, default=0,
                   help="override E (a smaller copy of the workload, e.g. for profiler captures)")
    p.add_argument("--tokens", type=int, default=0, help="override M (with --experts: a smaller copy)")
    p.add_argument("--topk", type=int, default=0, help="override top_k (with --experts)")
    p.add_argument("--tp-emulate", type=int, default=0,
                   help="time the tensor-parallel finalize with this many ranks emulated on one GPU (one cooperative "
                        "launch; partial rows are seeded random bf16 of the workload's shape)")
    p.add_argument("--route-only", action="store_true",
                   help="time moe_route alone on the workload's router inputs (no expert weights allocated; "
                        "a small target for profiler captures of the router kernels)")
    p.add_argument("--probe-tma", action="store_true",
                   help="time the TMA weight-panel stream of the grouped GEMMs without their MMAs "
                        "(moe_measure_tma_stream) from HBM and from L2, beside the plain streaming read")
    return p.parse_args(argv)


def workload(args, cid=None):
    from prefill_sigmoid_top_b200 import inputs
    cfg = inputs.WORKLOADS[args.config if cid is None else cid]
    if args.experts:
        cfg = cfg.with_(E=args.experts, name=f"{cfg.name}_E{args.experts}")
    if args.tokens:
        cfg = cfg.with_(M=args.tokens, name=f"{cfg.name}_M{args.tokens}")
    if args.topk:
        cfg = cfg.with_(K=args.topk, name=f"{cfg.name}_K{args.topk}")
    return cfg


def workload_list(args):
    """The workload ids one run measures, headline first."""
    overridden = bool(args.experts or args.tokens or args.topk)
    w = args.workloads
    if w == "default":
        rest = list(DEFAULT_WORKLOADS) if (args.config == 1 and not overridden) else []
    elif w == "all":
        rest = list(DEFAULT_WORKLOADS)
    elif w == "none":
        rest = []
    else:
        rest = [int(v) for v in w.split(",") if v.strip()]
    return [args.config] + [c for c in rest if c != args.config]


# ------------------------------------------------------------------ ranks
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))


def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a float over all ranks (identity at world size 1)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(per_rank_units: float, max_seconds: float, world: int) -> float:
    """Whole-job throughput: units processed by all ranks / slowest rank's time."""
    return per_rank_units * world / max_seconds


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons through NVML
    every 2 ms while the timed region runs (read-only queries)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device_index: int, period_s: float = 0.002):
        self.dev = torch_device_index
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self.error = None
        self._stop = threading.Event()
        self._ready = threading.Event()
        self._thread = None

    def _handle(self, nv):
        import torch
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            return nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.dev)

    def _run(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            while True:
                self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)), int(get_reasons(h))))
                self._ready.set()
                if self._stop.is_set():
                    break
                time.sleep(self.period)
            nv.nvmlShutdown()
        except Exception as e:  # no NVML: report no clock record rather than fail the bench
            self.error = repr(e)
        finally:
            self._ready.set()

    def __enter__(self):
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        self._ready.wait(timeout=5.0)  # the timed region starts once sampling has begun
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return None if self.error is None else {"error": self.error}
        reasons = set()
        for _, r in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ workload accounting
def algorithmic_bytes(cfg, touched: int, nvfp4: bool = False):
    """Bytes the layer must move at minimum: touched experts' weights, router weights, x in, out.
    NVFP4 weights take 0.5 byte per element plus one e4m3 scale per 16 elements."""
    wb = 0.5625 if nvfp4 else 2.0
    per_expert = 3 * cfg.I * cfg.H * wb
    return dict(layer=int(touched * per_expert + cfg.E * cfg.H * 2 + 2 * cfg.M * cfg.H * 2),
                up=int(touched * 2 * cfg.I * cfg.H * wb + cfg.M * cfg.H * 2),
                down=int(touched * cfg.I * cfg.H * wb),
                finalize=cfg.M * cfg.K * cfg.H * 2 + 2 * cfg.M * cfg.H * 2)


def layer_flops(cfg) -> float:
    """Dense-equivalent flops of the expert projections: 2 * (gate + up + down) * H * I per routed slot."""
    return 2.0 * 3 * cfg.H * cfg.I * cfg.M * cfg.K


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def tensor_peak(bf16_tflops: float, nvfp4: bool) -> float:
    """Dense tensor peak for the workload's MMA type: the measured bf16 peak, times the nominal
    fp4 / bf16 ratio (9 / 2.25 PFLOP/s) for NVFP4 weights and activations."""
    return bf16_tflops * (4.0 if nvfp4 else 1.0)


def layer_bound(cfg) -> str:
    """The roofline a workload is graded against: the tensor pipe for the compute-shaped prefill
    workload (its target is stated as a fraction of the dense bf16 tensor peak), HBM for the
    weight-streaming ones.  Both fractions are always reported."""
    return "tensor" if (cfg.wdtype == "bf16" and cfg.M * cfg.K / cfg.E >= 96) else "hbm"


def layer_roofline(cfg, touched, seconds, hbm_peak, tc_peak_bf16, read_ceiling=None):
    nvfp4 = cfg.wdtype == "nvfp4"
    ab = algorithmic_bytes(cfg, touched, nvfp4)["layer"]
    gbs = ab / seconds / 1e9
    tflops = layer_flops(cfg) / seconds / 1e12
    tpk = tensor_peak(tc_peak_bf16, nvfp4)
    r = {"algorithmic_bytes": ab, "GBps": gbs, "frac_hbm": gbs / hbm_peak, "hbm_peak_gbs": hbm_peak,
         "tflops": tflops, "frac_tensor": tflops / tpk, "tensor_peak_tflops": tpk,
         "tensor_dtype": "fp4 (measured bf16 x 4)" if nvfp4 else "bf16"}
    if read_ceiling:
        r["read_ceiling_gbs"] = read_ceiling
        r["frac_read_ceiling"] = gbs / read_ceiling
    bound = layer_bound(cfg)
    r["bound"] = bound
    r["frac"] = r["frac_tensor"] if bound == "tensor" else r["frac_hbm"]
    return r


# ------------------------------------------------------------------ our arm
def measure_read_ceiling(moe, torch, buf, reps=5):
    """Device-timed streaming read (moe_measure_hbm_read) of buf: the best GB/s of reps reads."""
    sink = torch.zeros(1, dtype=torch.int32, device=buf.device)
    for _ in range(2):
        moe.measure_hbm_read(buf, sink)
    torch.cuda.synchronize()
    best = 0.0
    stream = torch.cuda.current_stream()
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        moe.measure_hbm_read(buf, sink)
        e1.record(stream)
        torch.cuda.synchronize()
        best = max(best, buf.numel() * buf.element_size() / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    return best


def e2e_overlapped(torch, layer_step, x_src, out_shape, steps, warmup):
    """End-to-end device time of `steps` layer calls whose inputs come from pinned host memory and whose
    outputs go back to it, every step: x is copied in on one stream, the layer runs on the current stream,
    out is copied back on a third, with two buffers each, so step k+1's upload and step k-1's download run
    under step k's layer.  Returns (seconds, the last step's host output, bytes in, bytes out per step)."""
    comp = torch.cuda.current_stream()
    up_s, down_s = torch.cuda.Stream(), torch.cuda.Stream()
    x_host = x_src.cpu().pin_memory()
    x_dev = [torch.empty_like(x_src) for _ in range(2)]
    out_dev = [torch.empty(out_shape, dtype=torch.bfloat16, device=x_src.device) for _ in range(2)]
    out_host = [torch.empty(out_shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]

    def run(n):
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_done = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        up_s.wait_stream(comp)
        down_s.wait_stream(comp)
        t0.record(up_s)
        for k in range(n):
            b = k % 2
            with torch.cuda.stream(up_s):
                if k >= 2:
                    up_s.wait_event(ev_done[k - 2])   # layer k-2 has read x_dev[b]
                x_dev[b].copy_(x_host, non_blocking=True)
                ev_in[k].record(up_s)
            comp.wait_event(ev_in[k])
            if k >= 2:
                comp.wait_event(ev_out[k - 2])        # out_dev[b] has been read back
            layer_step(x_dev[b], out_dev[b])
            ev_done[k].record(comp)
            with torch.cuda.stream(down_s):
                down_s.wait_event(ev_done[k])
                out_host[b].copy_(out_dev[b], non_blocking=True)
                ev_out[k].record(down_s)
        t1.record(down_s)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) * 1e-3

    run(max(3, warmup))
    secs = run(steps)
    last = out_host[(steps - 1) % 2].clone()
    return secs, last, x_src.numel() * x_src.element_size(), last.numel() * last.element_size()


def measure_workload(cfg, args, dev, world, rank, want_cpu, read_ceiling_box):
    """Times one workload; returns its result dict (see the module docstring)."""
    import torch

    import prefill_sigmoid_top_b200 as moe
    from prefill_sigmoid_top_b200 import inputs

    nvfp4 = cfg.wdtype == "nvfp4"
    d = inputs.make_inputs(cfg, dev)
    shape = moe.Shape(cfg.M, cfg.H, cfg.I, cfg.E, cfg.K, cfg.B)
    stream = torch.cuda.current_stream()

    # the HBM read ceiling, measured once per run on the first workload's weights (8 GB of them)
    if read_ceiling_box.get("gbs") is None and d["w_gate"].numel() * 2 >= (4 << 30):
        flat = d["w_gate"].view(-1)
        read_ceiling_box["gbs"] = measure_read_ceiling(moe, torch, flat[: min(flat.numel(), 4 << 30)])
        read_ceiling_box["how"] = ("moe_measure_hbm_read: streaming 16-byte non-caching loads of 8 GB of this "
                                   "run's expert weights, 4 CTAs x 512 threads per SM, best of 5 (CUDA events)")

    # the oracle's inputs for the CPU baseline, taken before the bf16 weights can be dropped (NVFP4)
    cpu_inputs = None
    if want_cpu:
        cpu_inputs = oracle_sample_inputs(cfg, d, n=4 if nvfp4 else min(cfg.M, 8))

    nw = None
    if nvfp4:  # weight preparation (quantise + repack) happens once, before any timing
        nw = moe.nvfp4_weights(d["w_gate"], d["w_up"], d["w_down"], shape)
        torch.cuda.synchronize()
        del d["w_gate"], d["w_up"], d["w_down"]
        torch.cuda.empty_cache()

    # ---- staged pass: the separate entry points in turn, per-stage events
    route_ws = torch.empty(moe.route_workspace_size(shape), dtype=torch.uint8, device=dev)
    ids = torch.empty(cfg.M, cfg.K, dtype=torch.int32, device=dev)
    tw = torch.empty(cfg.M, cfg.K, dtype=torch.float32, device=dev)
    cap = moe.align_capacity(shape)
    plan = dict(sorted_ids=torch.empty(cap, dtype=torch.int32, device=dev),
                block_expert=torch.empty(cap // cfg.B + 1, dtype=torch.int32, device=dev),
                expert_counts=torch.empty(cfg.E, dtype=torch.int32, device=dev),
                expert_offsets=torch.empty(cfg.E + 1, dtype=torch.int32, device=dev),
                num_tokens_post_padded=torch.empty(1, dtype=torch.int32, device=dev))
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    wdt = moe.MOE_W_NVFP4 if nvfp4 else moe.MOE_W_BF16
    up_ws_bytes = moe.up_workspace_size(shape, wdt)
    up_ws = torch.empty(up_ws_bytes, dtype=torch.uint8, device=dev) if up_ws_bytes else None
    down_ws_bytes = moe.down_workspace_size(shape, wdt)
    down_ws = torch.empty(down_ws_bytes, dtype=torch.uint8, device=dev) if down_ws_bytes else None
    h = torch.empty(cap, cfg.I, dtype=torch.bfloat16, device=dev)
    y = torch.empty(cfg.M * cfg.K, cfg.H, dtype=torch.bfloat16, device=dev)
    out = torch.empty(cfg.M, cfg.H, dtype=torch.bfloat16, device=dev)
    stages = ["route", "align", "up", "down", "finalize"]

    def step(evs=None):
        def mark(i):
            if evs is not None:
                evs[i].record(stream)
        mark(0)
        moe.route(d["x"], d["w_router"], d["bias"], cfg.K, topk_ids=ids, topk_w=tw, ws=route_ws)
        mark(1)
        moe.align_block_size(ids, cfg.E, cfg.B, err_flag=err, out=plan)
        mark(2)
        if nvfp4:
            moe.grouped_up_swiglu_nvfp4(d["x"], nw, plan, shape, h=h, err_flag=err, ws=up_ws)
        else:
            moe.grouped_up_swiglu(d["x"], d["w_gate"], d["w_up"], plan, shape, h=h, err_flag=err, ws=up_ws)
        mark(3)
        if nvfp4:
            moe.grouped_down_nvfp4(h, nw, plan, shape, y=y, err_flag=err, ws=down_ws)
        else:
            moe.grouped_down(h, d["w_down"], plan, shape, y=y, err_flag=err)
        mark(4)
        moe.finalize_rmsnorm(d["x"], y, tw, d["gamma"], cfg.eps, out=out)
        mark(5)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if moe.get_device_error(err) != 0:
        raise SystemExit(f"device error during warm-up ({cfg.name})")
    touched = int((plan["expert_counts"] > 0).sum().item())

    # Workloads whose weights fit in L2 a few times over get L2 flushed (a 256 MB
    # write) before every timed step; the flush is outside the timed work.
    ab = algorithmic_bytes(cfg, touched, nvfp4)
    flush_l2 = ab["layer"] < 4 * 126_000_000
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush_l2 else None

    def flush():
        if flush_buf is not None:
            flush_buf.zero_()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    torch.cuda.synchronize()
    for k in range(args.steps):
        flush()
        step(evs[k])
    torch.cuda.synchronize()
    staged_ms = statistics.mean(e[0].elapsed_time(e[5]) for e in evs)
    out_staged = out.clone()  # the staged pass's result, compared with moe_layer's below
    stage_ms = {s: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs) for i, s in enumerate(stages)}
    del route_ws, up_ws, down_ws, h, y

    # ---- the timed layer: moe_layer (the public entry point, one call per step) on resident inputs
    ws = torch.empty(moe.layer_workspace_size(shape, wdt), dtype=torch.uint8, device=dev)
    out_layer = torch.empty_like(out)

    def layer_step(x_in, out_buf):
        if nvfp4:
            moe.layer_nvfp4(x_in, d["w_router"], d["bias"], nw, d["gamma"], cfg.eps, cfg.K, cfg.B, cfg.I, ws=ws,
                            out=out_buf)
        else:
            moe.layer(x_in, d["w_router"], d["bias"], d["w_gate"], d["w_up"], d["w_down"], d["gamma"], cfg.eps,
                      cfg.K, cfg.B, ws=ws, out=out_buf)

    for _ in range(max(3, args.warmup)):
        layer_step(d["x"], out_layer)
    torch.cuda.synchronize()

    def timed_loop(body):
        """Device time (ms) of args.steps calls of body(): one event pair around all of them, or, when L2 is
        flushed before every call, one pair per call (the flush outside) summed."""
        if not flush_l2:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                body()
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1)
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)]
        for a, b in pairs:
            flush()
            a.record(stream)
            body()
            b.record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in pairs)

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clocks:
        t_wall0 = time.perf_counter()
        total_ms = timed_loop(lambda: layer_step(d["x"], out_layer))
        t_wall = time.perf_counter() - t_wall0
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms_per_step = total_ms / args.steps
    max_s = reduce_max(total_ms / 1e3, world, dev)
    value = aggregate(cfg.M * args.steps, max_s, world)
    eo = moe.layer_workspace_layout(shape, wdt)["err_flag"]
    if moe.get_device_error(ws[eo:eo + 4].view(torch.int32)) != 0:
        raise SystemExit(f"device error in the timed layer calls ({cfg.name})")

    # ---- the same call replayed from a CUDA graph (launch work taken off the host)
    graph_ms = None
    if world == 1:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            layer_step(d["x"], out_layer)
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            layer_step(d["x"], out_layer)
        for _ in range(max(3, args.warmup)):
            graph.replay()
        torch.cuda.synchronize()
        graph_ms = timed_loop(graph.replay) / args.steps
        del graph

    # ---- end to end through the public entry point (moe_layer) with host buffers, copies overlapped
    if world > 1:
        torch.distributed.barrier()
    e2e_s, out_host, h2d_b, d2h_b = e2e_overlapped(torch, layer_step, d["x"], (cfg.M, cfg.H), args.steps,
                                                   args.warmup)
    e2e_s = reduce_max(e2e_s, world, dev)
    e2e_value = aggregate(cfg.M * args.steps, e2e_s, world)
    # the e2e output (host), the timed layer's output and the staged pass's output are the same bits
    same = bool(torch.equal(out_host, out_staged.cpu())) and bool(torch.equal(out_layer, out_staged))

    hbm_peak, tc_peak, peak_kind = peaks()
    up_s = stage_ms["up"] / 1e3
    up_achieved = ab["up"] / up_s / 1e9
    default_size = not (args.experts or args.tokens or args.topk)
    cid = next((k for k, v in inputs.WORKLOADS.items() if v.name == cfg.name), None)

    def ncu_traffic(kernel):
        tr = NCU_TRAFFIC.get((cid, kernel)) if default_size else None
        return tr[0] if tr is not None and tr[1] == kernel_hash(kernel) else None

    lroof = layer_roofline(cfg, touched, ms_per_step / 1e3, hbm_peak, tc_peak, read_ceiling_box.get("gbs"))
    # The dominant kernel: on decode shapes moe_layer is one launch (the whole layer); otherwise the up
    # projection (the largest share of the staged pass).
    fused = (not nvfp4) and moe.layer_kernel_count(shape, wdt) == 1
    if fused:
        dom = {"kernel": "layer_fused_kernel (moe_layer: route, plan, up, down, finalize)",
               "achieved": ab["layer"] / (ms_per_step / 1e3) / 1e9, "algorithmic_bytes": ab["layer"],
               "traffic": ncu_traffic("layer_fused")}
    else:
        pair = (not nvfp4) and cid in (2, 3)
        # the NVFP4 up projection runs on 2-SM pairs when I is a multiple of 256, unless MOE_NVFP4_PAIR=0
        nvfp4_pair = nvfp4 and cfg.I % 256 == 0 and os.environ.get("MOE_NVFP4_PAIR") != "0"
        if pair:
            name, key = ": pair_gemm_kernel<up>", "pair_up"
        elif nvfp4:
            name, key = ((": nvfp4_pair_kernel<up>", "nvfp4_pair_up") if nvfp4_pair
                         else (": persistent_nvfp4_kernel<up>", "nvfp4_up"))
        else:
            name, key = "", None
        dom = {"kernel": "grouped_up_swiglu (staged pass)" + name,
               "achieved": up_achieved, "algorithmic_bytes": ab["up"],
               "traffic": ncu_traffic(key) if key else None}
    dom.update(bound="hbm", peak=hbm_peak, unit="GB/s", frac=dom["achieved"] / hbm_peak, peak_source=peak_kind)
    if read_ceiling_box.get("gbs"):
        dom["read_ceiling_gbs"] = read_ceiling_box["gbs"]
        dom["frac_read_ceiling"] = dom["achieved"] / read_ceiling_box["gbs"]
    if dom["frac"] > 1.0:
        dom["note"] = ("frac > 1: the peak is the pool's measured copy (read + write); a read-only stream runs "
                       "above it, and frac_read_ceiling compares it with a pure read measured in this run")

    cs = clocks.summary() or {}
    if cs.get("sm_mhz"):
        cs["ms_x_mhz"] = ms_per_step * cs["sm_mhz"]  # time x clock: comparable across power-capped runs
    res = {
        "workload": cfg.name,
        "config": {"workload": cfg.name, "M": cfg.M, "H": cfg.H, "I": cfg.I, "E": cfg.E, "top_k": cfg.K,
                   "block_size": cfg.B, "seed": cfg.seed, "router_bias": cfg.bias, "touched_experts": touched,
                   "weights": cfg.wdtype,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": ("flush: a 256 MB write before every timed step, outside the timed work" if flush_l2 else
                          "no flush: each step streams GBs of expert weights, far above the 126 MB L2")},
        "dtype": ("nvfp4 weights+activations (e2m1, e4m3 block-16 scales), fp32 accumulate, bf16 I/O" if nvfp4
                  else "bf16"),
        "value": value, "unit": "tokens/s", "ms_per_step": ms_per_step, "us_per_layer": ms_per_step * 1e3,
        "steps": args.steps,
        "kernels_us": {s: v * 1e3 for s, v in stage_ms.items()},
        "staged_us_per_layer": staged_ms * 1e3,
        "graph_us_per_layer": None if graph_ms is None else graph_ms * 1e3,
        "gpu_launches_per_step": moe.layer_kernel_count(shape, wdt),
        "layer_roofline": lroof,
        "dominant_kernel": dom,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d_b, "d2h_bytes_per_step": d2h_b,
                "entry_point": "moe_layer",
                "copies": "x in from pinned host memory and out back to it every step, on two copy streams "
                          "(double-buffered) under the layer of the neighbouring steps",
                "matches_staged": same},
        "clocks": cs,
        "wall_s_timed": t_wall,
    }
    del ws, out_layer, d, nw
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    if cpu_inputs is not None:
        res["cpu_baseline"] = cpu_baseline(cfg, cpu_inputs, target_s=args.cpu_seconds)
    return res


def run_ours(args):
    import torch

    import prefill_sigmoid_top_b200 as moe

    rank, local_rank, world = dist_env()
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    moe.library()  # fail loudly if the CUDA library cannot be loaded

    ids = workload_list(args)
    read_ceiling = {}
    results = []
    for cid in ids:
        cfg = workload(args, cid)
        want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
        results.append(measure_workload(cfg, args, dev, world, rank, want_cpu, read_ceiling))
    head = results[0]

    hbm_peak, tc_peak, peak_kind = peaks()
    dom = head["dominant_kernel"]
    result = {
        "metric": METRIC,
        "value": head["value"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(3, args.warmup),
        "ms_per_step": head["ms_per_step"],
        "us_per_layer": head["us_per_layer"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": head["dtype"],
        "data": "synthetic (seeded; random-init weights of the workload's shapes)",
        "config": head["config"],
        "kernels_us": head["kernels_us"],
        "staged_us_per_layer": head["staged_us_per_layer"],
        "graph_us_per_layer": head["graph_us_per_layer"],
        "gpu_launches": head["gpu_launches_per_step"] * args.steps,
        "roofline": {k: dom[k] for k in ("bound", "kernel", "achieved", "peak", "unit", "frac", "traffic",
                                         "algorithmic_bytes", "peak_source", "read_ceiling_gbs",
                                         "frac_read_ceiling", "note") if k in dom},
        "layer_roofline": head["layer_roofline"],
        "e2e": head["e2e"],
        "clocks": head["clocks"],
        "peaks": {"hbm_copy_gbs": hbm_peak, "bf16_tflops": tc_peak, "source": peak_kind,
                  "hbm_read_ceiling_gbs": read_ceiling.get("gbs"), "hbm_read_ceiling_how": read_ceiling.get("how")},
        "workloads": {r["workload"]: {k: v for k, v in r.items() if k != "workload"} for r in results},
        "wall_s_timed": sum(r["wall_s_timed"] for r in results),
    }
    if "cpu_baseline" in head:
        result["cpu_baseline"] = head["cpu_baseline"]
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# ------------------------------------------------------------------ oracle timing
def oracle_sample_inputs(cfg, d, n):
    """Host inputs of the oracle for the first n tokens of the workload: x, router, gamma, and the weights
    of the experts those tokens route to (bf16 bits; for NVFP4 workloads quantised by the oracle itself)."""
    import oracle
    from prefill_sigmoid_top_b200.inputs import bf16_bits
    x, wr, b, g = (bf16_bits(d["x"][:n]), bf16_bits(d["w_router"]), d["bias"].cpu().numpy(),
                   bf16_bits(d["gamma"]))
    ids, _ = oracle.route(x, wr, b, cfg.K)
    need = sorted(set(int(e) for e in ids.ravel()))
    wg, wu, wd = [None] * cfg.E, [None] * cfg.E, [None] * cfg.E
    for e in need:
        wg[e], wu[e], wd[e] = bf16_bits(d["w_gate"][e]), bf16_bits(d["w_up"][e]), bf16_bits(d["w_down"][e])
        if cfg.wdtype == "nvfp4":
            wg[e], wu[e], wd[e] = (oracle.nvfp4_quantize_bf16(wg[e]), oracle.nvfp4_quantize_bf16(wu[e]),
                                   oracle.nvfp4_quantize_bf16(wd[e]))
    return dict(x=x, wr=wr, b=b, g=g, wg=wg, wu=wu, wd=wd, n=n, experts=len(need))


def cpu_baseline(cfg, ci, target_s=10.0):
    """Times the CPU oracle (as it stands) on a bounded sample of the workload: the first n tokens, as one
    layer call, repeated until target_s seconds have passed."""
    import oracle
    n = ci["n"]
    t0 = time.perf_counter()
    reps = 0
    while True:
        if cfg.wdtype == "nvfp4":
            oracle.layer_nvfp4(ci["x"], ci["wr"], ci["b"], ci["wg"], ci["wu"], ci["wd"], ci["g"], cfg.eps, cfg.K)
        else:
            oracle.layer(ci["x"], ci["wr"], ci["b"], ci["wg"], ci["wu"], ci["wd"], ci["g"], cfg.eps, cfg.K)
        reps += 1
        if time.perf_counter() - t0 >= target_s:
            break
    el = time.perf_counter() - t0
    kind = "NVFP4 layer" if cfg.wdtype == "nvfp4" else "layer"
    return {"value": n * reps / el, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{reps} x the {kind} on the first {n} of {cfg.M} tokens of {cfg.name} as one call "
                      f"({ci['experts']} experts; fp64 C++ oracle, OpenMP), {el:.1f} s"}


def run_reference(args):
    rank, local_rank, world = dist_env()
    if rank != 0:
        return
    import numpy as np
    import torch
    import oracle
    from prefill_sigmoid_top_b200 import inputs
    cfg = workload(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    d = inputs.make_inputs(cfg, dev)
    ci = oracle_sample_inputs(cfg, d, cfg.M if cfg.wdtype == "bf16" else min(cfg.M, 8))
    del d
    touched = ci["experts"]

    def call(n):  # the layer on the first n tokens (NVFP4: those tokens as one call)
        if cfg.wdtype == "nvfp4":
            oracle.layer_nvfp4(ci["x"][:n], ci["wr"], ci["b"], ci["wg"], ci["wu"], ci["wd"], ci["g"], cfg.eps, cfg.K)
        else:
            oracle.layer(ci["x"], ci["wr"], ci["b"], ci["wg"], ci["wu"], ci["wd"], ci["g"], cfg.eps, cfg.K,
                         tokens=np.arange(n, dtype=np.int32))

    # size one step so that the whole run stays within a few minutes
    t0 = time.perf_counter()
    call(1)
    per_token = time.perf_counter() - t0
    budget_per_step = 120.0 / max(1, args.steps + args.warmup)
    n = int(max(1, min(ci["n"], budget_per_step // max(per_token, 1e-3))))
    for _ in range(args.warmup):
        call(n)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        call(n)
    el = time.perf_counter() - t0
    value = n * args.steps / el
    sample = f"{n} of {cfg.M} tokens of {cfg.name} per step (fp64 C++ oracle, OpenMP)"
    print(json.dumps({
        "impl": "reference", "metric": METRIC,
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": cfg.name, "M": cfg.M, "H": cfg.H, "I": cfg.I, "E": cfg.E, "top_k": cfg.K,
                   "block_size": cfg.B, "seed": cfg.seed, "router_bias": cfg.bias, "touched_experts": touched,
                   "weights": cfg.wdtype, "parallelism": "host cores (CPU oracle)",
                   "l2": "no flush: each step streams GBs of expert weights, far above the 126 MB L2"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_route_only(args):
    """moe_route (logits + top-k) on the workload's x, W_r and bias: device time per call and the rate of
    the logits' fma (M*E*H per call).  A kernel measurement, not a layer number."""
    import torch
    import prefill_sigmoid_top_b200 as moe
    from prefill_sigmoid_top_b200 import inputs
    cfg = workload(args)
    w_router, bias, _, x = inputs.router_inputs(cfg)
    x, w_router, bias = x.cuda(), w_router.cuda(), bias.cuda()
    for _ in range(max(3, args.warmup)):
        moe.route(x, w_router, bias, cfg.K)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        moe.route(x, w_router, bias, cfg.K)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / args.steps
    fma = float(cfg.M) * cfg.E * cfg.H
    print(json.dumps({"kernel": "moe_route", "workload": cfg.name, "M": cfg.M, "E": cfg.E, "H": cfg.H,
                      "top_k": cfg.K, "us_per_call": us, "fma_per_s": fma / (us * 1e-6),
                      "steps": args.steps}), flush=True)


def run_tp_emulated(args):
    """The tensor-parallel finalize (cross-rank reduction fused with residual + RMSNorm) with G ranks emulated
    on one GPU: device time per call and the bytes it moves per rank.  A kernel measurement: the exchange goes
    through this GPU's memory, not NVLink."""
    import torch
    import prefill_sigmoid_top_b200 as moe
    from prefill_sigmoid_top_b200 import inputs, tp
    cfg = workload(args)
    G = args.tp_emulate
    g = torch.Generator(device="cuda").manual_seed(cfg.seed)
    x = torch.randn(cfg.M, cfg.H, generator=g, device="cuda").to(torch.bfloat16)
    gamma = torch.ones(cfg.H, dtype=torch.bfloat16, device="cuda")
    tw = torch.softmax(torch.randn(cfg.M, cfg.K, generator=g, device="cuda"), dim=1)
    ys = [(0.1 * torch.randn(cfg.M * cfg.K, cfg.H, generator=g, device="cuda")).to(torch.bfloat16) for _ in range(G)]
    bufs = [torch.zeros(tp.buffer_bytes(G, cfg.M, cfg.H), dtype=torch.uint8, device="cuda") for _ in range(G)]
    outs = [torch.empty_like(x) for _ in range(G)]
    for _ in range(max(3, args.warmup)):
        tp.tp_finalize_emulated(x, ys, tw, gamma, cfg.eps, cfg.M, bufs, outs)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        tp.tp_finalize_emulated(x, ys, tw, gamma, cfg.eps, cfg.M, bufs, outs)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / args.steps
    proto = tp.protocol(cfg.M, G, cfg.M)
    row = cfg.H * 4
    sent = (G - 1) * cfg.M * row if proto == "oneshot" else (G - 1) / G * cfg.M * (row + 2 * cfg.H)
    print(json.dumps({"kernel": "tp_finalize_kernel (emulated ranks, one GPU)", "workload": cfg.name, "ranks": G,
                      "protocol": proto, "M": cfg.M, "H": cfg.H, "top_k": cfg.K, "us_per_call": us,
                      "y_bytes_per_rank": cfg.M * cfg.K * cfg.H * 2, "exchange_bytes_sent_per_rank": int(sent),
                      "steps": args.steps}), flush=True)


# (boxes per stage, stages in flight, contiguous, issuing warps): one 16 KB box per stage as a single panel
# walk; two boxes per stage as the up kernels' gate + up panels (the 2-SM pair kernels: 5 stages, one
# issuing thread); three boxes; and the two-box walk taken in turn by 2 and 4 issuing warps
TMA_PROBES = [(1, 10, False, 1), (2, 5, False, 1), (3, 4, False, 1), (1, 10, True, 1), (2, 5, True, 1),
              (3, 4, True, 1), (2, 6, False, 2), (2, 4, False, 4), (3, 4, False, 4)]


# the copy mixes of moe_measure_tma_mix: what a k-step copies besides its two 16 KB code boxes
TMA_MIXES = {0: "code boxes only",
             1: "+ 8 KB token box (second warp)",
             2: "+ token box and three 2 KB scale chunks, all four from the second warp (the NVFP4 kernels' stage)",
             3: "+ token box and three 2 KB scale chunks, one of them from the first warp",
             4: "+ token box; every fourth step three 8 KB chunks (the scales of four steps)"}


def run_probe_tma(args):
    """The weight-panel stream of the grouped GEMMs on its own: one CTA per SM copying 128 x 64 bf16 boxes
    of 128-row panels into a ring of shared-memory stages (moe_measure_tma_stream), from an 8 GB buffer
    (HBM) and from its first 32 MB (resident in L2), for the probes of TMA_PROBES; best of 3 device-timed
    calls each, beside the plain streaming read of the same 8 GB.  A measurement of the memory system, not
    of the layer."""
    import torch
    import prefill_sigmoid_top_b200 as moe
    buf = torch.ones(8 << 30, dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rows = []

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            moved = fn()
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1) * 1e-3)
        return moved, best

    for where, view in (("hbm", buf), ("l2", buf[: 32 << 20])):
        for boxes, stages, contiguous, warps in TMA_PROBES:
            steps = max(stages, int((4 << 30) / (148 * boxes * 16384)))
            moved, sec = timed(lambda: moe.measure_tma_stream(view, boxes, stages, contiguous, steps, err,
                                                              warps=warps))
            rows.append({"source": where, "boxes_per_stage": boxes, "stages": stages, "issuing_warps": warps,
                         "copy": "bulk 16 KB (panel stored box by box)" if contiguous else "2-D tensor box 128 x 64",
                         "in_flight_kb_per_sm": boxes * stages * 16, "GBps": moved / sec / 1e9,
                         "us_per_stage": sec * 1e6 / steps})
    mixes = []
    for mix in TMA_MIXES:
        per_step = {0: 32768, 1: 40960, 2: 47104, 3: 47104, 4: 47104}[mix]
        steps = int((4 << 30) / (148 * per_step))
        moved, sec = timed(lambda: moe.measure_tma_mix(buf, mix, 4, steps, err))
        mixes.append({"mix": mix, "copies": TMA_MIXES[mix], "stages": 4, "GBps": moved / sec / 1e9,
                      "us_per_step": sec * 1e6 / steps})
    if moe.get_device_error(err) != 0:
        raise RuntimeError("moe_measure_tma_stream / moe_measure_tma_mix: a bounded wait expired")
    read_gbs = measure_read_ceiling(moe, torch, buf)
    print(json.dumps({"kernel": "tma_stream_kernel (moe_measure_tma_stream)",
                      "ctas": "one per SM; one thread per issuing warp waits and issues",
                      "panel": "128 rows x 7168 bf16 columns, 64-column steps", "hbm_read_ceiling_gbs": read_gbs,
                      "probes": rows}), flush=True)
    print(json.dumps({"kernel": "tma_mix_kernel (moe_measure_tma_mix)",
                      "ctas": "one per SM; the first lanes of two warps issue",
                      "step": "one k-step of 256 e2m1 elements: two 128 x 128-byte code boxes (32 KB) from HBM, "
                              "token rows from L2, scale chunks from HBM",
                      "mixes": mixes}), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    elif args.tp_emulate:
        run_tp_emulated(args)
    elif args.route_only:
        run_route_only(args)
    elif args.probe_tma:
        run_probe_tma(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
