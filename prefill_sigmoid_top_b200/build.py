"""Build libmoe_b200.so in-tree with nvcc for sm_100a (run: python -m prefill_sigmoid_top_b200.build)."""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libmoe_b200.so")
SOURCES = ["api.cu", "router.cu", "router_screen.cu", "align.cu", "finalize.cu", "gemm_bf16.cu", "gemm_persistent.cu",
           "gemm_pair.cu", "nvfp4.cu", "nvfp4_pair.cu", "layer_fused.cu", "measure.cu", "tp_finalize.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17", "-DNDEBUG", "-Xcompiler", "-fPIC",
         "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include"), "-I", CSRC]


def _stale(out: str, deps: list[str]) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


TRACE_LIB = os.path.join(PKG, "libmoe_b200_trace.so")


def build(force: bool = False, verbose: bool = False, extra_flags: list[str] | None = None,
          trace: bool = False) -> str:
    """Compile the library; trace=True builds the timeline variant instead (-DMOE_PAIR_TRACE for the
    2-SM pair GEMMs, -DMOE_LAYER_TRACE for the single-launch layer, into libmoe_b200_trace.so; see
    pair_trace.py and layer_trace.py), never loaded by the package."""
    build_dir = BUILD + ("_trace" if trace else "")
    lib = TRACE_LIB if trace else LIB
    os.makedirs(build_dir, exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    inc = os.path.join(ROOT, "include")
    headers += [os.path.join(inc, f) for f in os.listdir(inc) if f.endswith(".h")]
    flags = FLAGS + (["-DMOE_PAIR_TRACE", "-DMOE_LAYER_TRACE"] if trace else []) + (extra_flags or [])
    jobs = []
    objs = []
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(build_dir, src.replace(".cu", ".o"))
        objs.append(obj)
        if force or _stale(obj, [path, *headers]):
            jobs.append([NVCC, *flags, "-c", path, "-o", obj])
    with cf.ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        for cmd, res in zip(jobs, ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), jobs)):
            if verbose or res.returncode != 0:
                sys.stderr.write(res.stdout + res.stderr)
            if res.returncode != 0:
                raise RuntimeError(f"nvcc failed: {' '.join(cmd)}")
    if force or jobs or _stale(lib, objs):
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", *objs, "-o", tmp])
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, trace="--trace" in sys.argv))
