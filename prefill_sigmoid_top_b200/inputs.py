"""Seeded synthetic inputs for the routed-MoE layer.

This module only draws random numbers and lays them out; it holds none of the
layer's arithmetic, and both the CUDA library's callers and the CPU oracle's
tests take their inputs from it.

Workloads (shapes of the pages' named GLM decode / batch / prefill routes:
flashinfer PR #6511 analysis, §2-§4, glm_decode_m8 / glm_batch_m512 /
glm_decode_m1000 / glm_prefill_m2048; H=7168, top_k=16 from the flashinfer
PR #5701 analysis, intro):

====  ===================  ======  =====  =====  ===  ==  ===  ======
 id   name                  M       H      I      E   K   B    bias
====  ===================  ======  =====  =====  ===  ==  ===  ======
 0    tiny                 16      256    128    8    2   16   zero
 1    decode_m8            8       7168   2048   256  16  16   normal
 2    batch_m512           512     7168   2048   256  16  64   normal
 3    prefill_m2048_zipf   2048    7168   2048   256  16  128  zipf
 4    nvfp4_m1000          1000    7168   2048   256  16  16   normal
====  ===================  ======  =====  =====  ===  ==  ===  ======

Recipe (all values drawn in fp32 then rounded to bf16 with round-to-nearest-even):

* Router-side tensors are drawn on the CPU from ``torch.Generator().manual_seed(seed)``
  in this order: ``w_router ~ N(0, 1/H)`` [E,H]; ``bias`` [E] (fp32, kept fp32);
  ``gamma = 1 + 0.1*N(0,1)`` [H]; ``x ~ N(0,1)`` [M,H].  They are small, so the
  same values are produced on any machine and then copied to the device.
* ``bias``: ``zero`` -> all 0; ``normal`` -> N(0, 0.1) (variance 0.1);
  ``zipf`` -> ``-ZIPF_ALPHA * 1.1 * ln(rank_e)`` with ``rank`` a random
  permutation of 1..E, giving a Zipf(s=1.1)-shaped popularity over experts.
* Expert weights are drawn on the target device from
  ``torch.Generator(device).manual_seed(seed + 1000)``, expert by expert:
  ``w_gate[e] ~ N(0, 1/H)`` [I,H], then ``w_up[e] ~ N(0, 1/H)`` [I,H], then
  ``w_down[e] ~ N(0, 1/I)`` [H,I].  Layout: ``w_gate``/``w_up`` [E,I,H] and
  ``w_down`` [E,H,I], row-major (the contraction dimension is contiguous).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

# Temperature of the Zipf-shaped router bias of the prefill workload.  Chosen
# so that the busiest expert receives about 10x the mean number of routed
# slots on the seed-3 M=2048 inputs; the value is produced, and its ratio
# recorded, by tests/golden/calibrate_zipf_alpha.py (which routes with the
# CPU oracle).
ZIPF_ALPHA = 0.4023


@dataclass(frozen=True)
class MoEConfig:
    name: str
    M: int
    H: int
    I: int
    E: int
    K: int
    B: int
    seed: int
    bias: str = "normal"        # zero | normal | zipf
    wdtype: str = "bf16"        # bf16 | nvfp4
    eps: float = 1e-5

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)


WORKLOADS = {
    0: MoEConfig("tiny", M=16, H=256, I=128, E=8, K=2, B=16, seed=0, bias="zero"),
    1: MoEConfig("decode_m8", M=8, H=7168, I=2048, E=256, K=16, B=16, seed=1),
    2: MoEConfig("batch_m512", M=512, H=7168, I=2048, E=256, K=16, B=64, seed=2),
    3: MoEConfig("prefill_m2048_zipf", M=2048, H=7168, I=2048, E=256, K=16, B=128, seed=3, bias="zipf"),
    4: MoEConfig("nvfp4_m1000", M=1000, H=7168, I=2048, E=256, K=16, B=16, seed=4, wdtype="nvfp4"),
}


def router_inputs(cfg: MoEConfig, alpha: float | None = None):
    """(w_router bf16 [E,H], bias fp32 [E], gamma bf16 [H], x bf16 [M,H]) on the CPU."""
    g = torch.Generator().manual_seed(cfg.seed)
    w_router = (torch.randn(cfg.E, cfg.H, generator=g) * math.sqrt(1.0 / cfg.H)).to(torch.bfloat16)
    if cfg.bias == "zero":
        bias = torch.zeros(cfg.E, dtype=torch.float32)
    elif cfg.bias == "normal":
        bias = torch.randn(cfg.E, generator=g) * math.sqrt(0.1)
    elif cfg.bias == "zipf":
        a = ZIPF_ALPHA if alpha is None else alpha
        rank = torch.randperm(cfg.E, generator=g).to(torch.float64) + 1.0
        bias = (-a * 1.1 * torch.log(rank)).to(torch.float32)
    else:
        raise ValueError(cfg.bias)
    gamma = (1.0 + 0.1 * torch.randn(cfg.H, generator=g)).to(torch.bfloat16)
    x = torch.randn(cfg.M, cfg.H, generator=g).to(torch.bfloat16)
    return w_router, bias.contiguous(), gamma, x


def expert_weights(cfg: MoEConfig, device="cpu"):
    """(w_gate [E,I,H], w_up [E,I,H], w_down [E,H,I]) bf16 on ``device``."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(cfg.seed + 1000)
    w_gate = torch.empty(cfg.E, cfg.I, cfg.H, dtype=torch.bfloat16, device=device)
    w_up = torch.empty_like(w_gate)
    w_down = torch.empty(cfg.E, cfg.H, cfg.I, dtype=torch.bfloat16, device=device)
    sg, sd = math.sqrt(1.0 / cfg.H), math.sqrt(1.0 / cfg.I)
    for e in range(cfg.E):
        w_gate[e] = (torch.randn(cfg.I, cfg.H, generator=g, device=device) * sg).to(torch.bfloat16)
        w_up[e] = (torch.randn(cfg.I, cfg.H, generator=g, device=device) * sg).to(torch.bfloat16)
        w_down[e] = (torch.randn(cfg.H, cfg.I, generator=g, device=device) * sd).to(torch.bfloat16)
    return w_gate, w_up, w_down


def make_inputs(cfg: MoEConfig, device="cpu"):
    """All layer inputs as a dict of tensors on ``device`` (router side drawn on the CPU)."""
    w_router, bias, gamma, x = router_inputs(cfg)
    w_gate, w_up, w_down = expert_weights(cfg, device)
    dev = torch.device(device)
    return dict(x=x.to(dev), w_router=w_router.to(dev), bias=bias.to(dev), gamma=gamma.to(dev),
                w_gate=w_gate, w_up=w_up, w_down=w_down)


def bf16_bits(t: torch.Tensor):
    """Raw bf16 bit patterns of a (CPU or device) tensor as a numpy uint16 array."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")
