"""GPU parity of the NVFP4 path (e2m1 weights and activations, e4m3 block-16 scales).

* The GPU quantiser is bit-exact against the oracle's (codes, scales, global
  scale): the same fp32 recipe takes every rounding decision on both sides.
* The prepared blob keeps the codes and regroups the scales into 512-byte
  atoms (checked against the atom index formula).
* Grouped projections and the whole layer against the oracle's NVFP4 layer:
  h elementwise as for bf16 (both sides quantise x identically, only the
  accumulation order differs); y and out within the NVFP4 bound of
  6e-2 x RMS (h is re-quantised from slightly different bf16 values).
"""
import numpy as np
import pytest
import torch

import oracle
import prefill_sigmoid_top_b200 as moe
from prefill_sigmoid_top_b200 import inputs
from tests._util import bf16_bits, bits_to_f64, rms, sample_tokens, token_tile

pytestmark = pytest.mark.gpu
DEV = "cuda"


def unpack_codes(packed):
    p = np.asarray(packed, np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def _special_matrices():
    rng = np.random.default_rng(3)
    mats = []
    m = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    m[0, :16] = 0.0                           # an all-zero block
    m[1, :16] = 1e-30                         # a block far below the matrix amax
    m[2, 16:32] = np.linspace(-3, 3, 16)      # includes exact e2m1 midpoints after scaling
    mats.append(m)
    mats.append((rng.standard_normal((64, 256)) * 50).astype(np.float32))
    mats.append(np.zeros((64, 256), np.float32))  # amax 0 -> gs 1
    mats.append(_tie_matrix())
    return torch.tensor(np.stack(mats)).to(torch.bfloat16)


def _bf16_step(v, up):
    """The bf16 value next to v (a bf16-exact float32) towards +inf (up) or -inf."""
    b = np.array([v], np.float32).view(np.uint32)[0] >> 16
    b = b + 1 if (v >= 0) == up else b - 1
    return np.array([b << 16], np.uint32).view(np.float32)[0]


def _tie_matrix():
    """Quotients exactly on the e2m1 rounding midpoints.  The matrix amax is 2688 = 6 * 448, so the global
    scale is exactly 1; a block whose amax is 6 d, d a value of e4m3 (3 mantissa bits), gets the scale d
    exactly, and its elements m * d (bf16-exact) divide to m for every midpoint m of the e2m1 grid: the
    code must take the tie to even.  The blocks also hold the bf16 neighbours of those elements."""
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    m = np.zeros((64, 256), np.float32)
    for r in range(64):
        for b in range(16):
            k, j = (r * 16 + b) % 13 - 6, (r + b) % 8  # d = 2^k (1 + j/8), from 2^-6 up to 120
            d = np.float32(2.0 ** k * (1 + j / 8))
            blk = [6 * d] + [mi * d for mi in mids] + [_bf16_step(np.float32(mi * d), i % 2 == 0)
                                                       for i, mi in enumerate(mids)] + [-2.5 * d]
            m[r, 16 * b:16 * b + 16] = blk
    m[0, 0] = 2688.0  # the matrix amax (its block: d = 448)
    return m


def test_quantize_bitexact_against_oracle():
    w = _special_matrices()
    codes, scales, gs = moe.quantize_nvfp4(w.to(DEV))
    torch.cuda.synchronize()
    codes, scales, gs = unpack_codes(codes.cpu().numpy()), scales.cpu().numpy(), gs.cpu().numpy()
    wb = bf16_bits(w)
    for m in range(w.shape[0]):
        oc, osc, ogs = oracle.nvfp4_quantize_bf16(wb[m])
        assert np.float32(ogs) == gs[m]
        assert np.array_equal(osc, scales[m])
        assert np.array_equal(oc, codes[m])


def test_quantize_bitexact_expert_weights():
    cfg = inputs.WORKLOADS[0].with_(E=4, I=256, H=512, seed=17)
    wg, _, wd = inputs.expert_weights(cfg, DEV)
    for w in (wg, wd):
        codes, scales, gs = moe.quantize_nvfp4(w)
        torch.cuda.synchronize()
        codes, scales, gs = unpack_codes(codes.cpu().numpy()), scales.cpu().numpy(), gs.cpu().numpy()
        for e in range(cfg.E):
            oc, osc, ogs = oracle.nvfp4_quantize_bf16(bf16_bits(w[e]))
            assert np.float32(ogs) == gs[e] and np.array_equal(osc, scales[e]) and np.array_equal(oc, codes[e])


def test_prepared_blob_layout():
    shape = moe.Shape(M=4, H=512, I=256, E=2, top_k=1, block_size=16)
    w = torch.randn(2, 256, 512, device=DEV).to(torch.bfloat16)
    codes, scales, gs = moe.quantize_nvfp4(w)
    blob = moe.prepare_nvfp4_weights(codes, scales, shape, 0).cpu().numpy()
    codes, scales = codes.cpu().numpy().reshape(512, 256), scales.cpu().numpy().reshape(512, 32)
    nb = codes.size
    assert np.array_equal(blob[:nb], codes.ravel())
    atoms = blob[nb:]
    assert atoms.size == scales.size
    r, j = np.meshgrid(np.arange(512), np.arange(32), indexing="ij")
    idx = ((r // 128) * 8 + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + j % 4
    assert np.array_equal(atoms[idx], scales)


def _oracle_weights(d, E):
    q = lambda t: [oracle.nvfp4_quantize_bf16(bf16_bits(t[e])) for e in range(E)]
    return q(d["w_gate"]), q(d["w_up"]), q(d["w_down"])


def _close(got, ref, rel, abs_rms):
    tol = rel * np.abs(ref) + abs_rms * rms(ref)
    d = np.abs(got - ref)
    return (d <= tol).all(), float(d.max()), int((d > tol).sum())


NVFP4_CASES = [dict(M=40, H=512, I=256, E=16, K=4, B=16), dict(M=300, H=256, I=512, E=8, K=4, B=16),
               dict(M=7, H=768, I=256, E=32, K=6, B=32),
               dict(M=300, H=1024, I=512, E=8, K=4, B=16),   # ~150 rows per expert: two token tiles
               dict(M=5, H=512, I=256, E=2, K=1, B=16)]      # a few rows per expert: N = 16


# "pair": the default (2-SM pair kernels wherever the weight blocks divide the expert: up I % 256 == 0,
# down H % 512 == 0); "single": MOE_NVFP4_PAIR=0, the single-SM kernels.
@pytest.mark.parametrize("kernels", ["pair", "single"])
@pytest.mark.parametrize("case", NVFP4_CASES, ids=lambda c: f"M{c['M']}_H{c['H']}_E{c['E']}")
def test_nvfp4_grouped_and_layer(case, kernels, monkeypatch):
    if kernels == "single":
        monkeypatch.setenv("MOE_NVFP4_PAIR", "0")
    cfg = inputs.WORKLOADS[0].with_(bias="normal", seed=case["M"] + 5, **case)
    d = inputs.make_inputs(cfg, DEV)
    shape = moe.Shape(cfg.M, cfg.H, cfg.I, cfg.E, cfg.K, cfg.B)
    nw = moe.nvfp4_weights(d["w_gate"], d["w_up"], d["w_down"], shape)
    gq, uq, dq = _oracle_weights(d, cfg.E)
    hb = dict(x=bf16_bits(d["x"]), wr=bf16_bits(d["w_router"]), b=d["bias"].cpu().numpy(), g=bf16_bits(d["gamma"]))
    r = oracle.layer_nvfp4(hb["x"], hb["wr"], hb["b"], gq, uq, dq, hb["g"], cfg.eps, cfg.K)
    # grouped projections on the oracle's plan
    plan_o = oracle.align(r["ids_all"], cfg.E, cfg.B)
    cap = moe.align_capacity(shape)
    sorted_full = np.full(cap, -1, np.int32)
    sorted_full[: plan_o["ntpp"]] = plan_o["sorted_ids"]
    bexp = np.zeros(cap // cfg.B + 1, np.int32)
    bexp[: len(plan_o["block_expert"])] = plan_o["block_expert"]
    plan = dict(sorted_ids=torch.from_numpy(sorted_full).to(DEV), block_expert=torch.from_numpy(bexp).to(DEV),
                expert_counts=torch.from_numpy(plan_o["counts"]).to(DEV),
                expert_offsets=torch.from_numpy(plan_o["offsets"]).to(DEV),
                num_tokens_post_padded=torch.tensor([plan_o["ntpp"]], dtype=torch.int32, device=DEV))
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    h = moe.grouped_up_swiglu_nvfp4(d["x"], nw, plan, shape, err_flag=err)
    y = moe.grouped_down_nvfp4(h, nw, plan, shape, err_flag=err)
    torch.cuda.synchronize()
    assert moe.get_device_error(err) == 0
    real = plan_o["sorted_ids"] < cfg.M * cfg.K
    rows, slots = np.nonzero(real)[0], plan_o["sorted_ids"][real]
    # only the real plan rows: the padding rows were never written and may hold any bits
    ok, e, nbad = _close(bits_to_f64(bf16_bits(h)[rows]), bits_to_f64(r["h_all"])[slots], 2.0 ** -7, 1e-2)
    assert ok, ("h", e, nbad)
    y_ref = bits_to_f64(r["y"].reshape(cfg.M * cfg.K, cfg.H))
    ok, e, nbad = _close(bits_to_f64(bf16_bits(y)), y_ref, 2.0 ** -3, 6e-2)
    assert ok, ("y", e, nbad)
    # the whole layer
    ids = torch.empty(cfg.M, cfg.K, dtype=torch.int32, device=DEV)
    out = moe.layer_nvfp4(d["x"], d["w_router"], d["bias"], nw, d["gamma"], cfg.eps, cfg.K, cfg.B, cfg.I,
                          topk_ids=ids)
    torch.cuda.synchronize()
    assert np.array_equal(ids.cpu().numpy(), r["ids_all"])
    ref = r["out_f64"]
    assert np.abs(bits_to_f64(bf16_bits(out)) - ref).max() <= 6e-2 * rms(ref)


@pytest.mark.parametrize("case", NVFP4_CASES[3:4] + NVFP4_CASES[0:1] + NVFP4_CASES[4:5],
                         ids=lambda c: f"M{c['M']}_H{c['H']}_E{c['E']}")
def test_nvfp4_pair_equals_single_sm(case, monkeypatch):
    """The pair kernels compute every output element from the same operands, scales and K order as the
    single-SM kernels (one block-scaled MMA of K = 64 after another), so h and y agree bit for bit."""
    cfg = inputs.WORKLOADS[0].with_(bias="normal", seed=case["M"] + 11, **case)
    d = inputs.make_inputs(cfg, DEV)
    shape = moe.Shape(cfg.M, cfg.H, cfg.I, cfg.E, cfg.K, cfg.B)
    nw = moe.nvfp4_weights(d["w_gate"], d["w_up"], d["w_down"], shape)
    ids, _ = moe.route(d["x"], d["w_router"], d["bias"], cfg.K)
    plan = moe.align_block_size(ids, cfg.E, cfg.B)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)

    def run():
        h = moe.grouped_up_swiglu_nvfp4(d["x"], nw, plan, shape, err_flag=err)
        y = moe.grouped_down_nvfp4(h, nw, plan, shape, err_flag=err)
        torch.cuda.synchronize()
        return h, y

    h_p, y_p = run()
    monkeypatch.setenv("MOE_NVFP4_PAIR", "0")
    h_s, y_s = run()
    assert moe.get_device_error(err) == 0
    sorted_ids = plan["sorted_ids"].cpu().numpy()[: int(plan["num_tokens_post_padded"].item())]
    rows = np.nonzero(sorted_ids < cfg.M * cfg.K)[0]
    rows_t = torch.from_numpy(rows).to(DEV)
    assert torch.equal(h_p.view(torch.int16)[rows_t], h_s.view(torch.int16)[rows_t])
    assert torch.equal(y_p.view(torch.int16), y_s.view(torch.int16))


def test_nvfp4_rejects_unsupported_intermediate():
    shape = moe.Shape(M=4, H=256, I=128, E=2, top_k=1, block_size=16)  # I % 256 != 0
    x = torch.zeros(4, 256, dtype=torch.bfloat16, device=DEV)
    blob = torch.zeros(1 << 20, dtype=torch.uint8, device=DEV)
    gs = torch.ones(2, dtype=torch.float32, device=DEV)
    nw = moe.NVFP4Weights(blob, blob, blob, gs, gs, gs)
    with pytest.raises(moe.MoEError) as ei:
        moe.layer_nvfp4(x, torch.zeros(2, 256, dtype=torch.bfloat16, device=DEV), None, nw,
                        torch.ones(256, dtype=torch.bfloat16, device=DEV), 1e-5, 1, 16, 128)
    assert ei.value.status == 2


@pytest.mark.slow
def test_nvfp4_layer_full_size_sampled():
    cfg = inputs.WORKLOADS[4]
    d = inputs.make_inputs(cfg, DEV)
    shape = moe.Shape(cfg.M, cfg.H, cfg.I, cfg.E, cfg.K, cfg.B)
    nw = moe.nvfp4_weights(d["w_gate"], d["w_up"], d["w_down"], shape)
    ids = torch.empty(cfg.M, cfg.K, dtype=torch.int32, device=DEV)
    out = moe.layer_nvfp4(d["x"], d["w_router"], d["bias"], nw, d["gamma"], cfg.eps, cfg.K, cfg.B, cfg.I,
                          topk_ids=ids)
    torch.cuda.synchronize()
    gq, uq, dq = _oracle_weights(d, cfg.E)
    del d["w_gate"], d["w_up"], d["w_down"]
    hb = dict(x=bf16_bits(d["x"]), wr=bf16_bits(d["w_router"]), b=d["bias"].cpu().numpy(), g=bf16_bits(d["gamma"]))
    ids_np = ids.cpu().numpy()
    tokens = sample_tokens(ids_np, 64, 4, token_tile(cfg))
    tokens = np.union1d(tokens, np.array([0, 1, cfg.M - 2, cfg.M - 1], np.int32)).astype(np.int32)
    r = oracle.layer_nvfp4(hb["x"], hb["wr"], hb["b"], gq, uq, dq, hb["g"], cfg.eps, cfg.K, tokens=tokens)
    assert np.array_equal(ids.cpu().numpy(), r["ids_all"])
    ref = r["out_f64"]
    got = bits_to_f64(bf16_bits(out))[tokens]
    assert np.abs(got - ref).max() <= 6e-2 * rms(ref)
