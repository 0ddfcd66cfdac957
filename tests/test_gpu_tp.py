"""GPU tests of the tensor-parallel layer (include/moe_b200_tp.h) on one B200.

* One rank: moe_tp_layer returns moe_layer's bits (out, residual, routing) on decode, batch-like and
  many-token shapes.
* G = 2, 4, 8 ranks emulated by one cooperative launch (every rank's CTAs, buffers and partial rows on this
  GPU; the same kernel and exchange as separate GPUs), with both exchange protocols: every rank ends with
  the same bits, and they match the oracle's tensor-parallel layer (each rank's partial rows elementwise,
  the output within the bf16 bar).  The per-rank partial rows come from the library's own grouped kernels
  on each rank's weight slice.
* Consecutive calls and CUDA-graph replays reuse the group buffers (the call number lives on the device).
* A rank whose peer never sends: the bounded wait expires, MOE_ERR_TIMEOUT reaches the host, and the
  device stays usable.
"""
import numpy as np
import pytest
import torch

import oracle
import prefill_sigmoid_top_b200 as moe
from prefill_sigmoid_top_b200 import inputs, tp
from tests._util import bf16_bits, bits_to_f64, rms

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _close(got, ref, rel=2.0 ** -7, abs_rms=1e-2):
    tol = rel * np.abs(ref) + abs_rms * rms(ref)
    d = np.abs(np.asarray(got, np.float64) - ref)
    return bool((d <= tol).all()), float(d.max())


def _host(d, cfg):
    return dict(x=bf16_bits(d["x"]), wr=bf16_bits(d["w_router"]), b=d["bias"].cpu().numpy(), g=bf16_bits(d["gamma"]),
                wg=[bf16_bits(d["w_gate"][e]) for e in range(cfg.E)], wu=[bf16_bits(d["w_up"][e]) for e in range(cfg.E)],
                wd=[bf16_bits(d["w_down"][e]) for e in range(cfg.E)])


ONE_RANK = [
    inputs.WORKLOADS[0],
    inputs.WORKLOADS[0].with_(M=40, H=512, I=256, E=16, K=4, B=16, seed=11, bias="normal"),
    inputs.WORKLOADS[0].with_(M=100, H=768, I=256, E=32, K=8, B=64, seed=12, bias="zipf"),
    inputs.WORKLOADS[1].with_(E=32, seed=5),  # decode shape: moe_layer takes its single launch
]


@pytest.mark.parametrize("cfg", ONE_RANK, ids=lambda c: f"M{c.M}_H{c.H}_E{c.E}")
def test_one_rank_is_moe_layer(cfg):
    d = inputs.make_inputs(cfg, DEV)
    shape = moe.Shape(cfg.M, cfg.H, cfg.I, cfg.E, cfg.K, cfg.B)
    out_l, res_l = torch.empty_like(d["x"]), torch.empty_like(d["x"])
    ids_l = torch.empty(cfg.M, cfg.K, dtype=torch.int32, device=DEV)
    w_l = torch.empty(cfg.M, cfg.K, dtype=torch.float32, device=DEV)
    moe.layer(d["x"], d["w_router"], d["bias"], d["w_gate"], d["w_up"], d["w_down"], d["gamma"], cfg.eps, cfg.K,
              cfg.B, out=out_l, residual_out=res_l, topk_ids=ids_l, topk_w=w_l)
    group = tp.TPGroup(0, 1, cfg.M, cfg.H)
    out_t = torch.full_like(d["x"], float("nan"))
    res_t = torch.full_like(d["x"], float("nan"))
    ids_t = torch.full((cfg.M, cfg.K), -1, dtype=torch.int32, device=DEV)
    w_t = torch.full((cfg.M, cfg.K), float("nan"), dtype=torch.float32, device=DEV)
    ws = torch.empty(tp.layer_workspace_size_tp(shape), dtype=torch.uint8, device=DEV)
    tp.tp_layer(d["x"], d["w_router"], d["bias"], d["w_gate"], d["w_up"], d["w_down"], d["gamma"], cfg.eps, cfg.K,
                cfg.B, group, ws=ws, out=out_t, residual_out=res_t, topk_ids=ids_t, topk_w=w_t)
    torch.cuda.synchronize()
    assert moe.get_device_error(ws[:4].view(torch.int32)) == 0
    assert torch.equal(ids_t, ids_l) and torch.equal(w_t, w_l)
    assert torch.equal(out_t, out_l) and torch.equal(res_t, res_l)


def _rank_partials(d, cfg, G):
    """Each rank's y_r from the library's grouped kernels on that rank's weight slice, and the routing."""
    Ir = cfg.I // G
    shape = moe.Shape(cfg.M, cfg.H, Ir, cfg.E, cfg.K, cfg.B)
    ids, tw = moe.route(d["x"], d["w_router"], d["bias"], cfg.K)
    plan = moe.align_block_size(ids, cfg.E, cfg.B)
    ys = []
    for r in range(G):
        g_r, u_r, d_r = tp.shard_weights(d["w_gate"], d["w_up"], d["w_down"], r, G)
        h = moe.grouped_up_swiglu(d["x"], g_r, u_r, plan, shape)
        ys.append(moe.grouped_down(h, d_r, plan, shape))
    return ids, tw, ys


def _emulate(d, cfg, tw, ys, max_tokens, bufs=None, residual=True):
    G = len(ys)
    if bufs is None:
        bufs = [torch.zeros(tp.buffer_bytes(G, max_tokens, cfg.H), dtype=torch.uint8, device=DEV) for _ in range(G)]
    outs = [torch.full_like(d["x"], float("nan")) for _ in range(G)]
    ress = [torch.full_like(d["x"], float("nan")) for _ in range(G)] if residual else None
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    tp.tp_finalize_emulated(d["x"], ys, tw, d["gamma"], cfg.eps, max_tokens, bufs, outs, ress, err_flag=err)
    torch.cuda.synchronize()
    assert moe.get_device_error(err) == 0
    return outs, ress, bufs


@pytest.mark.parametrize("protocol", ["oneshot", "twoshot"])
@pytest.mark.parametrize("G", [2, 4, 8])
@pytest.mark.parametrize("M", [5, 24, 67])
def test_emulated_ranks_match_the_oracle(G, M, protocol, monkeypatch):
    if protocol == "oneshot" and M > 24:
        pytest.skip("the one-shot exchange is sized for up to 24 tokens")
    monkeypatch.setenv("MOE_TP_PROTOCOL", protocol)
    cfg = inputs.WORKLOADS[0].with_(M=M, H=512, I=1024, E=16, K=4, B=16, seed=100 + 10 * G + M, bias="normal")
    assert tp.protocol(M, G, 96) == protocol
    d = inputs.make_inputs(cfg, DEV)
    ids, tw, ys = _rank_partials(d, cfg, G)
    outs, ress, _ = _emulate(d, cfg, tw, ys, max_tokens=96)
    for r in range(1, G):  # every rank holds the same bits
        assert torch.equal(outs[r], outs[0]) and torch.equal(ress[r], ress[0])
    h = _host(d, cfg)
    ref = oracle.layer_tp(h["x"], h["wr"], h["b"], h["wg"], h["wu"], h["wd"], h["g"], cfg.eps, cfg.K, G,
                          want_y_parts=True)
    assert np.array_equal(ids.cpu().numpy(), ref["ids"])
    for r in range(G):
        ok, e = _close(bits_to_f64(bf16_bits(ys[r])).reshape(M, cfg.K, cfg.H), bits_to_f64(ref["y_parts"][r]))
        assert ok, ("y partial", r, e)
    ok, e = _close(bits_to_f64(bf16_bits(outs[0])), ref["out_f64"])
    assert ok, ("out", e)
    assert np.abs(bits_to_f64(bf16_bits(outs[0])) - ref["out_f64"]).max() <= 2e-2 * rms(ref["out_f64"])
    assert np.abs(bits_to_f64(bf16_bits(ress[0])) - ref["residual_f64"]).max() <= 2e-2 * rms(ref["residual_f64"])


@pytest.mark.parametrize("M", [8, 67])
def test_emulated_one_rank_group_is_the_finalize(M):
    # G = 1 through the emulated entry point: the single-GPU finalize's bits
    cfg = inputs.WORKLOADS[0].with_(M=M, H=512, I=256, E=16, K=4, B=16, seed=7 + M, bias="normal")
    d = inputs.make_inputs(cfg, DEV)
    ids, tw, ys = _rank_partials(d, cfg, 1)
    outs, ress, _ = _emulate(d, cfg, tw, ys, max_tokens=M)
    out, res = moe.finalize_rmsnorm(d["x"], ys[0], tw, d["gamma"], cfg.eps, want_residual=True)
    assert torch.equal(outs[0], out) and torch.equal(ress[0], res)


def test_consecutive_calls_and_graph_replay_reuse_the_buffers():
    G, M = 2, 40
    cfg = inputs.WORKLOADS[0].with_(M=M, H=512, I=512, E=16, K=4, B=16, seed=55, bias="normal")
    d = inputs.make_inputs(cfg, DEV)
    ids, tw, ys = _rank_partials(d, cfg, G)
    ref_outs, _, _ = _emulate(d, cfg, tw, ys, max_tokens=64)
    ys2 = [y.flip(0).contiguous() for y in ys]  # other partial rows: other results
    ref2, _, _ = _emulate(d, cfg, tw, ys2, max_tokens=64)
    assert not torch.equal(ref2[0], ref_outs[0])
    bufs = [torch.zeros(tp.buffer_bytes(G, 64, cfg.H), dtype=torch.uint8, device=DEV) for _ in range(G)]
    for it in range(6):  # alternate inputs across calls on the same buffers (both data parities, twice)
        cur, want = (ys, ref_outs) if it % 2 == 0 else (ys2, ref2)
        outs, _, _ = _emulate(d, cfg, tw, cur, max_tokens=64, bufs=bufs, residual=False)
        assert all(torch.equal(o, want[0]) for o in outs), it
    # the same call captured once and replayed, with the partial rows changed in place between replays
    yin = [y.clone() for y in ys]
    outs = [torch.empty_like(d["x"]) for _ in range(G)]
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        tp.tp_finalize_emulated(d["x"], yin, tw, d["gamma"], cfg.eps, 64, bufs, outs, None, err_flag=err)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        tp.tp_finalize_emulated(d["x"], yin, tw, d["gamma"], cfg.eps, 64, bufs, outs, None, err_flag=err)
    for it in range(4):
        src, want = (ys2, ref2) if it % 2 == 0 else (ys, ref_outs)
        for a, b in zip(yin, src):
            a.copy_(b)
        for o in outs:
            o.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert all(torch.equal(o, want[0]) for o in outs), it
    assert moe.get_device_error(err) == 0
    del graph


def test_missing_peer_times_out_and_the_device_stays_usable():
    # rank 0 of a two-rank group whose rank 1 never runs: its waits expire (2 s), MOE_ERR_TIMEOUT is
    # reported on the host, and nothing faults or hangs
    cfg = inputs.WORKLOADS[0].with_(M=4, H=512, I=256, E=16, K=4, B=16, seed=9, bias="normal")
    d = inputs.make_inputs(cfg, DEV)
    ids, tw, ys = _rank_partials(d, cfg, 1)
    bufs = [torch.zeros(tp.buffer_bytes(2, 8, cfg.H), dtype=torch.uint8, device=DEV) for _ in range(2)]
    group = tp.TPGroup(0, 1, 8, cfg.H)
    c = group.c()
    c.world = 2
    c.bufs[0], c.bufs[1] = bufs[0].data_ptr(), bufs[1].data_ptr()
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    tp.tp_finalize(d["x"], ys[0], tw, d["gamma"], cfg.eps, group, err_flag=err)
    assert moe.get_device_error(err) == 5  # MOE_ERR_TIMEOUT
    # the context is intact: a one-rank call gives the finalize's bits afterwards
    test_emulated_one_rank_group_is_the_finalize(8)
