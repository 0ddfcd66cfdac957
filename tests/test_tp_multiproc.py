"""The tensor-parallel layer's host side on two gloo ranks (CPU): the weight slices each rank takes, the
exchange of group-buffer handles, and the reduction semantics -- every rank's partial (computed by the
oracle on that rank's slice of the weights), summed across the ranks with an all-reduce, then normalised,
is the oracle's two-rank layer bit for bit and the unsharded layer within the bf16 bar (2e-2 x RMS)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
        dist.init_process_group("gloo", rank=rank, world_size=world)
        import oracle
        from prefill_sigmoid_top_b200 import inputs, tp
        from prefill_sigmoid_top_b200.inputs import bf16_bits

        # handles travel as host bytes, in rank order
        got = tp.exchange_handles(bytes([rank + 1]) * tp.HANDLE_BYTES)
        assert got == [bytes([r + 1]) * tp.HANDLE_BYTES for r in range(world)]

        cfg = inputs.WORKLOADS[0].with_(M=5, H=256, I=256, E=8, K=3, bias="normal", seed=77)
        d = inputs.make_inputs(cfg, "cpu")
        gate_r, up_r, down_r = tp.shard_weights(d["w_gate"], d["w_up"], d["w_down"], rank, world)
        assert gate_r.shape == (cfg.E, cfg.I // world, cfg.H) and down_r.shape == (cfg.E, cfg.H, cfg.I // world)
        E = cfg.E
        full = [[bf16_bits(w[e]) for e in range(E)] for w in (d["w_gate"], d["w_up"], d["w_down"])]
        mine = [[bf16_bits(w[e]) for e in range(E)] for w in (gate_r, up_r, down_r)]
        x, wr, b, g = bf16_bits(d["x"]), bf16_bits(d["w_router"]), d["bias"].numpy(), bf16_bits(d["gamma"])
        # the slice this rank holds is the oracle's rank-r partition of I: same partial rows
        part = oracle.tp_partial(x, wr, b, *full, cfg.K, world, rank, want_y=True)
        own = oracle.tp_partial(x, wr, b, *mine, cfg.K, 1, 0, want_y=True)
        assert np.array_equal(part["y"], own["y"])
        # reduce the fp64 partials across the ranks, then normalise
        s = torch.from_numpy(part["p"].copy())
        dist.all_reduce(s, op=dist.ReduceOp.SUM)
        out, res, o64 = oracle.rmsnorm_rows(s.numpy(), g, cfg.eps)
        ref_tp = oracle.layer_tp(x, wr, b, *full, g, cfg.eps, cfg.K, world)
        assert np.array_equal(out, ref_tp["out"]) and np.array_equal(res, ref_tp["residual"])
        ref = oracle.layer(x, wr, b, *full, g, cfg.eps, cfg.K)
        err = float(np.abs(o64 - ref["out_f64"]).max())
        tol = 2e-2 * float(np.sqrt(np.mean(ref["out_f64"] ** 2)))
        q.put((rank, err, tol, out.tobytes()))
        dist.barrier()
        dist.destroy_process_group()
    except BaseException as e:  # report instead of hanging the parent
        q.put((rank, repr(e), None, None))
        raise


def test_two_rank_reduction_matches_the_oracle():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
    for rank, err, tol, out in res:
        assert tol is not None, err
        assert err <= tol, (rank, err, tol)
    assert res[0][3] == res[1][3]  # both ranks hold the same output bits
    assert all(p.exitcode == 0 for p in procs)


def test_shard_weights_rejects_an_uneven_split():
    from prefill_sigmoid_top_b200 import tp
    w = torch.zeros(2, 6, 256)
    with pytest.raises(ValueError):
        tp.shard_weights(w, w, torch.zeros(2, 256, 6), 0, 4)
