"""Multi-rank host logic on CPU (gloo, world size 2): the weak-scaling value
uses the slowest rank, and a batch split by rows over ranks reproduces the
unsplit scan (checked with the oracle, since this runs without a GPU)."""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist

    import oracle
    from test_sequence_layers_02_b200.workloads import make_inputs

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # slowest rank decides
        value, t_max = bench.weak_scaling_value(1000.0, 1.0 + rank, world, dist)
        out[f"value{rank}"] = value
        out[f"tmax{rank}"] = t_max
        # each rank scans its own rows of one batch; gather and compare
        B, H, T, d, b = 5, 2, 37, 16, 8
        inp = make_inputs(B, H, T, d, seed=9, random_affine=True, mask_p=0.5, b=b)
        r0, r1 = bench.shard_rows(B, world, rank)
        f = lambda a: np.asarray(a, np.float64)
        o, W = oracle.forward(f(inp["q"][r0:r1]), f(inp["k"][r0:r1]), f(inp["v"][r0:r1]),
                              f(inp["eta_logit"][r0:r1]), f(inp["gate_logit"][r0:r1]),
                              f(inp["W0"][r0:r1]), f(inp["gamma"]), f(inp["beta"]), eps=1e-6,
                              mode=2, b=b, mask=inp["mask"][r0:r1])
        parts = [None] * world
        dist.all_gather_object(parts, (r0, r1, o, W))
        if rank == 0:
            parts.sort(key=lambda x: x[0])
            o_all = np.concatenate([p[2] for p in parts], axis=0)
            W_all = np.concatenate([p[3] for p in parts], axis=0)
            ro, rW = oracle.forward(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["eta_logit"]),
                                    f(inp["gate_logit"]), f(inp["W0"]), f(inp["gamma"]),
                                    f(inp["beta"]), eps=1e-6, mode=2, b=b, mask=inp["mask"])
            out["rows"] = [(p[0], p[1]) for p in parts]
            out["same_o"] = bool(np.array_equal(o_all, ro))
            out["same_W"] = bool(np.array_equal(W_all, rW))
    finally:
        dist.destroy_process_group()


def test_shard_rows_covers_batch():
    for B in (1, 2, 5, 16):
        for world in (1, 2, 3, 4, 8):
            spans = [bench.shard_rows(B, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == B
            for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                assert a1 == b0 and a0 <= a1
            sizes = [s1 - s0 for s0, s1 in spans]
            assert max(sizes) - min(sizes) <= 1


@pytest.mark.timeout(300)
def test_two_ranks_gloo():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res["tmax0"] == res["tmax1"] == 2.0
    assert res["value0"] == res["value1"] == pytest.approx(1000.0 * 2 / 2.0)
    assert res["rows"] == [(0, 3), (3, 5)]
    assert res["same_o"] and res["same_W"]
