"""Data-parallel path on CPU: two gloo ranks, the oracle as the compute.

Each rank takes a contiguous token block of one global batch; forward and dx
rows need no exchange, and summing the per-rank dW/db with an all-reduce
reproduces the gradients of the whole batch.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from group_circulant_linear_b200 import dp, inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, T, Cp, Dp, N, out):
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = inputs.make_inputs(T, Cp, Dp, N, "f32", seed=5)
        a, b = dp.shard_range(N, rank, world)
        y = oracle.forward(inp["x"][a:b], inp["W"], inp["b"])
        dx = oracle.backward_dx(inp["gy"][a:b], inp["W"])
        dW, db = oracle.backward_dw(inp["x"][a:b], inp["gy"][a:b], T, Cp, Dp)
        g = [torch.from_numpy(dW.copy()), torch.from_numpy(db.copy())]
        dp.allreduce_grads(g)
        out[rank] = (a, b, y, dx, g[0].numpy(), g[1].numpy())
    finally:
        torch.distributed.destroy_process_group()


def test_shard_range_partitions():
    for n in (0, 1, 7, 128, 12608):
        for w in (1, 2, 3, 8):
            got = [dp.shard_range(n, r, w) for r in range(w)]
            assert got[0][0] == 0 and got[-1][1] == n
            assert all(got[i][1] == got[i + 1][0] for i in range(w - 1))
            sizes = [e - s for s, e in got]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        dp.shard_range(4, 2, 2)


def test_two_rank_gradients_match_whole_batch():
    import oracle
    oracle.build()
    T, Cp, Dp, N = 4, 3, 2, 37
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    try:
        out = manager.dict()
        mp.spawn(_worker, args=(world, port, T, Cp, Dp, N, out), nprocs=world, join=True)
        out = dict(out)
    finally:
        manager.shutdown()
    inp = inputs.make_inputs(T, Cp, Dp, N, "f32", seed=5)
    y = oracle.forward(inp["x"], inp["W"], inp["b"])
    dx = oracle.backward_dx(inp["gy"], inp["W"])
    dW, db = oracle.backward_dw(inp["x"], inp["gy"], T, Cp, Dp)
    for r in range(world):
        a, b, yr, dxr, dWr, dbr = out[r]
        np.testing.assert_allclose(yr, y[a:b], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dxr, dx[a:b], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dWr, dW, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dbr, db, rtol=1e-12, atol=1e-12)
