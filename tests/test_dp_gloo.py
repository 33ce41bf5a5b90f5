"""Multi-process (world size 2, gloo, CPU) checks of the data-parallel host
logic: token sharding and the single flat all-reduce of the adapter
gradients, whose result must equal the gradient of the unsharded batch."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_nf4_quantized_02_b200.dp import FlatGrads, shard_rows
from oracle import qlora_linear


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        g = np.random.default_rng(0)   # every rank draws the same full batch
        M, K, N, r, s = 37, 64, 24, 8, 0.5
        X = g.standard_normal((M, K))
        W = g.standard_normal((N, K)) * 0.02
        L1 = g.standard_normal((K, r)) / 8
        L2 = g.standard_normal((r, N)) * 0.1
        dY = g.standard_normal((M, N))
        a, b = shard_rows(M, rank, world)
        _, dl1, dl2 = qlora_linear.backward(dY[a:b], X[a:b], W, L1, L2, s)
        grads = FlatGrads([(K, N, r)], device="cpu", dtype=torch.float64)
        grads.views[0][0].copy_(torch.from_numpy(dl1))
        grads.views[0][1].copy_(torch.from_numpy(dl2))
        grads.allreduce()
        _, full1, full2 = qlora_linear.backward(dY, X, W, L1, L2, s)
        ok = (np.allclose(grads.views[0][0].numpy(), full1, atol=1e-12, rtol=1e-12) and
              np.allclose(grads.views[0][1].numpy(), full2, atol=1e-12, rtol=1e-12))
        q.put((rank, ok, b - a))
    finally:
        dist.destroy_process_group()


def test_shard_rows_partition():
    for total in (0, 1, 7, 8192, 8193):
        for world in (1, 2, 3, 8):
            spans = [shard_rows(total, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            assert max(b - a for a, b in spans) - min(b - a for a, b in spans) <= 1


def test_flat_grad_views_share_storage():
    fg = FlatGrads([(64, 24, 8), (128, 16, 4)], device="cpu")
    fg.views[1][1].fill_(3.0)
    assert fg.flat[-16 * 4:].eq(3.0).all() and fg.flat[:-16 * 4].eq(0).all()
    assert fg.views[0][0].shape == (64, 8) and fg.views[1][1].shape == (4, 16)


def test_two_rank_allreduce_matches_full_batch():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    results = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[0] for r in results] == [0, 1]
    assert all(r[1] for r in results), results
    assert sum(r[2] for r in results) == 37
    assert all(p.exitcode == 0 for p in procs)
