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


def _leaver(rank, world, port, q, steps_before_leaving, stall=0.0):
    """Rank 1 takes part in `steps_before_leaving` exchanges, then leaves
    between steps: it exits without its next all-reduce, or (stall > 0) stays
    alive that many seconds without joining it.  Rank 0 keeps stepping and
    must get an error from its next exchange, not wait for ever."""
    import datetime
    import time
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    grads = FlatGrads([(64, 24, 8)], device="cpu")
    for step in range(steps_before_leaving):
        grads.flat.fill_(float(rank + 1))
        grads.allreduce()
        assert grads.flat.eq(3.0).all()
    if rank == 1:
        q.put((rank, "left", 0.0))
        time.sleep(stall)
        q.close()
        q.join_thread()        # the message is out before the process goes
        os._exit(0)            # no destroy, no further collective: the process is gone
    t0 = time.monotonic()
    try:
        grads.allreduce()
        q.put((rank, "no error", time.monotonic() - t0))
    except Exception as e:    # gloo reports the lost peer (or the timeout) as an error
        q.put((rank, type(e).__name__, time.monotonic() - t0))
    q.close()
    q.join_thread()
    os._exit(0)


@pytest.mark.parametrize("stall", [0.0, 15.0])
def test_rank_leaving_between_steps_ends_the_next_exchange_with_an_error(stall):
    """A rank that exits (stall 0) or stops taking part (stall 15 s, three
    times the 5 s process-group timeout) between steps: the other rank's next
    gradient exchange ends with an error, the peer loss at once, the silent
    rank at the timeout."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_leaver, args=(r, 2, port, q, 2, stall)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank was still waiting after 120 s"
    results = dict((r, (what, dt)) for r, what, dt in (q.get(timeout=10) for _ in range(2)))
    assert results[1][0] == "left"
    what, dt = results[0]
    assert what != "no error", "the exchange with a departed rank completed"
    assert dt < (14.0 if stall else 4.0), f"the error came after {dt:.1f} s"
