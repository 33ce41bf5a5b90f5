"""Data-parallel plumbing for QLoRA adapter training (host side).

Each rank holds the same NF4 + DQ frozen weights and LoRA factors and runs
the linear forward/backward on its own tokens.  The only exchange per step is
the sum of the adapter gradients dL1, dL2 over ranks.  They live as views of
one flat fp32 buffer so the exchange is one all-reduce over NCCL (NVLink /
NVSwitch on a B200 node; gloo on CPU in the tests).
"""

from __future__ import annotations

import torch
import torch.distributed as dist


class FlatGrads:
    """dL1 [K, r] and dL2 [r, N] of several linears as views of one buffer."""

    def __init__(self, shapes, device, dtype=torch.float32):
        # shapes: list of (k_in, n_out, r)
        sizes = [k * r + r * n for k, n, r in shapes]
        self.flat = torch.zeros(sum(sizes), dtype=dtype, device=device)
        self.views = []
        off = 0
        for (k, n, r), size in zip(shapes, sizes):
            dl1 = self.flat[off:off + k * r].view(k, r)
            dl2 = self.flat[off + k * r:off + size].view(r, n)
            self.views.append((dl1, dl2))
            off += size

    def allreduce(self, group=None, average: bool = False) -> None:
        """Sum (or average) the gradients over the ranks of `group` in place."""
        if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
            return
        dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group)
        if average:
            self.flat.div_(dist.get_world_size(group))


def shard_rows(total: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous [start, stop) of `total` token rows owned by `rank` (sizes differ by at most 1)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)
