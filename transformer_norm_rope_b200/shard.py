"""Token-sharded data parallelism of the hot path: one process per GPU.

Every row (token, or token x head) of the normalization and RoPE passes is independent, in the
forwards and in dx alike, so a rank runs the kernels on its own contiguous range of rows or
tokens - with the matching rows of the RoPE cos/sin tables - and exchanges no activations. The
one exchange of a training step is the sum over ranks of the weight gradients: dw (and db) of
the norms, dw_q and dw_k of the qk-norm. They are small fp32 vectors, so they live as views of
one flat bucket and a single all-reduce sums them all (NCCL over NVLink / NVSwitch between GPUs;
gloo between CPU processes).

This module holds only host logic (shard bounds, table slicing, the bucket); the kernels are the
library's.
"""
from __future__ import annotations

from typing import Dict, Iterable, Tuple

import torch
import torch.distributed as dist


def shard_bounds(n: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous range [start, stop) of n items owned by `rank` of `world`; the sizes differ
    by at most one and the ranges tile [0, n) in rank order."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError(f"bad shard request n={n} world={world} rank={rank}")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def token_shard(x: torch.Tensor, world: int, rank: int, dim: int = 1) -> torch.Tensor:
    """This rank's contiguous slice of x along the token dimension (dim 1 of [B, S, H, D],
    dim 0 of [rows, hidden] or of a [S, D/2] RoPE table), made contiguous so that the kernels
    can take it (row strides must be 16-byte aligned)."""
    s0, s1 = shard_bounds(x.shape[dim], world, rank)
    return x.narrow(dim, s0, s1 - s0).contiguous()


class GradBucket:
    """Named fp32 weight-gradient buffers as views of one flat tensor, summed over the ranks of
    a process group by one all-reduce.

    The library's backward entry points write each gradient through a plain pointer, so they
    write straight into the views; `allreduce()` then sums the whole bucket in place.
    """

    def __init__(self, sizes: Dict[str, int], device) -> None:
        if any(int(n) <= 0 for n in sizes.values()):
            raise ValueError("gradient sizes must be positive")
        total = sum(int(n) for n in sizes.values())
        # every view starts on a 16-byte boundary (4 floats): the kernels' stores need no more,
        # and the padding (zero, never written) adds nothing to the sums
        pad = lambda n: (int(n) + 3) // 4 * 4  # noqa: E731
        self.flat = torch.zeros(sum(pad(n) for n in sizes.values()) or total, dtype=torch.float32, device=device)
        self.views: Dict[str, torch.Tensor] = {}
        off = 0
        for name, n in sizes.items():
            self.views[name] = self.flat.narrow(0, off, int(n))
            off += pad(n)

    def __getitem__(self, name: str) -> torch.Tensor:
        return self.views[name]

    def names(self) -> Iterable[str]:
        return self.views.keys()

    def allreduce(self, group=None) -> None:
        """Sum the bucket over the group's ranks, in place (no-op without a process group or
        with one rank)."""
        if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
            dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group)
