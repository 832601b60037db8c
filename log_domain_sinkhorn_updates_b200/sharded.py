"""One problem's alternating Sinkhorn solve sharded by rows over G ranks.

The f-update of row i needs all of Y and g but nothing of the other rows
("FlashSinkhorn: IO-aware EOT on GPU", Metodologia section 1: a row-wise LSE),
and the g-update of column j likewise needs all of X and f.  So rank r owns

  * the rows  [r s_n, min(n, (r + 1) s_n)) of X for the f-update, and
  * the rows  [r s_m, min(m, (r + 1) s_m)) of Y for the g-update,

with s_n = ceil(n / G) and s_m = ceil(m / G).  Every half-iteration updates the
owned slice of one potential on the rank's GPU, then all-gathers the slices
(NCCL over NVLink under torch.distributed), so each rank holds the whole
potential for the next half-iteration.  Each rank's share of the n x m work is
1/G; the exchange is n + m floats per iteration.

The per-rank compute is an object with two methods, ``update_f(g_full, f_out)``
and ``update_g(f_full, g_out)``.  The library's own is ``FsShard``: two handles
per rank, (X_r, Y) for the f-update and (X, Y_r) for the g-update.  Weights a
handle does not use (a for the f-update, b for the g-update) are left uniform,
which changes nothing in its update.  The gather is a callable too, so that
one process can also run every shard of a problem (``LocalGather``); that is
how the sharded arithmetic is checked on a single device.
"""
from __future__ import annotations

import math
from typing import Callable, List, Sequence

__all__ = ["shard_ranges", "FsShard", "LocalGather", "DistGather", "solve_row_sharded"]


def shard_ranges(count: int, world: int):
    """[(start, stop)] of the rows each of `world` ranks owns: contiguous, ceil(count / world)
    per rank, the last ones shorter (or empty when world does not divide the padding)."""
    if count < 1 or world < 1:
        raise ValueError("count and world must be >= 1")
    size = math.ceil(count / world)
    return [(min(count, r * size), min(count, (r + 1) * size)) for r in range(world)], size


class FsShard:
    """One rank's share on its GPU: the f-update of its rows of X and the g-update of its rows
    of Y, each through a handle of the library (X, Y: [batch, n|m, d] CUDA tensors)."""

    def __init__(self, X, Y, a, b, eps, rows, cols, prec="auto"):
        from . import binding as fs
        self._fs = fs
        r0, r1 = rows
        c0, c1 = cols
        self.rows, self.cols = rows, cols
        self.hf = fs.fs_create(X[:, r0:r1].contiguous(), Y, None, b, eps=eps, prec=prec) if r1 > r0 else None
        self.hg = fs.fs_create(X, Y[:, c0:c1].contiguous(), a, None, eps=eps, prec=prec) if c1 > c0 else None

    def update_f(self, g_full, f_out):
        if self.hf is not None:
            self._fs.fs_update_f(self.hf, g_full, f_out)

    def update_g(self, f_full, g_out):
        if self.hg is not None:
            self._fs.fs_update_g(self.hg, f_full, g_out)

    def close(self):
        for h in (self.hf, self.hg):
            if h is not None:
                self._fs.fs_destroy(h)
        self.hf = self.hg = None


class LocalGather:
    """All shards in this process: the gather concatenates their slices."""

    def __call__(self, slices: Sequence, out):
        import torch
        torch.cat(list(slices), dim=1, out=out)


class DistGather:
    """One shard per rank: all_gather_into_tensor over the process group (NCCL on GPUs, gloo on
    CPUs), then the [world, batch, size] result laid out as [batch, world * size]."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)

    def __call__(self, slices: Sequence, out):
        import torch
        (mine,) = slices
        batch, size = mine.shape
        buf = torch.empty(self.world * batch * size, dtype=mine.dtype, device=mine.device)
        self.dist.all_gather_into_tensor(buf, mine.reshape(-1).contiguous(), group=self.group)
        out.copy_(buf.view(self.world, batch, size).permute(1, 0, 2).reshape(batch, self.world * size))


def solve_row_sharded(shards: List, gather: Callable, n: int, m: int, batch: int, world: int, iters: int,
                      dtype=None, device=None, g0=None):
    """`iters` alternating iterations (f from g, then g from the new f) from g0 (default 0),
    computed by `shards` (the shards this process runs: one under torch.distributed, all of
    them with LocalGather) and exchanged by `gather`.  Returns the whole f [batch, n] and
    g [batch, m] on every rank."""
    import torch
    _, sn = shard_ranges(n, world)
    _, sm = shard_ranges(m, world)
    dtype = dtype or torch.float32
    f_full = torch.zeros(batch, world * sn, dtype=dtype, device=device)
    g_full = torch.zeros(batch, world * sm, dtype=dtype, device=device)
    if g0 is not None:
        g_full[:, :m] = g0
    f_loc = [torch.zeros(batch, sn, dtype=dtype, device=device) for _ in shards]
    g_loc = [torch.zeros(batch, sm, dtype=dtype, device=device) for _ in shards]
    for _ in range(iters):
        g_in = g_full[:, :m].contiguous()
        for sh, fl in zip(shards, f_loc):
            r0, r1 = sh.rows
            if r1 > r0:
                out = fl[:, : r1 - r0]
                tmp = torch.empty(batch, r1 - r0, dtype=dtype, device=device)
                sh.update_f(g_in, tmp)
                out.copy_(tmp)
        gather(f_loc, f_full)
        f_in = f_full[:, :n].contiguous()
        for sh, gl in zip(shards, g_loc):
            c0, c1 = sh.cols
            if c1 > c0:
                tmp = torch.empty(batch, c1 - c0, dtype=dtype, device=device)
                sh.update_g(f_in, tmp)
                gl[:, : c1 - c0].copy_(tmp)
        gather(g_loc, g_full)
    return f_full[:, :n].contiguous(), g_full[:, :m].contiguous()
