"""The row-sharded solve of one problem (log_domain_sinkhorn_updates_b200.sharded).

The orchestration (which rows each rank owns, the two half-iterations, the
all-gather of the owned slices) is checked on CPU with the oracle as the
per-rank compute: world_size-2 gloo ranks must give the single-process result
bit for bit, since every row's update is the same arithmetic wherever it runs
("FlashSinkhorn: IO-aware EOT on GPU", Metodologia section 1: the updates are
row-wise LSEs).  On a GPU, the library's shards (two handles per share) run
every share of a problem in one process, gathered locally, against the
oracle's own solve.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from helpers import make_problem

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class OracleShard:
    """A rank's share computed by the oracle (test infrastructure): f on rows [r0, r1), g on
    columns [c0, c1), one problem, float64 tensors on the CPU."""

    def __init__(self, Xo, Yo, loga, logb, eps, rows, cols):
        self.X, self.Y, self.loga, self.logb, self.eps = Xo, Yo, loga, logb, eps
        self.rows, self.cols = rows, cols

    def update_f(self, g_full, f_out):
        r0, r1 = self.rows
        f = oracle.update_f_rows(np.arange(r0, r1), self.X, self.Y, self.logb, g_full[0].numpy(), self.eps)
        f_out[0] = torch.from_numpy(f)

    def update_g(self, f_full, g_out):
        c0, c1 = self.cols
        g = oracle.update_f_rows(np.arange(c0, c1), self.Y, self.X, self.loga, f_full[0].numpy(), self.eps)
        g_out[0] = torch.from_numpy(g)


def _problem():
    prob = make_problem("middim", n=301, m=257, d=8)  # ragged: neither size splits evenly
    return prob, oracle.problem_arrays(prob)


def _solve(world, rank=None, gather=None, iters=6):
    from log_domain_sinkhorn_updates_b200.sharded import LocalGather, shard_ranges, solve_row_sharded
    prob, (Xo, Yo, loga, logb) = _problem()
    rr, _ = shard_ranges(prob.n, world)
    cc, _ = shard_ranges(prob.m, world)
    ranks = range(world) if rank is None else [rank]
    shards = [OracleShard(Xo, Yo, loga, logb, prob.eps, rr[r], cc[r]) for r in ranks]
    return solve_row_sharded(shards, gather or LocalGather(), prob.n, prob.m, 1, world, iters, dtype=torch.float64)


def test_shard_ranges_cover_every_row_once():
    from log_domain_sinkhorn_updates_b200.sharded import shard_ranges
    for count in (1, 5, 10, 301, 4096):
        for world in (1, 2, 3, 4, 8):
            ranges, size = shard_ranges(count, world)
            assert size == -(-count // world)
            covered = [i for a, b in ranges for i in range(a, b)]
            assert covered == list(range(count))
            assert all(a == min(count, r * size) for r, (a, _) in enumerate(ranges))


def test_local_shards_match_one_shard_bit_for_bit():
    f1, g1 = _solve(1)
    f3, g3 = _solve(3)
    assert torch.equal(f1, f3) and torch.equal(g1, g3)
    prob, (Xo, Yo, loga, logb) = _problem()
    fo, go = oracle.solve(Xo, Yo, loga, logb, prob.eps, 6)
    assert np.abs(f1.numpy()[0] - fo).max() <= 1e-12 * np.abs(fo).max()
    assert np.abs(g1.numpy()[0] - go).max() <= 1e-12 * np.abs(go).max()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from log_domain_sinkhorn_updates_b200.sharded import DistGather
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    f, g = _solve(world, rank=rank, gather=DistGather())
    out.put((rank, f.numpy().tobytes(), g.numpy().tobytes()))
    dist.barrier()
    dist.destroy_process_group()


def test_gloo_ranks_match_one_process_bit_for_bit():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    f1, g1 = _solve(1)
    for _, fb, gb in res:  # every rank holds the whole potentials
        assert fb == f1.numpy().tobytes() and gb == g1.numpy().tobytes()


@pytest.mark.gpu
@pytest.mark.parametrize("name,kw", [("middim", dict(n=1000, m=900)), ("highdim", dict(n=700, m=650))])
def test_fs_shards_on_one_device_against_the_oracle(cuda_device, name, kw):
    """Three shares of one problem, each two library handles, gathered locally: the potentials
    after the recipe's iterations against the oracle's own solve, after removing the common
    gauge constant, within the single-update bar 1e-4 max C (the bar the unsharded solve meets)."""
    from helpers import device_inputs, max_cost
    from log_domain_sinkhorn_updates_b200.sharded import FsShard, LocalGather, shard_ranges, solve_row_sharded
    prob = make_problem(name, **kw)
    X, Y, a, b = device_inputs(prob)
    world = 3
    rr, _ = shard_ranges(prob.n, world)
    cc, _ = shard_ranges(prob.m, world)
    shards = [FsShard(X, Y, a, b, prob.eps, rr[r], cc[r]) for r in range(world)]
    f, g = solve_row_sharded(shards, LocalGather(), prob.n, prob.m, 1, world, prob.iters, device=cuda_device)
    torch.cuda.synchronize()
    for sh in shards:
        sh.close()
    Xo, Yo, loga, logb = oracle.problem_arrays(prob)
    fo, go = oracle.solve(Xo, Yo, loga, logb, prob.eps, prob.iters)
    fg, gg = f.cpu().numpy()[0].astype(np.float64), g.cpu().numpy()[0].astype(np.float64)
    c = np.exp(loga) @ (fg - fo)
    err = max(np.abs(fg - fo - c).max(), np.abs(gg - go + c).max())
    bar = 1e-4 * max_cost(prob)[0]
    print(f"{name}: sharded gauge-fixed potential error {err:.3e} (bar {bar:.3e})")
    assert err <= bar
