"""Write the oracle's full-size solve results to tests/golden/<workload>.json.

Calls only the CPU oracle (``oracle/``) and the seeded input generator.  For
each workload at its full size: alternating Sinkhorn from f = g = 0 for the
workload's iteration count, then the marginal errors, the dual and primal
objectives, max C, and the potentials at a fixed seeded sample of indices.
Every number is a plain double-precision oracle result (see
"FlashSinkhorn: IO-aware EOT on GPU", Metodologia section 1, for the updates).

Usage:  python tests/golden/make_golden.py [workload ...]
Long: the 65536 x 65536, d=128 solve took 5 hours on 6 host threads.
"""
import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from log_domain_sinkhorn_updates_b200.workloads import WORKLOADS, make_problem  # noqa: E402

SAMPLE = 64


def sample_indices(count, seed):
    rng = np.random.default_rng(seed)
    idx = np.unique(np.concatenate([[0, count - 1], rng.choice(count, size=min(SAMPLE, count), replace=False)]))
    return idx


def golden(name):
    prob = make_problem(name)
    out = dict(workload=name, batch=prob.batch, n=prob.n, m=prob.m, d=prob.d, dtype=prob.dtype, eps=prob.eps,
               iters=prob.iters, seed=prob.seed, oracle_threads=oracle.num_threads(), problems=[])
    t0 = time.time()
    for k in range(prob.batch):
        X, Y, loga, logb = oracle.problem_arrays(prob, k)
        f, g = oracle.solve(X, Y, loga, logb, prob.eps, prob.iters)
        er, ec = oracle.marginal_error(X, Y, loga, logb, f, g, prob.eps)
        co = oracle.costs(X, Y, loga, logb, f, g, prob.eps)
        ri = sample_indices(prob.n, 10 + k)
        ci = sample_indices(prob.m, 20 + k)
        out["problems"].append(dict(
            err_row=er, err_col=ec, dual=co["dual"], primal=co["primal"], entropic_primal=co["entropic_primal"],
            sum_p=co["sum_p"], max_cost=co["max_cost"], min_cost=co["min_cost"],
            sum_af=float(np.exp(loga) @ f), sum_bg=float(np.exp(logb) @ g),
            f_idx=ri.tolist(), f_val=f[ri].tolist(), g_idx=ci.tolist(), g_val=g[ci].tolist()))
        print(f"{name}[{k}] err {er:.6e} {ec:.6e} dual {co['dual']:.12g} ({time.time() - t0:.0f}s)", flush=True)
    out["oracle_seconds"] = time.time() - t0
    with open(os.path.join(HERE, f"{name}.json"), "w") as fh:
        json.dump(out, fh, indent=1)


if __name__ == "__main__":
    for name in (sys.argv[1:] or list(WORKLOADS)):
        golden(name)
