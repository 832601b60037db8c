"""Write the oracle's full-size solve results to tests/golden/<workload>.json.

Calls only the CPU oracle (``oracle/``) and the seeded input generator.  For
each workload at its full size: alternating Sinkhorn from f = g = 0 for the
workload's iteration count, then the marginal errors, the dual and primal
objectives, max C, and the potentials at a fixed seeded sample of indices.
Every number is a plain double-precision oracle result (see
"FlashSinkhorn: IO-aware EOT on GPU", Metodologia section 1, for the updates).

It also stores the fp32 floor of the marginal error, ``tau_f32``: how far the
plan's marginals move, in L1, when the oracle's own potentials are rounded to
float32, sum_i |r_i(fl f, fl g) - r_i(f, g)| + sum_j |c_j(fl f, fl g) - c_j(f, g)|.
By the triangle inequality it bounds the change of the marginal L1 error that
the rounding alone causes, so no float32 representation of the solution can be
held closer; a float32 solver's marginal error is compared with the oracle's
within 1e-3 relative plus this floor.  ``err_row_f32`` / ``err_col_f32`` are
the oracle's marginal errors at the rounded potentials.

Usage:  python tests/golden/make_golden.py [--potentials-dir DIR] [workload ...]
--potentials-dir also saves the full double-precision potentials there
(``<workload>.npz``, arrays f and g of shape [batch][n] and [batch][m]); they
are not part of the stored expectations.
Long: the 65536 x 65536, d=128 workload (the solve, its measurements and the
fp32 floor) took 18000 s on 6 host threads without the floor, 24900 s with it.
"""
import argparse
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


def fp32_floor(X, Y, loga, logb, f, g, eps):
    """(tau, err_row, err_col) at the potentials rounded to float32: tau is the L1 shift of
    both marginals that the rounding causes, err_* the marginal errors there."""
    f32 = f.astype(np.float32).astype(np.float64)
    g32 = g.astype(np.float32).astype(np.float64)
    r, c = oracle.marginals(X, Y, loga, logb, f, g, eps)
    r32, c32 = oracle.marginals(X, Y, loga, logb, f32, g32, eps)
    tau = float(np.abs(r32 - r).sum() + np.abs(c32 - c).sum())
    return tau, float(np.abs(r32 - np.exp(loga)).sum()), float(np.abs(c32 - np.exp(logb)).sum())


def golden(name, potentials_dir=None):
    prob = make_problem(name)
    out = dict(workload=name, batch=prob.batch, n=prob.n, m=prob.m, d=prob.d, dtype=prob.dtype, eps=prob.eps,
               iters=prob.iters, seed=prob.seed, oracle_threads=oracle.num_threads(), problems=[])
    t0 = time.time()
    fs, gs = [], []
    for k in range(prob.batch):
        X, Y, loga, logb = oracle.problem_arrays(prob, k)
        f, g = oracle.solve(X, Y, loga, logb, prob.eps, prob.iters)
        er, ec = oracle.marginal_error(X, Y, loga, logb, f, g, prob.eps)
        tau, er32, ec32 = fp32_floor(X, Y, loga, logb, f, g, prob.eps)
        co = oracle.costs(X, Y, loga, logb, f, g, prob.eps)
        ri = sample_indices(prob.n, 10 + k)
        ci = sample_indices(prob.m, 20 + k)
        out["problems"].append(dict(
            err_row=er, err_col=ec, tau_f32=tau, err_row_f32=er32, err_col_f32=ec32, dual=co["dual"], primal=co["primal"],
            entropic_primal=co["entropic_primal"], sum_p=co["sum_p"], max_cost=co["max_cost"],
            min_cost=co["min_cost"], sum_af=float(np.exp(loga) @ f), sum_bg=float(np.exp(logb) @ g),
            f_idx=ri.tolist(), f_val=f[ri].tolist(), g_idx=ci.tolist(), g_val=g[ci].tolist()))
        fs.append(f)
        gs.append(g)
        print(f"{name}[{k}] err {er:.6e} {ec:.6e} fp32 floor {tau:.3e} dual {co['dual']:.12g} "
              f"({time.time() - t0:.0f}s)", flush=True)
    out["oracle_seconds"] = time.time() - t0
    with open(os.path.join(HERE, f"{name}.json"), "w") as fh:
        json.dump(out, fh, indent=1)
    if potentials_dir:
        os.makedirs(potentials_dir, exist_ok=True)
        np.savez(os.path.join(potentials_dir, f"{name}.npz"), f=np.stack(fs), g=np.stack(gs))


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--potentials-dir", default=None)
    ap.add_argument("workloads", nargs="*")
    args = ap.parse_args()
    for name in (args.workloads or list(WORKLOADS)):
        golden(name, args.potentials_dir)
