"""The measurements after a solve reuse the solve's tail.

An alternating fs_solve reduces, in the epilogue of its final g-pass, the
column marginal of the pair it leaves (the plan's column sums at the stored g
are c_j = b_j exp((g_j - g~_j)/eps) with g~ the exact update), and keeps a copy
of its output potentials.  fs_marginal_err and fs_ot_cost at that pair then
skip the column-direction measure pass and share one row-direction pass, as
long as f and g still equal the solve's output bit for bit.

Checked here, through the C ABI:
* the fused results against the streamed measure passes at a bitwise copy of
  the same potentials (other buffers, so nothing is reused): the row-direction
  results (row error, dual, primal) must be identical, the column error must
  agree within 1e-3 relative plus the fp32 evaluation bound of a column LSE
  (2^-21 sum_j b_j (|g_j| + max C)/eps, as in the measure-parity test);
* a write to g after the solve turns the reuse off, and the results then equal
  a fresh measurement;
* the symmetric schedule never reuses.
"""
import numpy as np
import pytest

from helpers import device_inputs, max_cost, make_problem

pytestmark = pytest.mark.gpu


def _fs():
    import log_domain_sinkhorn_updates_b200 as fs
    return fs


@pytest.mark.parametrize("name,kw", [("middim", dict(n=1000, m=900)), ("batched", dict(batch=3, n=600, m=520)),
                                     ("highdim", dict(n=700, m=650))])
def test_fused_measurements_match_streamed_ones(cuda_device, name, kw):
    import torch
    fs = _fs()
    prob = make_problem(name, **kw)
    X, Y, a, b = device_inputs(prob)
    h = fs.fs_create(X, Y, a, b, eps=prob.eps)
    f = torch.zeros(prob.batch, prob.n, device=cuda_device)
    g = torch.zeros(prob.batch, prob.m, device=cuda_device)
    fs.fs_solve(h, f, g, prob.iters)
    er, ec = fs.fs_marginal_err(h, f, g)
    assert fs.fs_get_info(h)["last_measure_fused"] == 1
    dual, primal = fs.fs_ot_cost(h, f, g)
    assert fs.fs_get_info(h)["last_measure_fused"] == 1
    f2, g2 = f.clone(), g.clone()
    er2, ec2 = fs.fs_marginal_err(h, f2, g2)
    assert fs.fs_get_info(h)["last_measure_fused"] == 0
    dual2, primal2 = fs.fs_ot_cost(h, f2, g2)
    np.testing.assert_array_equal(er, er2)
    np.testing.assert_array_equal(dual, dual2)
    np.testing.assert_array_equal(primal, primal2)
    bw = np.ones((prob.batch, prob.m)) / prob.m if prob.b_dev is None else prob.b_dev.astype(np.float64)
    gh = g.cpu().numpy().astype(np.float64)
    tau = 2.0 ** -21 * (bw * (np.abs(gh) + max_cost(prob)[:, None])).sum(axis=1) / prob.eps
    print(f"{name}: err_col fused {ec} streamed {ec2} bound {tau}")
    assert np.all(np.abs(ec - ec2) <= 1e-3 * ec2 + tau), (ec, ec2, tau)


def test_write_after_solve_turns_reuse_off(cuda_device):
    import torch
    fs = _fs()
    prob = make_problem("middim", n=1000, m=900)
    X, Y, a, b = device_inputs(prob)
    h = fs.fs_create(X, Y, a, b, eps=prob.eps)
    f = torch.zeros(prob.batch, prob.n, device=cuda_device)
    g = torch.zeros(prob.batch, prob.m, device=cuda_device)
    fs.fs_solve(h, f, g, 20)
    g[0, 17] += 0.25
    er, ec = fs.fs_marginal_err(h, f, g)
    assert fs.fs_get_info(h)["last_measure_fused"] == 0
    dual, primal = fs.fs_ot_cost(h, f, g)
    assert fs.fs_get_info(h)["last_measure_fused"] == 0
    er2, ec2 = fs.fs_marginal_err(h, f.clone(), g.clone())
    dual2, primal2 = fs.fs_ot_cost(h, f.clone(), g.clone())
    np.testing.assert_array_equal(er, er2)
    np.testing.assert_array_equal(ec, ec2)
    np.testing.assert_array_equal(dual, dual2)
    np.testing.assert_array_equal(primal, primal2)


def test_symmetric_schedule_does_not_reuse(cuda_device):
    import torch
    fs = _fs()
    prob = make_problem("tiny")
    X, Y, a, b = device_inputs(prob)
    h = fs.fs_create(X, Y, a, b, eps=prob.eps)
    f = torch.zeros(prob.batch, prob.n, device=cuda_device)
    g = torch.zeros(prob.batch, prob.m, device=cuda_device)
    fs.fs_solve(h, f, g, 10, schedule="symmetric")
    fs.fs_marginal_err(h, f, g)
    assert fs.fs_get_info(h)["last_measure_fused"] == 0
