"""Parity at the full workload sizes, in the launch configuration the benchmark times.

Two kinds of check:

* one f-update and one g-update on the full problem, compared at a seeded
  sample of rows (columns) that the oracle computes one by one
  ("FlashSinkhorn: IO-aware EOT on GPU", Metodologia section 1, the two
  log-domain updates);
* a full alternating solve from f = g = 0 with the workload's iteration count,
  compared with the oracle's own full-size solve stored in tests/golden/ (written
  by tests/golden/make_golden.py, which calls only the oracle).

Tolerances:

* Single updates use the same tolerance as at small sizes, 1e-4 * max C / 4.
  Here max C is taken over the sampled rows, which is stricter than the whole
  problem's max C.
* Solves compare the gauge-invariant results (dual and primal objective, within
  1e-3 relative) and the sampled potentials after removing the common gauge
  constant (within 1e-3 * max C).
* The marginal error is compared within 1e-3 relative, plus twice the
  oracle's own fp32 floor ``tau_f32`` stored beside it: how far the plan's
  marginals move, in L1, when the oracle's potentials are rounded to float32
  (once for the rounding of the stored potential, once for the float32
  arguments of the LSE that produced it; see test_gpu_parity.oracle_fp32_floor).
"""
import json
import os

import numpy as np
import pytest

import oracle
from helpers import device_inputs, smooth_potential
from log_domain_sinkhorn_updates_b200.workloads import WORKLOADS, make_problem

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
SAMPLE = 256


def _fs():
    import log_domain_sinkhorn_updates_b200 as fs
    return fs


def _problems_checked(batch):
    return sorted({0, batch // 2, batch - 1})


def _sample_max_cost(Xs, Y):
    """max over the sampled rows of max_j C_ij (oracle, double)."""
    _, _, cmax = oracle.minplus_bounds(Xs, Y, np.zeros(Y.shape[0]), np.zeros(Y.shape[0]), 1.0)
    return float(cmax.max())


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_full_size_updates_sampled(cuda_device, name):
    import torch
    fs = _fs()
    prob = make_problem(name)
    X, Y, a_d, b_d = device_inputs(prob)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps)
    rng = np.random.default_rng(4242)
    g_in = np.stack([smooth_potential(rng, prob.m, 0.5) for _ in range(prob.batch)])
    f_in = np.stack([smooth_potential(rng, prob.n, 0.5) for _ in range(prob.batch)])
    f = torch.empty(prob.batch, prob.n, device=cuda_device)
    g = torch.empty(prob.batch, prob.m, device=cuda_device)
    fs.fs_update_f(h, torch.from_numpy(g_in).to(cuda_device), f)
    fs.fs_update_g(h, torch.from_numpy(f_in).to(cuda_device), g)
    fs.fs_sync(h)
    fg, gg = f.cpu().numpy(), g.cpu().numpy()
    for k in _problems_checked(prob.batch):
        Xo, Yo, loga, logb = oracle.problem_arrays(prob, k)
        rows = np.unique(np.concatenate([[0, prob.n - 1], rng.choice(prob.n, SAMPLE, replace=False)]))
        cols = np.unique(np.concatenate([[0, prob.m - 1], rng.choice(prob.m, SAMPLE, replace=False)]))
        fo = oracle.update_f_rows(rows, Xo, Yo, logb, g_in[k].astype(np.float64), prob.eps)
        # the g-update is the f-update with the two sides exchanged
        go = oracle.update_f_rows(cols, Yo, Xo, loga, f_in[k].astype(np.float64), prob.eps)
        tol_f = 1e-4 * _sample_max_cost(Xo[rows], Yo) / 4
        tol_g = 1e-4 * _sample_max_cost(Yo[cols], Xo) / 4
        ef = np.abs(fg[k][rows] - fo).max()
        eg = np.abs(gg[k][cols] - go).max()
        print(f"{name}[{k}] max|df|={ef:.3e} (tol {tol_f:.3e})  max|dg|={eg:.3e} (tol {tol_g:.3e})")
        assert ef <= tol_f, (name, k, ef, tol_f)
        assert eg <= tol_g, (name, k, eg, tol_g)


def _golden(name):
    path = os.path.join(GOLDEN, f"{name}.json")
    if not os.path.exists(path):
        pytest.skip(f"no stored oracle solve for {name}")
    with open(path) as fh:
        return json.load(fh)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_full_size_solve_against_stored_oracle(cuda_device, name):
    import torch
    fs = _fs()
    gold = _golden(name)
    prob = make_problem(name)
    assert (gold["n"], gold["m"], gold["d"], gold["batch"], gold["iters"], gold["seed"]) == (
        prob.n, prob.m, prob.d, prob.batch, prob.iters, prob.seed)
    X, Y, a_d, b_d = device_inputs(prob)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps)
    f = torch.zeros(prob.batch, prob.n, device=cuda_device)
    g = torch.zeros(prob.batch, prob.m, device=cuda_device)
    fs.fs_solve(h, f, g, prob.iters)
    er, ec = fs.fs_marginal_err(h, f, g)
    dual, primal = fs.fs_ot_cost(h, f, g)
    fg, gg = f.cpu().numpy().astype(np.float64), g.cpu().numpy().astype(np.float64)
    for k, gp in enumerate(gold["problems"]):
        fi, gi = np.array(gp["f_idx"]), np.array(gp["g_idx"])
        df = fg[k][fi] - np.array(gp["f_val"])
        dg = gg[k][gi] - np.array(gp["g_val"])
        c = 0.5 * (np.median(df) - np.median(dg))  # (f + c, g - c) is the same plan
        pot_err = max(np.abs(df - c).max(), np.abs(dg + c).max())
        e_gpu, e_o = er[k] + ec[k], gp["err_row"] + gp["err_col"]
        assert "tau_f32" in gp, f"{name}: stored solve predates the fp32 floor; rerun tests/golden/make_golden.py"
        floor = 2.0 * gp["tau_f32"]
        if k < 3 or k == len(gold["problems"]) - 1:
            print(f"{name}[{k}] dual {dual[k]:.9g} vs {gp['dual']:.9g}  primal {primal[k]:.9g} vs "
                  f"{gp['primal']:.9g}  err {e_gpu:.3e} vs {e_o:.3e} (floor {floor:.1e})  "
                  f"gauge {c:.2e} pot {pot_err:.3e} (tol {1e-3 * gp['max_cost']:.3e})")
        assert abs(dual[k] - gp["dual"]) <= 1e-3 * abs(gp["dual"]), (name, k, dual[k], gp["dual"])
        assert abs(primal[k] - gp["primal"]) <= 1e-3 * abs(gp["primal"]), (name, k, primal[k], gp["primal"])
        assert abs(e_gpu - e_o) <= 1e-3 * e_o + floor, (name, k, e_gpu, e_o, floor)
        assert pot_err <= 1e-3 * gp["max_cost"], (name, k, pot_err, gp["max_cost"])


@pytest.mark.parametrize("name", ["highdim", "middim", "cloud3d"])
def test_full_size_transport_sampled(cuda_device, name):
    """The barycentric map on the full workload (the configuration `bench.py --op
    transport` times), checked at sampled rows that the oracle computes one by one
    from the plan's definition.

    Potentials: a seeded smooth g, and f = the oracle's f-update of g.  The f-update
    makes every row sum r_i equal a_i, as at a solution.  Arbitrary potentials at
    these eps would put whole plan rows below the fp32 range; a solution never
    does.  On highdim the full oracle pass would take minutes, and its costs are
    small enough against eps that a seeded smooth f stays in range."""
    import torch
    fs = _fs()
    prob = make_problem(name)
    X, Y, a_d, b_d = device_inputs(prob)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps)
    rng = np.random.default_rng(777)
    g_in = smooth_potential(rng, prob.m, 0.05)[None]
    if name == "highdim":
        f_in = smooth_potential(rng, prob.n, 0.05)[None]
    else:
        Xo, Yo, _, logb = oracle.problem_arrays(prob, 0)
        f_in = oracle.update_f(Xo, Yo, logb, g_in[0].astype(np.float64), prob.eps).astype(np.float32)[None]
    fd, gd = torch.from_numpy(f_in).to(cuda_device), torch.from_numpy(g_in).to(cuda_device)
    T = torch.empty(1, prob.n, prob.d, device=cuda_device)
    fs.fs_barycentric_map(h, fd, gd, Y, T)
    fs.fs_sync(h)
    assert fs.fs_get_info(h)["last_apply_path"] in ("tc_q2", "tc_2s", "tc", "tc_pair")  # the kernel the bench times
    T = T.cpu().numpy()[0]
    Xo, Yo, loga, logb = oracle.problem_arrays(prob, 0)
    # 64 rows anywhere, 16 of the last eighth (at highdim the row blocks split over their columns)
    rows = np.unique(np.concatenate([[0, prob.n - 1], rng.choice(prob.n, 64, replace=False),
                                     rng.choice(np.arange(prob.n * 7 // 8, prob.n), 16, replace=False)]))
    fk, gk = f_in[0].astype(np.float64), g_in[0].astype(np.float64)
    out, r = oracle.transport_apply(Xo[rows], Yo, loga[rows], logb, fk[rows], gk, prob.eps, Yo)
    absw, _ = oracle.transport_apply(Xo[rows], Yo, loga[rows], logb, fk[rows], gk, prob.eps, np.abs(Yo))
    To = out / r[:, None]
    # relative error bound of the plan entries (see tests/test_gpu_transport.py), 2^-14 for the
    # tensor-core splits; T = (P Y)/r carries it twice
    xs_t = 0.5 * (Xo.mean(0) + Yo.mean(0))
    xs, ys = Xo[rows] - xs_t, Yo - xs_t
    LOG2E = 1.0 / np.log(2.0)
    alpha = loga[rows] * LOG2E + (fk[rows] - (xs ** 2).sum(1)) * LOG2E / prob.eps
    beta = logb * LOG2E + (gk - (ys ** 2).sum(1)) * LOG2E / prob.eps
    M = np.abs(alpha) + np.abs(beta).max() + (2 * prob.d + 2) * 2 * np.sqrt((xs ** 2).sum(1)) * \
        np.sqrt((ys ** 2).sum(1)).max() * LOG2E / prob.eps
    rel = np.log(2.0) * 2.0 ** -23 * M + 2.0 ** -21 + prob.m * 2.0 ** -24 + 2.0 ** -14
    err = (np.abs(T[rows] - To) / (2 * rel[:, None] * absw / r[:, None] + 1e-6 * np.abs(To))).max()
    print(f"{name} full-size barycentric map, sampled rows: worst err / bound = {err:.3f}")
    assert err <= 1.0


@pytest.mark.parametrize("name", ["highdim", "middim", "cloud3d"])
def test_full_size_one_column_sampled(cuda_device, name):
    """A one-column transport application on the full workload: the streamed LSE
    pass that weights column j by v_j (the form the HVP's conjugate gradient
    runs, with the bias inside the S product), checked at sampled rows that the
    oracle computes one by one.  Potentials as in the barycentric-map test; the
    bound is the transport bound without the bf16 split term (fp32 sums, no P~
    split), as at small sizes."""
    import torch
    fs = _fs()
    prob = make_problem(name)
    X, Y, a_d, b_d = device_inputs(prob)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps)
    rng = np.random.default_rng(778)
    g_in = smooth_potential(rng, prob.m, 0.05)[None]
    if name == "highdim":
        f_in = smooth_potential(rng, prob.n, 0.05)[None]
    else:
        Xo, Yo, _, logb = oracle.problem_arrays(prob, 0)
        f_in = oracle.update_f(Xo, Yo, logb, g_in[0].astype(np.float64), prob.eps).astype(np.float32)[None]
    v = rng.standard_normal((1, prob.m, 1)).astype(np.float32)
    fd, gd, vd = (torch.from_numpy(x).to(cuda_device) for x in (f_in, g_in, v))
    out = torch.empty(1, prob.n, 1, device=cuda_device)
    r = torch.empty(1, prob.n, device=cuda_device)
    fs.fs_transport_apply(h, fd, gd, vd, out, r)
    fs.fs_sync(h)
    assert fs.fs_get_info(h)["last_apply_path"] == "lse_vec"
    out, r = out.cpu().numpy()[0, :, 0], r.cpu().numpy()[0]
    Xo, Yo, loga, logb = oracle.problem_arrays(prob, 0)
    rows = np.unique(np.concatenate([[0, prob.n - 1], rng.choice(prob.n, 64, replace=False)]))
    fk, gk = f_in[0].astype(np.float64), g_in[0].astype(np.float64)
    oo, ro = oracle.transport_apply(Xo[rows], Yo, loga[rows], logb, fk[rows], gk, prob.eps, v[0].astype(np.float64))
    absw, _ = oracle.transport_apply(Xo[rows], Yo, loga[rows], logb, fk[rows], gk, prob.eps,
                                     np.abs(v[0]).astype(np.float64))
    xs_t = 0.5 * (Xo.mean(0) + Yo.mean(0))
    xs, ys = Xo[rows] - xs_t, Yo - xs_t
    LOG2E = 1.0 / np.log(2.0)
    alpha = loga[rows] * LOG2E + (fk[rows] - (xs ** 2).sum(1)) * LOG2E / prob.eps
    beta = logb * LOG2E + (gk - (ys ** 2).sum(1)) * LOG2E / prob.eps
    M = np.abs(alpha) + np.abs(beta).max() + (2 * prob.d + 2) * 2 * np.sqrt((xs ** 2).sum(1)) * \
        np.sqrt((ys ** 2).sum(1)).max() * LOG2E / prob.eps
    rel = np.log(2.0) * 2.0 ** -23 * M + 2.0 ** -21 + prob.m * 2.0 ** -24
    err = (np.abs(out[rows] - oo[:, 0]) / (rel * absw[:, 0])).max()
    rerr = (np.abs(r[rows] - ro) / (rel * ro)).max()
    print(f"{name} full-size one-column application, sampled rows: worst err / bound = {err:.3f}, "
          f"row sums {rerr:.3f}")
    assert err <= 1.0 and rerr <= 1.0

