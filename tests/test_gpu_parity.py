"""GPU parity against the CPU oracle, through the C ABI.

Single updates: every workload recipe at sizes the oracle finishes in seconds,
spanning several 128-row/256-column tiles with ragged tails; the bar is
max |f_gpu - f_oracle| <= 1e-4 * max_ij C_ij (both sides see the same float32
inputs, the oracle in double).  Full solves: marginal L1 error and dual cost
after the recipe's iteration count within 1e-3 relative (the marginal error
plus twice the oracle's own float32 floor, see oracle_fp32_floor), and the
gauge-fixed potentials within the single-update bar.
"""
import numpy as np
import pytest

import oracle
from helpers import device_inputs, max_cost, make_problem, oracle_arrays, smooth_potential

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": dict(),
    "middim": dict(n=1000, m=900),
    "cloud3d": dict(n=1500, m=1100),
    "highdim": dict(n=700, m=650),
    "batched": dict(batch=3, n=600, m=520),
}
# every mode that is meant to be ~fp32 accurate on the workload's inputs
PRECS = {
    "tiny": ["auto", "f32_simt", "3xtf32", "3xf16"],
    "middim": ["auto", "f32_simt", "3xf16", "3xtf32"],
    "cloud3d": ["auto", "f32_simt", "3xtf32", "3xf16"],
    "highdim": ["auto", "f32_simt"],
    "batched": ["auto", "f32_simt", "3xtf32", "3xf16"],
}
CASES = [(name, prec) for name in SMALL for prec in PRECS[name]]


def _fs():
    import log_domain_sinkhorn_updates_b200 as fs
    return fs


@pytest.mark.parametrize("name,prec", CASES)
def test_single_update_parity(cuda_device, name, prec):
    import torch
    fs = _fs()
    prob = make_problem(name, **SMALL[name])
    X, Y, a, b = device_inputs(prob)
    h = fs.fs_create(X, Y, a, b, eps=prob.eps, prec=prec)
    rng = np.random.default_rng(77)
    tol = 1e-4 * max_cost(prob)
    g_in = np.stack([smooth_potential(rng, prob.m, 0.5) for _ in range(prob.batch)])
    f_in = np.stack([smooth_potential(rng, prob.n, 0.5) for _ in range(prob.batch)])
    f = torch.empty(prob.batch, prob.n, device=cuda_device)
    g = torch.empty(prob.batch, prob.m, device=cuda_device)
    fs.fs_update_f(h, torch.from_numpy(g_in).to(cuda_device), f)
    fs.fs_update_g(h, torch.from_numpy(f_in).to(cuda_device), g)
    fs.fs_sync(h)
    f = f.cpu().numpy()
    g = g.cpu().numpy()
    for k, (Xo, Yo, loga, logb) in enumerate(oracle_arrays(prob)):
        fo = oracle.update_f(Xo, Yo, logb, g_in[k].astype(np.float64), prob.eps)
        go = oracle.update_g(Xo, Yo, loga, f_in[k].astype(np.float64), prob.eps)
        ef = np.abs(f[k] - fo).max()
        eg = np.abs(g[k] - go).max()
        assert ef <= tol[k], (name, prec, k, ef, tol[k])
        assert eg <= tol[k], (name, prec, k, eg, tol[k])
        # every mode here is ~fp32 accurate and must leave a 4x margin to the bar
        assert max(ef, eg) <= tol[k] / 4, (name, prec, k, ef, eg, tol[k])


@pytest.mark.parametrize("name", ["tiny", "middim", "cloud3d", "batched"])
def test_single_update_tf32_within_its_rounding_bound(cuda_device, name):
    """One-pass TF32 (operands rounded to 10 mantissa bits, the column bias added
    inside the S product in tf32 parts) is not fp32-accurate; it must stay within
    what its operand rounding allows.  With q = x - t and k = 2(y - t) each
    rounded to relative 2^-11, |S~_ij - S_ij| <= 2^-10 |q_i| |k_j| (Cauchy-
    Schwarz), and the LSE moves by at most the largest change of its arguments,
    so |f~_i - f_i| <= 2^-10 |q_i| max_j |k_j| (and symmetrically for g), plus the
    fp32 bar of the accurate modes."""
    import torch
    fs = _fs()
    prob = make_problem(name, **SMALL[name])
    X, Y, a, b = device_inputs(prob)
    h = fs.fs_create(X, Y, a, b, eps=prob.eps, prec="tf32")
    rng = np.random.default_rng(78)
    g_in = np.stack([smooth_potential(rng, prob.m, 0.5) for _ in range(prob.batch)])
    f_in = np.stack([smooth_potential(rng, prob.n, 0.5) for _ in range(prob.batch)])
    f = torch.empty(prob.batch, prob.n, device=cuda_device)
    g = torch.empty(prob.batch, prob.m, device=cuda_device)
    fs.fs_update_f(h, torch.from_numpy(g_in).to(cuda_device), f)
    fs.fs_update_g(h, torch.from_numpy(f_in).to(cuda_device), g)
    fs.fs_sync(h)
    f, g = f.cpu().numpy(), g.cpu().numpy()
    bar = 1e-4 * max_cost(prob) / 4
    for k, (Xo, Yo, loga, logb) in enumerate(oracle_arrays(prob)):
        t = 0.5 * (Xo.mean(axis=0) + Yo.mean(axis=0))
        qn = np.linalg.norm(Xo - t, axis=1)
        kn = 2 * np.linalg.norm(Yo - t, axis=1)
        fo = oracle.update_f(Xo, Yo, logb, g_in[k].astype(np.float64), prob.eps)
        go = oracle.update_g(Xo, Yo, loga, f_in[k].astype(np.float64), prob.eps)
        ef = np.abs(f[k] - fo) / (2.0 ** -10 * qn * kn.max() + bar[k])
        eg = np.abs(g[k] - go) / (2.0 ** -10 * kn * qn.max() + bar[k])
        print(f"tf32 {name}[{k}] worst err / bound: f {ef.max():.3f}, g {eg.max():.3f}")
        assert ef.max() <= 1.0 and eg.max() <= 1.0, (name, k, ef.max(), eg.max())


def test_unsupported_row_width_is_reported(cuda_device):
    """3xTF32 rows of d = 65 (640 bytes) exceed the 512-byte operand rows of the tensor-core pass."""
    import torch
    fs = _fs()
    rng = np.random.default_rng(4)
    X = torch.from_numpy(rng.standard_normal((300, 65)).astype(np.float32)).to(cuda_device)
    Y = torch.from_numpy(rng.standard_normal((310, 65)).astype(np.float32)).to(cuda_device)
    with pytest.raises(fs.FsError) as e:
        fs.fs_create(X, Y, eps=0.1, prec="3xtf32")
    assert e.value.status == 3
    fs.fs_create(X, Y, eps=0.1)  # the default (3xF16, 320-byte rows) runs


SOLVE = {
    "tiny": dict(),
    "middim": dict(n=1000, m=900),
    "cloud3d": dict(n=1500, m=1100),
    "highdim": dict(n=700, m=650),
    "batched": dict(batch=3, n=600, m=520),
}


def _gauge_fixed_diff(fg, gg, fo, go, a, b):
    """GPU - oracle potentials after removing the common constant (f + c, g - c leaves P unchanged)."""
    c = a @ (fg - fo)
    return fg - fo - c, gg - go + c


def oracle_fp32_floor(Xo, Yo, loga, logb, fo, go, eps):
    """How far the plan's marginals move, in L1, when the oracle's own potentials are rounded
    to float32: sum_i |r_i(fl f, fl g) - r_i(f, g)| + sum_j |c_j(fl f, fl g) - c_j(f, g)|.
    Computed by the oracle alone; by the triangle inequality it bounds the change of the
    marginal L1 error that one rounding of the potentials causes, the floor below which no
    float32 solution can be held.  A float32 solver rounds twice per update: once where it
    forms the LSE's arguments in float32 (the scaled score and the column bias, the leading
    term of its evaluation error) and once where it stores the potential.  Its solution is
    therefore compared within twice this floor."""
    f32 = fo.astype(np.float32).astype(np.float64)
    g32 = go.astype(np.float32).astype(np.float64)
    r, c = oracle.marginals(Xo, Yo, loga, logb, fo, go, eps)
    r32, c32 = oracle.marginals(Xo, Yo, loga, logb, f32, g32, eps)
    return float(np.abs(r32 - r).sum() + np.abs(c32 - c).sum())


@pytest.mark.parametrize("name", list(SOLVE))
def test_solve_parity(cuda_device, name):
    """fs_solve from g = 0 for the recipe's iteration count, then the measurements, against
    the oracle's own solve from the same inputs:

    * marginal L1 error within 1e-3 relative plus twice the oracle's fp32 floor
      (oracle_fp32_floor);
    * dual and primal objectives within 1e-3 relative;
    * the potentials, after removing the common gauge constant, within the single-update
      bar 1e-4 * max_ij C_ij.
    """
    import torch
    fs = _fs()
    prob = make_problem(name, **SOLVE[name])
    X, Y, a_d, b_d = device_inputs(prob)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps)
    f = torch.zeros(prob.batch, prob.n, device=cuda_device)
    g = torch.zeros(prob.batch, prob.m, device=cuda_device)
    fs.fs_solve(h, f, g, prob.iters)
    er, ec = fs.fs_marginal_err(h, f, g)
    dual, primal = fs.fs_ot_cost(h, f, g)
    assert fs.fs_get_info(h)["last_measure_fused"] == 1  # measured from the solve's tail
    fg, gg = f.cpu().numpy().astype(np.float64), g.cpu().numpy().astype(np.float64)
    for k, (Xo, Yo, loga, logb) in enumerate(oracle_arrays(prob)):
        fo, go = oracle.solve(Xo, Yo, loga, logb, prob.eps, prob.iters)
        eo = oracle.marginal_error(Xo, Yo, loga, logb, fo, go, prob.eps)
        co = oracle.costs(Xo, Yo, loga, logb, fo, go, prob.eps)
        tau = oracle_fp32_floor(Xo, Yo, loga, logb, fo, go, prob.eps)
        df, dg = _gauge_fixed_diff(fg[k], gg[k], fo, go, np.exp(loga), np.exp(logb))
        pot_err = max(np.abs(df).max(), np.abs(dg).max())
        pot_bar = 1e-4 * co["max_cost"]
        e_gpu, e_o = er[k] + ec[k], eo[0] + eo[1]
        print(f"{name}[{k}] err gpu={e_gpu:.6e} oracle={e_o:.6e} |diff|={abs(e_gpu - e_o):.3e} fp32 floor={tau:.3e} "
              f"dual {dual[k]:.9g} vs {co['dual']:.9g}  primal {primal[k]:.9g} vs {co['primal']:.9g} "
              f"gauge-fixed pot {pot_err:.3e} (bar {pot_bar:.3e})")
        assert abs(e_gpu - e_o) <= 1e-3 * e_o + 2.0 * tau, (name, k, e_gpu, e_o, tau)
        assert abs(dual[k] - co["dual"]) <= 1e-3 * abs(co["dual"]), (name, k, dual[k], co["dual"])
        assert abs(primal[k] - co["primal"]) <= 1e-3 * abs(co["primal"]), (name, k, primal[k], co["primal"])
        assert pot_err <= pot_bar, (name, k, pot_err, pot_bar)


@pytest.mark.parametrize("name", list(SOLVE))
def test_measure_parity(cuda_device, name):
    """fs_marginal_err / fs_ot_cost at the oracle's converged potentials (rounded to float32,
    the same bytes on both sides) against the oracle's measurements at those potentials."""
    import torch
    fs = _fs()
    prob = make_problem(name, **SOLVE[name])
    X, Y, a_d, b_d = device_inputs(prob)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps)
    pots = [oracle.solve(*arr, prob.eps, prob.iters) for arr in oracle_arrays(prob)]
    f32 = np.stack([p[0] for p in pots]).astype(np.float32)
    g32 = np.stack([p[1] for p in pots]).astype(np.float32)
    f = torch.from_numpy(f32).to(cuda_device)
    g = torch.from_numpy(g32).to(cuda_device)
    er, ec = fs.fs_marginal_err(h, f, g)
    dual, primal = fs.fs_ot_cost(h, f, g)
    for k, (Xo, Yo, loga, logb) in enumerate(oracle_arrays(prob)):
        fk, gk = f32[k].astype(np.float64), g32[k].astype(np.float64)
        eo = oracle.marginal_error(Xo, Yo, loga, logb, fk, gk, prob.eps)
        co = oracle.costs(Xo, Yo, loga, logb, fk, gk, prob.eps)
        # float32 LSE of each row carries a relative error ~2^-22 of its log-domain
        # argument (|pot| + max C)/eps; first-order effect on the marginal sums:
        cmax = co["max_cost"]
        a, b = np.exp(loga), np.exp(logb)
        tau = 2.0 ** -21 * (a @ (np.abs(fk) + cmax) + b @ (np.abs(gk) + cmax)) / prob.eps
        print(f"{name}[{k}] row {er[k]:.6e}/{eo[0]:.6e} col {ec[k]:.6e}/{eo[1]:.6e} tau={tau:.2e} "
              f"dual {dual[k]:.10g}/{co['dual']:.10g} primal {primal[k]:.10g}/{co['primal']:.10g}")
        assert abs(er[k] - eo[0]) <= 1e-3 * eo[0] + tau, (name, k, er[k], eo[0], tau)
        assert abs(ec[k] - eo[1]) <= 1e-3 * eo[1] + tau, (name, k, ec[k], eo[1], tau)
        assert abs(dual[k] - co["dual"]) <= 1e-3 * abs(co["dual"]), (name, k)
        assert abs(primal[k] - co["primal"]) <= 1e-3 * abs(co["primal"]), (name, k)


@pytest.mark.parametrize("name", ["middim", "highdim", "batched"])
def test_cta_pair_kernel_parity(cuda_device, name, monkeypatch):
    """The CTA-pair tensor-core pass (FS_CTA_PAIR=1, one MMA over two SMs) and the
    single-CTA pass that runs by default, both against the oracle."""
    import torch
    fs = _fs()
    prob = make_problem(name, **SMALL[name])
    X, Y, a, b = device_inputs(prob)
    rng = np.random.default_rng(78)
    g_in = torch.from_numpy(np.stack([smooth_potential(rng, prob.m, 0.5) for _ in range(prob.batch)])).to(cuda_device)
    outs = {}
    for pair in ("0", "1"):
        monkeypatch.setenv("FS_CTA_PAIR", pair)
        h = fs.fs_create(X, Y, a, b, eps=prob.eps)
        assert fs.fs_get_info(h)["cta_pair"] == int(pair)
        f = torch.empty(prob.batch, prob.n, device=cuda_device)
        fs.fs_update_f(h, g_in, f)
        fs.fs_sync(h)
        outs[pair] = f.cpu().numpy()
    tol = 1e-4 * max_cost(prob)
    for k, (Xo, Yo, _, logb) in enumerate(oracle_arrays(prob)):
        fo = oracle.update_f(Xo, Yo, logb, g_in[k].cpu().numpy().astype(np.float64), prob.eps)
        for pair in ("0", "1"):
            assert np.abs(outs[pair][k] - fo).max() <= tol[k] / 4, (name, pair, k)


@pytest.mark.parametrize("name", list(SMALL))
def test_row_block_pairing_parity(cuda_device, name, monkeypatch):
    """The single-CTA pass with two resident 128-row blocks per CTA (each K tile
    serves 256 rows; the default where it fits) and with one (FS_ROW_BLOCKS=1),
    both against the oracle, for the f- and the g-update."""
    import torch
    fs = _fs()
    prob = make_problem(name, **SMALL[name])
    X, Y, a, b = device_inputs(prob)
    rng = np.random.default_rng(79)
    g_in = np.stack([smooth_potential(rng, prob.m, 0.5) for _ in range(prob.batch)])
    f_in = np.stack([smooth_potential(rng, prob.n, 0.5) for _ in range(prob.batch)])
    outs = {}
    for mode in ("1", "2"):
        monkeypatch.setenv("FS_ROW_BLOCKS", mode)
        h = fs.fs_create(X, Y, a, b, eps=prob.eps)
        assert fs.fs_get_info(h)["block_rows"] == 128 * int(mode)
        f = torch.empty(prob.batch, prob.n, device=cuda_device)
        g = torch.empty(prob.batch, prob.m, device=cuda_device)
        fs.fs_update_f(h, torch.from_numpy(g_in).to(cuda_device), f)
        fs.fs_update_g(h, torch.from_numpy(f_in).to(cuda_device), g)
        fs.fs_sync(h)
        outs[mode] = (f.cpu().numpy(), g.cpu().numpy())
    tol = 1e-4 * max_cost(prob)
    for k, (Xo, Yo, loga, logb) in enumerate(oracle_arrays(prob)):
        fo = oracle.update_f(Xo, Yo, logb, g_in[k].astype(np.float64), prob.eps)
        go = oracle.update_g(Xo, Yo, loga, f_in[k].astype(np.float64), prob.eps)
        for mode in ("1", "2"):
            assert np.abs(outs[mode][0][k] - fo).max() <= tol[k] / 4, (name, mode, k, "f")
            assert np.abs(outs[mode][1][k] - go).max() <= tol[k] / 4, (name, mode, k, "g")
