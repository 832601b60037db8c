"""The cosine cost (C_ij = 1 - cos(x_i, y_j); "cosine distance after
normalisation", which "FlashSinkhorn: IO-aware EOT on GPU" names in its closing
remarks as the other cost the method covers) through the C ABI, against the
oracle's cosine cost. Same bars as the squared-Euclidean parity tests:
single updates within 1e-4 * max C / 4, solves within 1e-3 relative."""
import numpy as np
import pytest

import oracle
from helpers import device_inputs, make_problem, oracle_arrays, smooth_potential

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": dict(),
    "middim": dict(n=1000, m=900),
    "cloud3d": dict(n=1500, m=1100),
    "highdim": dict(n=700, m=650),
    "batched": dict(batch=3, n=600, m=520),
}
PRECS = ["auto", "f32_simt", "3xtf32"]


def _fs():
    import log_domain_sinkhorn_updates_b200 as fs
    return fs


def _max_cost(prob):
    out = []
    for X, Y, _, logb in oracle_arrays(prob):
        _, _, cm = oracle.minplus_bounds(X, Y, logb, np.zeros(Y.shape[0]), 1.0, cost="cosine")
        out.append(cm.max())
    return np.array(out)


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("prec", PRECS)
def test_cosine_single_update_parity(cuda_device, name, prec):
    import torch
    fs = _fs()
    prob = make_problem(name, **SMALL[name])
    if prec == "3xtf32" and prob.d > 64:
        pytest.skip("3xTF32 rows are limited to d <= 64")
    X, Y, a, b = device_inputs(prob)
    h = fs.fs_create(X, Y, a, b, eps=prob.eps, prec=prec, cost="cosine")
    rng = np.random.default_rng(91)
    g_in = np.stack([smooth_potential(rng, prob.m, 0.05) for _ in range(prob.batch)])
    f_in = np.stack([smooth_potential(rng, prob.n, 0.05) for _ in range(prob.batch)])
    f = torch.empty(prob.batch, prob.n, device=cuda_device)
    g = torch.empty(prob.batch, prob.m, device=cuda_device)
    fs.fs_update_f(h, torch.from_numpy(g_in).to(cuda_device), f)
    fs.fs_update_g(h, torch.from_numpy(f_in).to(cuda_device), g)
    fs.fs_sync(h)
    f, g = f.cpu().numpy(), g.cpu().numpy()
    tol = 1e-4 * _max_cost(prob)
    for k, (Xo, Yo, loga, logb) in enumerate(oracle_arrays(prob)):
        fo = oracle.update_f(Xo, Yo, logb, g_in[k].astype(np.float64), prob.eps, cost="cosine")
        go = oracle.update_g(Xo, Yo, loga, f_in[k].astype(np.float64), prob.eps, cost="cosine")
        ef, eg = np.abs(f[k] - fo).max(), np.abs(g[k] - go).max()
        assert max(ef, eg) <= tol[k] / 4, (name, prec, k, ef, eg, tol[k])


@pytest.mark.parametrize("name", ["tiny", "middim", "batched"])
def test_cosine_solve_parity(cuda_device, name):
    import torch
    fs = _fs()
    prob = make_problem(name, **SMALL[name])
    X, Y, a_d, b_d = device_inputs(prob)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps, cost="cosine")
    f = torch.zeros(prob.batch, prob.n, device=cuda_device)
    g = torch.zeros(prob.batch, prob.m, device=cuda_device)
    fs.fs_solve(h, f, g, prob.iters)
    er, ec = fs.fs_marginal_err(h, f, g)
    dual, primal = fs.fs_ot_cost(h, f, g)
    fg, gg = f.cpu().numpy().astype(np.float64), g.cpu().numpy().astype(np.float64)
    for k, (Xo, Yo, loga, logb) in enumerate(oracle_arrays(prob)):
        fo, go = oracle.solve(Xo, Yo, loga, logb, prob.eps, prob.iters, cost="cosine")
        eo = oracle.marginal_error(Xo, Yo, loga, logb, fo, go, prob.eps, cost="cosine")
        co = oracle.costs(Xo, Yo, loga, logb, fo, go, prob.eps, cost="cosine")
        a, b = np.exp(loga), np.exp(logb)
        c = a @ (fg[k] - fo)
        df, dg = fg[k] - fo - c, gg[k] - go + c
        tau = 2.0 * (a @ np.abs(df) + b @ np.abs(dg)) / prob.eps
        print(f"{name}[{k}] err {er[k] + ec[k]:.4e}/{eo[0] + eo[1]:.4e} tau {tau:.2e} dual {dual[k]:.9g}/"
              f"{co['dual']:.9g} primal {primal[k]:.9g}/{co['primal']:.9g}")
        assert abs(er[k] + ec[k] - eo[0] - eo[1]) <= 1e-3 * (eo[0] + eo[1]) + tau
        assert abs(dual[k] - co["dual"]) <= 1e-3 * abs(co["dual"])
        assert abs(primal[k] - co["primal"]) <= 1e-3 * abs(co["primal"])


def test_cosine_full_size_sampled(cuda_device):
    """highdim at full size (65536 x 65536, d = 128, bf16 inputs) under the cosine
    cost: 3xF16 rows of 512 bytes, i.e. the CTA-pair pass; checked at sampled rows."""
    import torch
    fs = _fs()
    prob = make_problem("highdim")
    X, Y, a_d, b_d = device_inputs(prob)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps, cost="cosine")
    info = fs.fs_get_info(h)
    assert info["prec"] == "3xf16" and info["cta_pair"] == 1
    rng = np.random.default_rng(92)
    g_in = smooth_potential(rng, prob.m, 0.05)[None]
    f = torch.empty(1, prob.n, device=cuda_device)
    fs.fs_update_f(h, torch.from_numpy(g_in).to(cuda_device), f)
    fs.fs_sync(h)
    Xo, Yo, _, logb = oracle.problem_arrays(prob, 0)
    rows = np.unique(np.concatenate([[0, prob.n - 1], rng.choice(prob.n, 256, replace=False)]))
    fo = oracle.update_f_rows(rows, Xo, Yo, logb, g_in[0].astype(np.float64), prob.eps, cost="cosine")
    _, _, cm = oracle.minplus_bounds(Xo[rows], Yo, logb, np.zeros(prob.m), 1.0, cost="cosine")
    err = np.abs(f.cpu().numpy()[0][rows] - fo).max()
    print(f"highdim cosine sampled max|df| = {err:.3e} (tol {1e-4 * cm.max() / 4:.3e})")
    assert err <= 1e-4 * cm.max() / 4


def test_cosine_rejects_zero_rows(cuda_device):
    import torch
    fs = _fs()
    rng = np.random.default_rng(93)
    X = rng.standard_normal((300, 8)).astype(np.float32)
    Y = rng.standard_normal((310, 8)).astype(np.float32)
    X[17] = 0.0
    with pytest.raises(fs.FsError) as e:
        fs.fs_create(torch.from_numpy(X).to(cuda_device), torch.from_numpy(Y).to(cuda_device), eps=0.1,
                     cost="cosine")
    assert e.value.status == 1
