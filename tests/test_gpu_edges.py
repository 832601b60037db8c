"""Edge cases, invariants and error paths of the CUDA path (through the C ABI)."""
import numpy as np
import pytest

import oracle
from helpers import device_inputs, make_problem, max_cost, oracle_arrays

pytestmark = pytest.mark.gpu


def _fs():
    import log_domain_sinkhorn_updates_b200 as fs
    return fs


def _cloud(n, m, d, seed, dtype="f32"):
    import torch
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((n, d)).astype(np.float32)
    Y = (rng.standard_normal((m, d)) * 0.8 + 0.3).astype(np.float32)
    if dtype == "bf16":
        Xt = torch.from_numpy(X).to(torch.bfloat16)
        Yt = torch.from_numpy(Y).to(torch.bfloat16)
        X = Xt.to(torch.float32).numpy()
        Y = Yt.to(torch.float32).numpy()
        return X, Y, Xt.cuda(), Yt.cuda()
    return X, Y, torch.from_numpy(X).cuda(), torch.from_numpy(Y).cuda()


@pytest.mark.parametrize("prec", ["auto", "f32_simt"])
def test_single_point_closed_form(cuda_device, prec):
    import torch
    fs = _fs()
    X, Y, Xd, Yd = _cloud(1, 1, 3, 1)
    C11 = float(((X.astype(np.float64) - Y) ** 2).sum())
    h = fs.fs_create(Xd, Yd, eps=0.1, prec=prec)
    f = torch.zeros(1, 1, device=cuda_device)
    g = torch.zeros(1, 1, device=cuda_device)
    fs.fs_solve(h, f, g, 3)
    er, ec = fs.fs_marginal_err(h, f, g)
    dual, primal = fs.fs_ot_cost(h, f, g)
    assert abs(f.item() - C11) <= 1e-5 * C11 and abs(g.item()) <= 1e-5 * C11
    assert er[0] < 1e-5 and ec[0] < 1e-5
    assert abs(dual[0] - C11) <= 1e-5 * C11 and abs(primal[0] - C11) <= 1e-5 * C11


SHAPES = [(1, 300, 5, "f32"), (300, 1, 5, "f32"), (129, 255, 1, "f32"), (257, 129, 17, "f32"),
          (130, 390, 128, "bf16"), (383, 200, 64, "f32"), (200, 520, 40, "bf16"), (127, 129, 8, "f32")]


@pytest.mark.parametrize("prec", ["auto", "f32_simt"])
@pytest.mark.parametrize("n,m,d,dtype", SHAPES)
def test_ragged_shapes(cuda_device, n, m, d, dtype, prec):
    import torch
    fs = _fs()
    X, Y, Xd, Yd = _cloud(n, m, d, n * 7 + m, dtype)
    eps = 0.05
    rng = np.random.default_rng(3)
    g_in = (0.3 * rng.standard_normal(m)).astype(np.float32)
    f_in = (0.3 * rng.standard_normal(n)).astype(np.float32)
    h = fs.fs_create(Xd, Yd, eps=eps, prec=prec)
    f = torch.empty(1, n, device=cuda_device)
    g = torch.empty(1, m, device=cuda_device)
    fs.fs_update_f(h, torch.from_numpy(g_in).cuda()[None], f)
    fs.fs_update_g(h, torch.from_numpy(f_in).cuda()[None], g)
    fs.fs_sync(h)
    Xo, Yo = X.astype(np.float64), Y.astype(np.float64)
    la, lb = np.full(n, -np.log(n)), np.full(m, -np.log(m))
    fo = oracle.update_f(Xo, Yo, lb, g_in.astype(np.float64), eps)
    go = oracle.update_g(Xo, Yo, la, f_in.astype(np.float64), eps)
    _, _, cm = oracle.minplus_bounds(Xo, Yo, lb, np.zeros(m), 1.0)
    tol = 1e-4 * cm.max()
    assert np.abs(f.cpu().numpy()[0] - fo).max() <= tol
    assert np.abs(g.cpu().numpy()[0] - go).max() <= tol


def test_solve_is_deterministic_and_resumable(cuda_device):
    """A solve equals the same sequence of single updates bit for bit, and splitting it
    into two solves (resume from the saved potentials) changes nothing."""
    import torch
    fs = _fs()
    prob = make_problem("highdim", n=600, m=700)
    X, Y, a, b = device_inputs(prob)
    h = fs.fs_create(X, Y, a, b, eps=prob.eps)

    def run(chunks):
        f = torch.zeros(1, prob.n, device=cuda_device)
        g = torch.zeros(1, prob.m, device=cuda_device)
        for c in chunks:
            fs.fs_solve(h, f, g, c)
        fs.fs_sync(h)
        return f.clone(), g.clone()

    f1, g1 = run([6])
    f2, g2 = run([6])
    f3, g3 = run([3, 3])
    f4, g4 = run([1] * 6)
    f5 = torch.zeros(1, prob.n, device=cuda_device)
    g5 = torch.zeros(1, prob.m, device=cuda_device)
    for _ in range(6):
        fs.fs_update_f(h, g5, f5)
        fs.fs_update_g(h, f5, g5)
    fs.fs_sync(h)
    for f_, g_ in [(f2, g2), (f3, g3), (f4, g4), (f5, g5)]:
        assert torch.equal(f1, f_) and torch.equal(g1, g_)


def test_gauge_and_swap(cuda_device):
    import torch
    fs = _fs()
    n, m, d = 300, 410, 16
    X, Y, Xd, Yd = _cloud(n, m, d, 11)
    eps = 0.1
    g0 = torch.from_numpy((0.2 * np.random.default_rng(5).standard_normal(m)).astype(np.float32)).cuda()[None]
    h = fs.fs_create(Xd, Yd, eps=eps)
    hs = fs.fs_create(Yd, Xd, eps=eps)
    f1 = torch.empty(1, n, device=cuda_device)
    f2 = torch.empty(1, n, device=cuda_device)
    f3 = torch.empty(1, n, device=cuda_device)
    fs.fs_update_f(h, g0, f1)
    fs.fs_update_f(h, g0 + 0.375, f2)     # gauge: g + c  ->  f - c
    fs.fs_update_g(hs, g0, f3)            # swap: the g-update of (Y, X)
    fs.fs_sync(h)
    fs.fs_sync(hs)
    _, _, cm = oracle.minplus_bounds(X.astype(np.float64), Y.astype(np.float64), np.zeros(m), np.zeros(m), 1.0)
    tol = 1e-4 * cm.max()
    assert (f2 - (f1 - 0.375)).abs().max().item() <= tol
    assert (f3 - f1).abs().max().item() <= tol


def test_symmetric_schedule_matches_oracle_jacobi(cuda_device):
    import torch
    fs = _fs()
    prob = make_problem("middim", n=500, m=450)
    X, Y, a, b = device_inputs(prob)
    h = fs.fs_create(X, Y, a, b, eps=prob.eps)
    iters = 20
    f = torch.zeros(1, prob.n, device=cuda_device)
    g = torch.zeros(1, prob.m, device=cuda_device)
    fs.fs_solve(h, f, g, iters, schedule="symmetric")
    Xo, Yo, loga, logb = oracle.problem_arrays(prob)
    fo, go = np.zeros(prob.n), np.zeros(prob.m)
    for _ in range(iters):  # Jacobi: both halves from the previous pair
        fo, go = oracle.update_f(Xo, Yo, logb, go, prob.eps), oracle.update_g(Xo, Yo, loga, fo, prob.eps)
    _, _, cm = oracle.minplus_bounds(Xo, Yo, logb, np.zeros(prob.m), 1.0)
    tol = 1e-4 * cm.max()
    assert np.abs(f.cpu().numpy()[0] - fo).max() <= tol
    assert np.abs(g.cpu().numpy()[0] - go).max() <= tol


def test_host_entry_point_matches_device_path(cuda_device):
    import torch
    fs = _fs()
    prob = make_problem("batched", batch=2, n=300, m=260)
    X, Y, a, b = device_inputs(prob)
    h = fs.fs_create(X, Y, a, b, eps=prob.eps)
    f = torch.zeros(2, prob.n, device=cuda_device)
    g = torch.zeros(2, prob.m, device=cuda_device)
    fs.fs_solve(h, f, g, 7)
    er, ec = fs.fs_marginal_err(h, f, g)
    dual, primal = fs.fs_ot_cost(h, f, g)
    fh, gh, er2, ec2, dual2, primal2 = fs.fs_solve_host(prob.X_dev, prob.Y_dev, prob.a_dev, prob.b_dev,
                                                        np.zeros((2, prob.m), np.float32), prob.eps, 7)
    assert np.array_equal(fh, f.cpu().numpy()) and np.array_equal(gh, g.cpu().numpy())
    assert np.array_equal(er, er2) and np.array_equal(ec, ec2)
    assert np.array_equal(dual, dual2) and np.array_equal(primal, primal2)


def test_input_validation(cuda_device):
    import torch
    fs = _fs()
    X, Y, Xd, Yd = _cloud(50, 60, 4, 2)
    a = torch.full((50,), 1.0 / 50, device=cuda_device)
    bad = a.clone()
    bad[3] = 0.0
    bad[4] += 1.0 / 50
    with pytest.raises(fs.FsError) as e:
        fs.fs_create(Xd, Yd, bad, None, eps=0.1)
    assert e.value.status == 1
    with pytest.raises(fs.FsError) as e:
        fs.fs_create(Xd, Yd, a * 1.01, None, eps=0.1)
    assert e.value.status == 1
    Xn = Xd.clone()
    Xn[7, 2] = float("nan")
    with pytest.raises(fs.FsError) as e:
        fs.fs_create(Xn, Yd, eps=0.1)
    assert e.value.status == 4
    h = fs.fs_create(Xd, Yd, a, None, eps=0.1)  # valid weights pass
    info = fs.fs_get_info(h)
    assert info["device_bytes"] < 100 * (50 + 60) * 4 * 64 + (1 << 20)


def test_bounded_wait_times_out_and_the_context_stays_usable(cuda_device):
    """A kernel waits on an mbarrier that nothing completes: the bounded wait ends,
    the status is FS_ERR_TIMEOUT, and the same handle then runs a correct update."""
    import time
    import torch
    import log_domain_sinkhorn_updates_b200 as fs
    prob = make_problem("tiny")
    X, Y, a, b = device_inputs(prob)
    h = fs.fs_create(X, Y, a, b, eps=prob.eps)
    t0 = time.perf_counter()
    st = fs.fs_selftest_wait(h, 50)
    dt = time.perf_counter() - t0
    assert st == 5 and dt >= 0.045, (st, dt)
    g_in = torch.zeros(1, prob.m, device=cuda_device)
    f = torch.empty(1, prob.n, device=cuda_device)
    fs.fs_update_f(h, g_in, f)
    fs.fs_sync(h)
    Xo, Yo, _, logb = oracle_arrays(prob)[0]
    fo = oracle.update_f(Xo, Yo, logb, np.zeros(prob.m), prob.eps)
    assert np.abs(f.cpu().numpy()[0] - fo).max() <= 1e-4 * max_cost(prob)[0] / 4
