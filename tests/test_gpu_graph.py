"""fs_solve as a CUDA graph: the replayed loop gives the same bits as the same
kernels launched one by one, a kept graph is replayed only for the buffers,
iteration count and schedule it was captured with, and the launch counter counts
the replayed kernels."""
import numpy as np
import pytest

from helpers import device_inputs, make_problem

pytestmark = pytest.mark.gpu


def _fs():
    import log_domain_sinkhorn_updates_b200 as fs
    return fs


def _solve(fs, h, prob, dev, iters, schedule, mode, monkeypatch, f=None, g=None):
    import torch
    monkeypatch.setenv("FS_SOLVE_GRAPH", mode)
    if f is None:
        rng = np.random.default_rng(11)
        f = torch.from_numpy(rng.standard_normal((prob.batch, prob.n)).astype(np.float32) * 0.1).to(dev)
        g = torch.from_numpy(rng.standard_normal((prob.batch, prob.m)).astype(np.float32) * 0.1).to(dev)
    k0 = fs.fs_kernel_launches()
    fs.fs_solve(h, f, g, iters, schedule=schedule)
    fs.fs_sync(h)
    launched = fs.fs_kernel_launches() - k0
    return f, g, launched, fs.fs_get_info(h)["last_solve_graph"]


@pytest.mark.parametrize("schedule", ["alternating", "symmetric"])
@pytest.mark.parametrize("name,kw", [("tiny", {}), ("highdim", dict(n=600, m=700)), ("batched", dict(batch=3, n=300, m=260))])
def test_graph_matches_direct_launches(cuda_device, name, kw, schedule, monkeypatch):
    fs = _fs()
    prob = make_problem(name, **kw)
    X, Y, a, b = device_inputs(prob)
    h = fs.fs_create(X, Y, a, b, eps=prob.eps)
    iters = 5
    per_iter, extra = (2, 1) if schedule == "alternating" else (4, 0)
    fd, gd, nd, how_d = _solve(fs, h, prob, cuda_device, iters, schedule, "0", monkeypatch)
    fg, gg, ng, how_g = _solve(fs, h, prob, cuda_device, iters, schedule, "1", monkeypatch)
    assert (how_d, how_g) == ("direct", "graph")
    assert nd == ng == per_iter * iters + extra
    assert np.array_equal(fd.cpu().numpy(), fg.cpu().numpy())
    assert np.array_equal(gd.cpu().numpy(), gg.cpu().numpy())
    fs.fs_destroy(h)


def test_graph_is_replayed_only_for_its_key(cuda_device, monkeypatch):
    """Two solves on the same buffers replay one graph (and continue from where the
    first stopped); a new iteration count or new buffers capture a new one.  Each
    result equals direct launches of the same total work."""
    import torch
    fs = _fs()
    prob = make_problem("tiny")
    X, Y, a, b = device_inputs(prob)
    h = fs.fs_create(X, Y, a, b, eps=prob.eps)
    z = lambda k: torch.zeros(1, k, device=cuda_device)  # noqa: E731

    def direct(iters):
        f, g = z(prob.n), z(prob.m)
        monkeypatch.setenv("FS_SOLVE_GRAPH", "0")
        fs.fs_solve(h, f, g, iters)
        fs.fs_sync(h)
        return f.cpu().numpy(), g.cpu().numpy()

    f, g = z(prob.n), z(prob.m)
    for _ in range(2):  # 3 + 3 iterations through one graph
        _, _, n, how = _solve(fs, h, prob, cuda_device, 3, "alternating", "1", monkeypatch, f, g)
        assert how == "graph" and n == 7
    fr, gr = direct(6)
    assert np.array_equal(f.cpu().numpy(), fr) and np.array_equal(g.cpu().numpy(), gr)
    _solve(fs, h, prob, cuda_device, 4, "alternating", "1", monkeypatch, f, g)  # new count: recaptured
    f2, g2 = z(prob.n), z(prob.m)
    _solve(fs, h, prob, cuda_device, 4, "alternating", "1", monkeypatch, f2, g2)  # new buffers: recaptured
    fr, gr = direct(4)
    assert np.array_equal(f2.cpu().numpy(), fr) and np.array_equal(g2.cpu().numpy(), gr)
    fs.fs_destroy(h)


def test_default_uses_the_graph_only_for_small_problems(cuda_device, monkeypatch):
    fs = _fs()
    monkeypatch.delenv("FS_SOLVE_GRAPH", raising=False)
    for name, kw, want in [("tiny", {}, "graph"), ("highdim", dict(n=8192, m=8192), "graph"),
                           ("highdim", dict(n=8192, m=8200), "direct")]:
        prob = make_problem(name, **kw)
        X, Y, a, b = device_inputs(prob)
        h = fs.fs_create(X, Y, a, b, eps=prob.eps)
        import torch
        f, g = torch.zeros(1, prob.n, device=cuda_device), torch.zeros(1, prob.m, device=cuda_device)
        fs.fs_solve(h, f, g, 2)
        fs.fs_sync(h)
        assert fs.fs_get_info(h)["last_solve_graph"] == want, (name, kw)
        fs.fs_destroy(h)


def test_solve_inside_a_caller_graph(cuda_device, monkeypatch):
    """A caller that captures the handle's stream gets fs_solve's kernels in its own
    graph (no private graph is captured inside that capture); replaying the caller's
    graph gives the bits of direct launches."""
    import torch
    fs = _fs()
    monkeypatch.delenv("FS_SOLVE_GRAPH", raising=False)
    prob = make_problem("tiny")
    X, Y, a, b = device_inputs(prob)
    s = torch.cuda.Stream()
    h = fs.fs_create(X, Y, a, b, eps=prob.eps, stream=s)
    f = torch.zeros(1, prob.n, device=cuda_device)
    g = torch.zeros(1, prob.m, device=cuda_device)
    torch.cuda.synchronize()
    caller = torch.cuda.CUDAGraph()
    with torch.cuda.graph(caller, stream=s):
        fs.fs_solve(h, f, g, 3)
    assert fs.fs_get_info(h)["last_solve_graph"] == "direct"
    caller.replay()
    torch.cuda.synchronize()
    monkeypatch.setenv("FS_SOLVE_GRAPH", "0")
    f2 = torch.zeros(1, prob.n, device=cuda_device)
    g2 = torch.zeros(1, prob.m, device=cuda_device)
    fs.fs_solve(h, f2, g2, 3)
    fs.fs_sync(h)
    assert np.array_equal(f.cpu().numpy(), f2.cpu().numpy())
    assert np.array_equal(g.cpu().numpy(), g2.cpu().numpy())
    del caller
    fs.fs_destroy(h)
