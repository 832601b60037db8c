"""Transport application (out_i = sum_j P_ij V_j, the barycentric map and the
position gradient; "FlashSinkhorn: IO-aware EOT on GPU", Metodologia section 3)
through the C ABI, against the oracle at the same float32 potentials.

Tolerance, derived from the arithmetic of the GPU path.  log2 P_ij =
alpha_i + beta_j + S_ij log2(e)/eps is formed in double from float32 terms:
- alpha_i and beta_j are each rounded to fp32;
- the score S_ij is an fp32 dot product of operands that are exact or split to
  about 2^-22.
So the exponent is off by at most 2^-23 M_i with
M_i = |alpha_i| + max_j (|beta_j| + (2d + 2) |S_ij| log2(e)/eps).
exp2f adds 2^-21, and the fp32 sum over m terms adds m 2^-24.  Hence

  |out_gpu - out_oracle|_i <= (ln2 2^-23 M_i + 2^-21 + m 2^-24) sum_j P_ij |V_j|.

The tensor-core path also splits P/a_i and V into bf16 hi + lo pairs, which
carry 2^-16 each and drop a term of 2^-16 relative size, so its bound adds
2^-14.  Every test runs five paths: the tensor-core kernel with two 128-row
blocks per CTA (FS_ROW_BLOCKS=2; the default for dv < 64 and rows of up to
256 bytes once the grid covers the SMs), the same kernel with one block shared
by both softmax groups taking alternate tiles (FS_ROW_BLOCKS=3; the default
for dv of 64 to 128 and for smaller grids), the one-block tensor-core kernel
(FS_ROW_BLOCKS=1), the
tensor-core kernel on CTA
pairs (FS_APPLY_PAIR=1; the default for 512-byte operand rows) and the
CUDA-core validation kernel (FS_APPLY_SIMT=1).
"""
import numpy as np
import pytest

import oracle
from helpers import device_inputs, make_problem, oracle_arrays

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": dict(),
    "middim": dict(n=1000, m=900),
    "cloud3d": dict(n=1500, m=1100),
    "highdim": dict(n=700, m=650),
    "batched": dict(batch=3, n=600, m=520),
}
LOG2E = 1.0 / np.log(2.0)


def _fs():
    import log_domain_sinkhorn_updates_b200 as fs
    return fs


def _potentials(prob, cost, iters=8):
    """A few oracle iterations from g = 0, rounded to float32 (the same bytes on both sides)."""
    fs_, gs_ = [], []
    for Xo, Yo, loga, logb in oracle_arrays(prob):
        f, g = oracle.solve(Xo, Yo, loga, logb, prob.eps, iters, cost=cost)
        fs_.append(f.astype(np.float32))
        gs_.append(g.astype(np.float32))
    return np.stack(fs_), np.stack(gs_)


def _rel_bound(Xo, Yo, loga, logb, f, g, eps, cost):
    d = Xo.shape[1]
    if cost == "cosine":
        xs = Xo / np.linalg.norm(Xo, axis=1, keepdims=True)
        ys = Yo / np.linalg.norm(Yo, axis=1, keepdims=True)
        xn = np.full(len(Xo), 0.5)
        yn = np.full(len(Yo), 0.5)
        nx, ny = np.ones(len(Xo)), np.ones(len(Yo))
    else:
        t = 0.5 * (Xo.mean(axis=0) + Yo.mean(axis=0))
        xs, ys = Xo - t, Yo - t
        xn, yn = (xs ** 2).sum(1), (ys ** 2).sum(1)
        nx, ny = 2 * np.sqrt(xn), np.sqrt(yn)
    alpha = loga * LOG2E + (f - xn) * LOG2E / eps
    beta = logb * LOG2E + (g - yn) * LOG2E / eps
    M = np.abs(alpha) + np.max(np.abs(beta)[None, :] + (2 * d + 2) * nx[:, None] * ny[None, :] * LOG2E / eps, axis=1)
    return np.log(2.0) * 2.0 ** -23 * M + 2.0 ** -21 + len(Yo) * 2.0 ** -24


# (FS_APPLY_SIMT, FS_APPLY_PAIR, FS_ROW_BLOCKS)
PATHS = {"tc_q2": ("0", "0", "2"), "tc_2s": ("0", "0", "3"), "tc": ("0", "0", "1"), "tc_pair": ("0", "1", "2"),
         "simt": ("1", "0", "2")}
SPLIT = {"tc_q2": 2.0 ** -14, "tc_2s": 2.0 ** -14, "tc": 2.0 ** -14, "tc_pair": 2.0 ** -14, "simt": 0.0}


def _set_path(monkeypatch, path):
    monkeypatch.setenv("FS_APPLY_SIMT", PATHS[path][0])
    monkeypatch.setenv("FS_APPLY_PAIR", PATHS[path][1])
    monkeypatch.setenv("FS_ROW_BLOCKS", PATHS[path][2])
    monkeypatch.setenv("FS_APPLY_VEC", "0")  # one-column applications through these kernels too


def _assert_path(fs, h, path, dv):
    """The kernel that ran, as the handle reports it: the CUDA-core one when it is
    forced; a tensor-core one otherwise whenever dv <= 128, where every operand
    width of these workloads fits the shared-memory plans (the two-block kernel
    by default, the one-block kernel with FS_ROW_BLOCKS=1); at larger dv, where
    the two-block kernel's TMEM does not hold two accumulators, the one-block
    kernel or (fp32 V in two bf16 planes, when its plan does not fit) the CUDA
    cores."""
    ran = fs.fs_get_info(h)["last_apply_path"]
    if path == "simt":
        assert ran == "simt", ran
    elif path == "tc_pair":  # the pair's plan fits every operand width here up to dv = 256
        assert ran == "tc_pair", ran
    elif dv <= 128:
        assert ran == path, ran
    else:
        assert ran in ("tc", "simt"), ran
    return ran


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("dv", [1, 5, 33, 70, 256])
def test_transport_apply_parity(cuda_device, name, dv, path, monkeypatch):
    import torch
    _set_path(monkeypatch, path)
    fs = _fs()
    prob = make_problem(name, **SMALL[name])
    X, Y, a_d, b_d = device_inputs(prob)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps)
    f32, g32 = _potentials(prob, "sqeuclidean")
    rng = np.random.default_rng(100 + dv)
    V = rng.standard_normal((prob.batch, prob.m, dv)).astype(np.float32)
    out = torch.empty(prob.batch, prob.n, dv, device=cuda_device)
    r = torch.empty(prob.batch, prob.n, device=cuda_device)
    fs.fs_transport_apply(h, torch.from_numpy(f32).to(cuda_device), torch.from_numpy(g32).to(cuda_device),
                          torch.from_numpy(V).to(cuda_device), out, r)
    fs.fs_sync(h)
    ran = _assert_path(fs, h, path, dv)
    out, r = out.cpu().numpy(), r.cpu().numpy()
    for k, (Xo, Yo, loga, logb) in enumerate(oracle_arrays(prob)):
        fk, gk = f32[k].astype(np.float64), g32[k].astype(np.float64)
        oo, ro = oracle.transport_apply(Xo, Yo, loga, logb, fk, gk, prob.eps, V[k].astype(np.float64))
        absw, _ = oracle.transport_apply(Xo, Yo, loga, logb, fk, gk, prob.eps, np.abs(V[k]).astype(np.float64))
        rel = _rel_bound(Xo, Yo, loga, logb, fk, gk, prob.eps, "sqeuclidean") + SPLIT[path]
        err = np.abs(out[k] - oo) / (rel[:, None] * absw)
        rerr = np.abs(r[k] - ro) / (rel * ro)
        print(f"{path} ({ran}) {name}[{k}] dv={dv} worst err / bound = {err.max():.3f}, row sums {rerr.max():.3f}")
        assert err.max() <= 1.0 and rerr.max() <= 1.0


@pytest.mark.parametrize("tail", ["1", "0"])
@pytest.mark.parametrize("dv", [3, 64, 128])
def test_split_row_blocks_parity(cuda_device, dv, tail, monkeypatch):
    """More 128-row blocks than SMs in the one-row-block mode: the row blocks past
    the last full wave are split over their column tiles, one CTA per part, and a
    merge kernel adds the parts' sums (FS_APPLY_TAIL=0: every row block whole).
    n = 19500 gives 154 row blocks; on 148 SMs the last 6 split into 4 parts of
    two tiles (m = 1100: 9 tiles)."""
    import torch
    _set_path(monkeypatch, "tc_2s")
    monkeypatch.setenv("FS_APPLY_TAIL", tail)
    fs = _fs()
    prob = make_problem("cloud3d", n=19500, m=1100)
    X, Y, a_d, b_d = device_inputs(prob)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps)
    f32, g32 = _potentials(prob, "sqeuclidean", iters=4)
    rng = np.random.default_rng(300 + dv)
    V = rng.standard_normal((1, prob.m, dv)).astype(np.float32)
    out = torch.empty(1, prob.n, dv, device=cuda_device)
    r = torch.empty(1, prob.n, device=cuda_device)
    fd, gd = torch.from_numpy(f32).to(cuda_device), torch.from_numpy(g32).to(cuda_device)
    fs.fs_transport_apply(h, fd, gd, torch.from_numpy(V).to(cuda_device), out, r)
    fs.fs_sync(h)
    info = fs.fs_get_info(h)
    assert info["last_apply_path"] == "tc_2s", info
    blocks = (prob.n + 255) // 256 * 2
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    rem, ntiles = blocks % sms, (prob.m + 127) // 128
    parts = min(8, sms // rem, ntiles // 2) if rem else 1
    assert info["last_apply_parts"] == (parts if tail == "1" and parts > 1 else 1), (info, parts)
    T = torch.empty(1, prob.n, prob.d, device=cuda_device)
    fs.fs_barycentric_map(h, fd, gd, Y, T)
    fs.fs_sync(h)
    out, r, T = out.cpu().numpy()[0], r.cpu().numpy()[0], T.cpu().numpy()[0]
    Xo, Yo, loga, logb = oracle.problem_arrays(prob, 0)
    fk, gk = f32[0].astype(np.float64), g32[0].astype(np.float64)
    oo, ro = oracle.transport_apply(Xo, Yo, loga, logb, fk, gk, prob.eps, V[0].astype(np.float64))
    absw, _ = oracle.transport_apply(Xo, Yo, loga, logb, fk, gk, prob.eps, np.abs(V[0]).astype(np.float64))
    rel = _rel_bound(Xo, Yo, loga, logb, fk, gk, prob.eps, "sqeuclidean") + SPLIT["tc_2s"]
    err = (np.abs(out - oo) / (rel[:, None] * absw)).max()
    rerr = (np.abs(r - ro) / (rel * ro)).max()
    To = oracle.barycentric_projection(Xo, Yo, loga, logb, fk, gk, prob.eps)
    py, _ = oracle.transport_apply(Xo, Yo, loga, logb, fk, gk, prob.eps, np.abs(Yo))
    et = (np.abs(T - To) / (2 * rel[:, None] * py / ro[:, None] + 1e-6 * np.abs(To))).max()
    print(f"split row blocks (tail={tail}, parts {info['last_apply_parts']}) dv={dv}: "
          f"err / bound {err:.3f}, row sums {rerr:.3f}, barycentric {et:.3f}")
    assert err <= 1.0 and rerr <= 1.0 and et <= 1.0


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("name", ["tiny", "middim", "highdim", "batched"])
def test_barycentric_map_and_grad_parity(cuda_device, name, path, monkeypatch):
    import torch
    _set_path(monkeypatch, path)
    fs = _fs()
    prob = make_problem(name, **SMALL[name])
    X, Y, a_d, b_d = device_inputs(prob)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps)
    f32, g32 = _potentials(prob, "sqeuclidean", iters=30)
    fd, gd = torch.from_numpy(f32).to(cuda_device), torch.from_numpy(g32).to(cuda_device)
    T = torch.empty(prob.batch, prob.n, prob.d, device=cuda_device)
    G = torch.empty(prob.batch, prob.n, prob.d, device=cuda_device)
    fs.fs_barycentric_map(h, fd, gd, Y, T)
    fs.fs_grad_x(h, fd, gd, X, Y, G)
    fs.fs_sync(h)
    T, G = T.cpu().numpy(), G.cpu().numpy()
    for k, (Xo, Yo, loga, logb) in enumerate(oracle_arrays(prob)):
        fk, gk = f32[k].astype(np.float64), g32[k].astype(np.float64)
        To = oracle.barycentric_projection(Xo, Yo, loga, logb, fk, gk, prob.eps)
        Go = oracle.grad_x(Xo, Yo, loga, logb, fk, gk, prob.eps)
        py, r = oracle.transport_apply(Xo, Yo, loga, logb, fk, gk, prob.eps, np.abs(Yo))
        rel = (_rel_bound(Xo, Yo, loga, logb, fk, gk, prob.eps, "sqeuclidean") + SPLIT[path])[:, None]
        # T = (P Y)/r: both factors carry rel; G = 2 (r x - P Y)
        tb = 2 * rel * py / r[:, None] + 1e-6 * np.abs(To)
        gb = 2 * rel * (r[:, None] * np.abs(Xo) + py) + 2.0 ** -22 * np.abs(Go)
        et, eg = (np.abs(T[k] - To) / tb).max(), (np.abs(G[k] - Go) / gb).max()
        print(f"{path} {name}[{k}] barycentric err/bound {et:.3f}  grad err/bound {eg:.3f}")
        assert et <= 1.0 and eg <= 1.0


@pytest.mark.parametrize("path", list(PATHS))
def test_transport_apply_cosine_parity(cuda_device, path, monkeypatch):
    import torch
    _set_path(monkeypatch, path)
    fs = _fs()
    prob = make_problem("middim", n=1000, m=900)
    X, Y, a_d, b_d = device_inputs(prob)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps, cost="cosine")
    f32, g32 = _potentials(prob, "cosine")
    rng = np.random.default_rng(7)
    V = rng.standard_normal((1, prob.m, 9)).astype(np.float32)
    out = torch.empty(1, prob.n, 9, device=cuda_device)
    fs.fs_transport_apply(h, torch.from_numpy(f32).to(cuda_device), torch.from_numpy(g32).to(cuda_device),
                          torch.from_numpy(V).to(cuda_device), out)
    fs.fs_sync(h)
    Xo, Yo, loga, logb = oracle.problem_arrays(prob, 0)
    fk, gk = f32[0].astype(np.float64), g32[0].astype(np.float64)
    oo, _ = oracle.transport_apply(Xo, Yo, loga, logb, fk, gk, prob.eps, V[0].astype(np.float64), cost="cosine")
    absw, _ = oracle.transport_apply(Xo, Yo, loga, logb, fk, gk, prob.eps, np.abs(V[0]).astype(np.float64),
                                     cost="cosine")
    rel = _rel_bound(Xo, Yo, loga, logb, fk, gk, prob.eps, "cosine") + SPLIT[path]
    err = (np.abs(out.cpu().numpy()[0] - oo) / (rel[:, None] * absw)).max()
    print(f"cosine transport err / bound {err:.3f}")
    assert err <= 1.0


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("name", ["tiny", "middim", "highdim", "batched"])
def test_cosine_grad_parity(cuda_device, name, path, monkeypatch):
    """fs_grad_x and fs_grad_y under the cosine cost against the oracle's
    cosine gradients.  grad_i = -(b_i - (x^_i.b_i) x^_i) / |x_i| with b = P Y^:
    b carries the transport bound (rel times P |Y^|, per component), and the
    projection adds at most |x^_k| sum_l |db_l| |x^_l| to component k; the fp32
    normalisation and projection add 2^-20 of the terms' sizes."""
    import torch
    _set_path(monkeypatch, path)
    fs = _fs()
    prob = make_problem(name, **SMALL[name])
    X, Y, a_d, b_d = device_inputs(prob)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps, cost="cosine")
    f32, g32 = _potentials(prob, "cosine", iters=30)
    fd, gd = torch.from_numpy(f32).to(cuda_device), torch.from_numpy(g32).to(cuda_device)
    Gx = torch.empty(prob.batch, prob.n, prob.d, device=cuda_device)
    fs.fs_grad_x(h, fd, gd, X, Y, Gx)
    fs.fs_sync(h)
    ran_x = fs.fs_get_info(h)["last_apply_path"]
    Gy = torch.empty(prob.batch, prob.m, prob.d, device=cuda_device)
    fs.fs_grad_y(h, fd, gd, X, Y, Gy)
    fs.fs_sync(h)
    Gx, Gy = Gx.cpu().numpy(), Gy.cpu().numpy()
    if path == "simt":
        assert ran_x == "simt"
    for k, (Xo, Yo, loga, logb) in enumerate(oracle_arrays(prob)):
        fk, gk = f32[k].astype(np.float64), g32[k].astype(np.float64)
        rel = _rel_bound(Xo, Yo, loga, logb, fk, gk, prob.eps, "cosine") + SPLIT[path]
        relt = _rel_bound(Yo, Xo, logb, loga, gk, fk, prob.eps, "cosine") + SPLIT[path]
        Gxo = oracle.grad_x(Xo, Yo, loga, logb, fk, gk, prob.eps, cost="cosine")
        Gyo = oracle.grad_y(Xo, Yo, loga, logb, fk, gk, prob.eps, cost="cosine")
        for G, Go, own, other, lw_own, lw_oth, p_own, p_oth, rl, label in (
                (Gx[k], Gxo, Xo, Yo, loga, logb, fk, gk, rel, "x"),
                (Gy[k], Gyo, Yo, Xo, logb, loga, gk, fk, relt, "y")):
            rho = np.linalg.norm(own, axis=1)
            uh = own / rho[:, None]
            oh = other / np.linalg.norm(other, axis=1)[:, None]
            bsum, _ = oracle.transport_apply(own, other, lw_own, lw_oth, p_own, p_oth, prob.eps, oh, cost="cosine")
            babs, _ = oracle.transport_apply(own, other, lw_own, lw_oth, p_own, p_oth, prob.eps, np.abs(oh),
                                             cost="cosine")
            e = rl[:, None] * babs
            proj = np.sum(e * np.abs(uh), axis=1)[:, None] * np.abs(uh)
            size = np.abs(bsum) + np.sum(np.abs(bsum * uh), axis=1)[:, None] * np.abs(uh)
            gb = (e + proj + 2.0 ** -20 * size) / rho[:, None]
            err = (np.abs(G - Go) / gb).max()
            print(f"{path} {name}[{k}] cosine grad_{label} err/bound {err:.3f}")
            assert err <= 1.0


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("name", ["tiny", "cloud3d", "highdim", "batched"])
def test_transposed_apply_and_grad_y_parity(cuda_device, name, path, monkeypatch):
    """out_j = sum_i P_ij U_i and the gradient with respect to Y (the backward pass's
    second half) against the oracle, whose transposed forms exchange the two
    clouds' roles (C is symmetric)."""
    import torch
    _set_path(monkeypatch, path)
    fs = _fs()
    prob = make_problem(name, **SMALL[name])
    X, Y, a_d, b_d = device_inputs(prob)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps)
    f32, g32 = _potentials(prob, "sqeuclidean", iters=20)
    fd, gd = torch.from_numpy(f32).to(cuda_device), torch.from_numpy(g32).to(cuda_device)
    rng = np.random.default_rng(123)
    U = rng.standard_normal((prob.batch, prob.n, 7)).astype(np.float32)
    out = torch.empty(prob.batch, prob.m, 7, device=cuda_device)
    c = torch.empty(prob.batch, prob.m, device=cuda_device)
    G = torch.empty(prob.batch, prob.m, prob.d, device=cuda_device)
    fs.fs_transport_apply_t(h, fd, gd, torch.from_numpy(U).to(cuda_device), out, c)
    fs.fs_grad_y(h, fd, gd, X, Y, G)
    fs.fs_sync(h)
    out, c, G = out.cpu().numpy(), c.cpu().numpy(), G.cpu().numpy()
    for k, (Xo, Yo, loga, logb) in enumerate(oracle_arrays(prob)):
        fk, gk = f32[k].astype(np.float64), g32[k].astype(np.float64)
        oo, co = oracle.transport_apply(Yo, Xo, logb, loga, gk, fk, prob.eps, U[k].astype(np.float64))
        absw, _ = oracle.transport_apply(Yo, Xo, logb, loga, gk, fk, prob.eps, np.abs(U[k]).astype(np.float64))
        px, _ = oracle.transport_apply(Yo, Xo, logb, loga, gk, fk, prob.eps, np.abs(Xo))
        Go = oracle.grad_y(Xo, Yo, loga, logb, fk, gk, prob.eps)
        rel = _rel_bound(Yo, Xo, logb, loga, gk, fk, prob.eps, "sqeuclidean") + SPLIT[path]
        e1 = (np.abs(out[k] - oo) / (rel[:, None] * absw)).max()
        e2 = (np.abs(c[k] - co) / (rel * co)).max()
        gb = 2 * rel[:, None] * (co[:, None] * np.abs(Yo) + px) + 2.0 ** -22 * np.abs(Go)
        e3 = (np.abs(G[k] - Go) / gb).max()
        print(f"{path} {name}[{k}] transposed err/bound {e1:.3f} col sums {e2:.3f} grad_y {e3:.3f}")
        assert e1 <= 1.0 and e2 <= 1.0 and e3 <= 1.0


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("n,m,d", [(1, 1, 3), (1, 300, 5), (300, 1, 5), (129, 65, 2), (257, 200, 33), (2, 129, 4),
                                   (130, 385, 7)])
def test_transport_apply_edge_shapes(cuda_device, n, m, d, path, monkeypatch):
    """Single points, one-column plans and ragged row/column counts around the
    128-row blocks, the 128-column tiles and their 64-column halves (one valid
    column in the last tile, whole halves of padding)."""
    import torch
    _set_path(monkeypatch, path)
    fs = _fs()
    rng = np.random.default_rng(n * 1000 + m + d)
    Xo = rng.standard_normal((n, d))
    Yo = rng.standard_normal((m, d)) + 0.3
    X = torch.from_numpy(Xo.astype(np.float32)).to(cuda_device)
    Y = torch.from_numpy(Yo.astype(np.float32)).to(cuda_device)
    eps = 0.2
    h = fs.fs_create(X, Y, eps=eps)
    Xd, Yd = X.double().cpu().numpy(), Y.double().cpu().numpy()
    loga, logb = np.full(n, -np.log(n)), np.full(m, -np.log(m))
    f, g = oracle.solve(Xd, Yd, loga, logb, eps, 10)
    f32, g32 = f.astype(np.float32), g.astype(np.float32)
    V = rng.standard_normal((m, 3)).astype(np.float32)
    out = torch.empty(1, n, 3, device=cuda_device)
    r = torch.empty(1, n, device=cuda_device)
    fs.fs_transport_apply(h, torch.from_numpy(f32[None]).to(cuda_device), torch.from_numpy(g32[None]).to(cuda_device),
                          torch.from_numpy(V[None]).to(cuda_device), out, r)
    fs.fs_sync(h)
    _assert_path(fs, h, path, 3)
    oo, ro = oracle.transport_apply(Xd, Yd, loga, logb, f32.astype(np.float64), g32.astype(np.float64), eps,
                                    V.astype(np.float64))
    absw, _ = oracle.transport_apply(Xd, Yd, loga, logb, f32.astype(np.float64), g32.astype(np.float64), eps,
                                     np.abs(V).astype(np.float64))
    rel = _rel_bound(Xd, Yd, loga, logb, f32.astype(np.float64), g32.astype(np.float64), eps, "sqeuclidean") + \
        SPLIT[path]
    err = (np.abs(out.cpu().numpy()[0] - oo) / (rel[:, None] * absw)).max()
    rerr = (np.abs(r.cpu().numpy()[0] - ro) / (rel * ro)).max()
    assert err <= 1.0 and rerr <= 1.0, (err, rerr)


@pytest.mark.parametrize("name,prec", [("tiny", "3xtf32"), ("cloud3d", "3xtf32"), ("batched", "3xtf32")])
def test_transport_apply_tf32_kind(cuda_device, name, prec):
    """The tensor-core application with the S product on the tf32 tensor-core kind
    (3xTF32 split operands; the default for these fp32 workloads is 3xF16 on the
    f16 kind), 64- and 128-byte swizzled rows.  The split leaves a score error of
    about 2^-21 relative per product, 2 d 2^-21 max|q| max|k| in all, which adds
    to the exponent of every plan entry on top of the bound used above."""
    import torch
    fs = _fs()
    prob = make_problem(name, **SMALL[name])
    X, Y, a_d, b_d = device_inputs(prob)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps, prec=prec)
    f32, g32 = _potentials(prob, "sqeuclidean")
    rng = np.random.default_rng(7)
    V = rng.standard_normal((prob.batch, prob.m, 5)).astype(np.float32)
    out = torch.empty(prob.batch, prob.n, 5, device=cuda_device)
    fs.fs_transport_apply(h, torch.from_numpy(f32).to(cuda_device), torch.from_numpy(g32).to(cuda_device),
                          torch.from_numpy(V).to(cuda_device), out, None)
    fs.fs_sync(h)
    assert fs.fs_get_info(h)["last_apply_path"] in ("tc", "tc_q2", "tc_2s")
    out = out.cpu().numpy()
    u = 2.0 ** -21
    for k, (Xo, Yo, loga, logb) in enumerate(oracle_arrays(prob)):
        fk, gk = f32[k].astype(np.float64), g32[k].astype(np.float64)
        oo, _ = oracle.transport_apply(Xo, Yo, loga, logb, fk, gk, prob.eps, V[k].astype(np.float64))
        absw, _ = oracle.transport_apply(Xo, Yo, loga, logb, fk, gk, prob.eps, np.abs(V[k]).astype(np.float64))
        t = 0.5 * (Xo.mean(axis=0) + Yo.mean(axis=0))
        xs, ys = Xo - t, Yo - t
        # score error of the operand rounding, in the exponent (natural log units)
        ds = 2 * prob.d * u * np.abs(xs).max() * np.abs(ys).max() * 2 / prob.eps
        rel = _rel_bound(Xo, Yo, loga, logb, fk, gk, prob.eps, "sqeuclidean") + SPLIT["tc"] + 2 * ds
        err = (np.abs(out[k] - oo) / (rel[:, None] * absw)).max()
        print(f"{prec} {name}[{k}] worst err / bound = {err:.3f}")
        assert err <= 1.0


@pytest.mark.parametrize("case", ["f32-d128-auto", "f32-d64-3xtf32", "cosine-d128-auto", "bf16-d256-auto"])
def test_transport_apply_wide_rows_on_cta_pairs(cuda_device, case, monkeypatch):
    """Handles whose packed operand rows are 512 bytes run their passes on CTA pairs; their
    transport application must run on the tensor cores too, by default, within the same
    bound: fp32 clouds at d = 128 (3xF16), 3xTF32 at d = 64, the cosine cost at d = 128,
    and bf16 clouds at d = 256 (one plane of 256 values).  Every one of these forms the
    score to about fp32 accuracy, which the bound assumes (one-pass TF32 does not)."""
    import torch
    monkeypatch.setenv("FS_APPLY_VEC", "0")  # dv = 1 through the pair kernel too
    fs = _fs()
    kind, dim, prec = case.split("-")
    name = "middim" if dim == "d64" else "highdim"
    prob = make_problem(name, **SMALL[name], **({"d": 256} if dim == "d256" else {}))
    cost = "cosine" if kind == "cosine" else "sqeuclidean"
    if kind == "bf16":
        X, Y, a_d, b_d = device_inputs(prob)
    else:
        # fp32 inputs (for highdim, the recipe's bf16 values, exactly)
        X = torch.from_numpy(prob.X[0].astype(np.float32))[None].to(cuda_device)
        Y = torch.from_numpy(prob.Y[0].astype(np.float32))[None].to(cuda_device)
        _, _, a_d, b_d = device_inputs(prob)
    kw = {} if prec == "auto" else {"prec": prec}
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps, cost=cost, **kw)
    info = fs.fs_get_info(h)
    assert info["cta_pair"] == 1 and info["row_bytes"] == 512, info
    f32, g32 = _potentials(prob, cost)
    rng = np.random.default_rng(321)
    for dv in (1, 64, 130):
        V = rng.standard_normal((1, prob.m, dv)).astype(np.float32)
        out = torch.empty(1, prob.n, dv, device=cuda_device)
        r = torch.empty(1, prob.n, device=cuda_device)
        fs.fs_transport_apply(h, torch.from_numpy(f32).to(cuda_device), torch.from_numpy(g32).to(cuda_device),
                              torch.from_numpy(V).to(cuda_device), out, r)
        fs.fs_sync(h)
        assert fs.fs_get_info(h)["last_apply_path"] == "tc_pair"
        Xo, Yo, loga, logb = oracle_arrays(prob)[0]
        fk, gk = f32[0].astype(np.float64), g32[0].astype(np.float64)
        oo, ro = oracle.transport_apply(Xo, Yo, loga, logb, fk, gk, prob.eps, V[0].astype(np.float64), cost=cost)
        absw, _ = oracle.transport_apply(Xo, Yo, loga, logb, fk, gk, prob.eps, np.abs(V[0]).astype(np.float64),
                                         cost=cost)
        rel = _rel_bound(Xo, Yo, loga, logb, fk, gk, prob.eps, cost) + 2.0 ** -14
        err = np.abs(out.cpu().numpy()[0] - oo) / (rel[:, None] * absw)
        rerr = np.abs(r.cpu().numpy()[0] - ro) / (rel * ro)
        print(f"{case} dv={dv}: worst err / bound = {err.max():.3f}, row sums {rerr.max():.3f}")
        assert err.max() <= 1.0 and rerr.max() <= 1.0


@pytest.mark.parametrize("transposed", [False, True])
@pytest.mark.parametrize("name", list(SMALL))
def test_one_column_through_the_lse_pass(cuda_device, name, transposed, monkeypatch):
    """dv = 1 on a tensor-core handle runs as a streamed LSE pass weighting each
    column by V_j (last_apply_path "lse_vec"): (P v)_i = r_i w_i / l_i with the
    running max, fp32 sums and no bf16 split, so the CUDA-core bound applies
    (no 2^-14 term)."""
    import torch
    monkeypatch.delenv("FS_APPLY_VEC", raising=False)
    monkeypatch.delenv("FS_APPLY_SIMT", raising=False)
    fs = _fs()
    prob = make_problem(name, **SMALL[name])
    X, Y, a_d, b_d = device_inputs(prob)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps)
    f32, g32 = _potentials(prob, "sqeuclidean")
    rng = np.random.default_rng(555)
    cnt_in, cnt_out = (prob.n, prob.m) if transposed else (prob.m, prob.n)
    V = rng.standard_normal((prob.batch, cnt_in, 1)).astype(np.float32)
    out = torch.empty(prob.batch, cnt_out, 1, device=cuda_device)
    r = torch.empty(prob.batch, cnt_out, device=cuda_device)
    fd, gd, Vd = (torch.from_numpy(x).to(cuda_device) for x in (f32, g32, V))
    if transposed:
        fs.fs_transport_apply_t(h, fd, gd, Vd, out, r)
    else:
        fs.fs_transport_apply(h, fd, gd, Vd, out, r)
    fs.fs_sync(h)
    assert fs.fs_get_info(h)["last_apply_path"] == "lse_vec"
    out, r = out.cpu().numpy(), r.cpu().numpy()
    for k, (Xo, Yo, loga, logb) in enumerate(oracle_arrays(prob)):
        fk, gk = f32[k].astype(np.float64), g32[k].astype(np.float64)
        if transposed:  # P^T v: the transposed problem's rows are Y's points
            args = (Yo, Xo, logb, loga, gk, fk)
        else:
            args = (Xo, Yo, loga, logb, fk, gk)
        oo, ro = oracle.transport_apply(*args, prob.eps, V[k].astype(np.float64))
        absw, _ = oracle.transport_apply(*args, prob.eps, np.abs(V[k]).astype(np.float64))
        rel = _rel_bound(*args, prob.eps, "sqeuclidean")
        err = (np.abs(out[k] - oo) / (rel[:, None] * absw)).max()
        rerr = (np.abs(r[k] - ro) / (rel * ro)).max()
        print(f"{name}[{k}] transposed={transposed}: worst err / bound {err:.3f}, row sums {rerr:.3f}")
        assert err <= 1.0 and rerr <= 1.0
