"""Streaming Hessian-vector product of the entropic OT cost with respect to X
(fs_hvp_x; "FlashSinkhorn: IO-aware EOT on GPU", Metodologia section 3) against
the dense oracle (explicit plan, exact linear solve), at potentials the oracle
converged and rounded to float32 (the same bytes on both sides).

Bound, per row i:  |H_gpu,i - H_oracle,i| <= 2^-14 (2/eps) S_i + 2^-10 max|H|,
with S_i = sum_j P_ij |x_i - y_j|^2 max_k |v_ik| the size of the largest term the
final combination subtracts (all of them are plan-weighted averages of
(2/eps) |x_i - y_j|^2 |v_i|-sized quantities).
* 2^-14 is the relative error of one transport product on the tensor-core
  path (its bf16 hi/lo splits; the CUDA-core path is more accurate), measured
  against the absolute size of what it sums.
* 2^-10 max|H| bounds what the conjugate-gradient solve of the potentials'
  response adds: it stops at a relative residual of 1e-7, but every operator
  application carries the 2^-14 product error, which the solve amplifies by the
  conditioning of the reduced system (at most 16 here).
The cases include the recipes' own dimensions, d = 64 (3xF16 operands) and
d = 128 (bf16 operands).  Three paths each: the tensor-core default, where the
transport-matrix term sum_j P_ij (v_i . y_j) y_j is one fused pass (a second
score v_i . y_j against the same K tile); the same term as d / nq transport
applications of column blocks of y (FS_HVP_FUSED=0); and the CUDA-core
validation kernels (FS_APPLY_SIMT=1).
"""
import numpy as np
import pytest

import oracle
from oracle import dense
from helpers import make_problem

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": dict(n=300, m=280),
    "cloud3d": dict(n=320, m=300),
    "middim": dict(n=260, m=240, d=16),
    "highdim": dict(n=256, m=240, d=16),
    # the recipes' own dimensions: d = 64 (3xF16 operands, two columns of y per
    # transport-matrix product) and d = 128 (bf16 operands, one column per product)
    "middim-d64": dict(n=512, m=480),
    "highdim-d128": dict(n=512, m=480),
}


PATHS = {"tc": ("0", "1"), "tc_blocked": ("0", "0"), "simt": ("1", "0")}  # (FS_APPLY_SIMT, FS_HVP_FUSED)


BATCHED = {
    # independent problems in one call, each with its own CG: the batched recipe
    # at d = 32 (3xF16 operands) and the highdim recipe at d = 128 (bf16 operands)
    "batched-b3": dict(batch=3, n=300, m=260),
    "highdim-b2": dict(batch=2, n=256, m=240),
}


def _oracle_case(prob, k, cost="sqeuclidean"):
    Xo, Yo, loga, logb = oracle.problem_arrays(prob, k)
    f, g = oracle.solve(Xo, Yo, loga, logb, prob.eps, 400, cost=cost)
    return Xo, Yo, loga, logb, f.astype(np.float32), g.astype(np.float32)


def _check_row_bound(path, name, its, H, Xo, Yo, loga, logb, f32, g32, eps, V):
    Ho = dense.hvp_x(Xo, Yo, loga, logb, f32.astype(np.float64), g32.astype(np.float64), eps, V.astype(np.float64))
    P = dense.plan(dense.cost_matrix(Xo, Yo), loga, logb, f32.astype(np.float64), g32.astype(np.float64), eps)
    S = (P * dense.cost_matrix(Xo, Yo)).sum(axis=1) * np.abs(V).max(axis=1)
    bound = 2.0 ** -14 * (2.0 / eps) * S + 2.0 ** -10 * np.abs(Ho).max()
    err = np.abs(H - Ho).max()
    rowerr = np.abs(H - Ho).max(axis=1)
    print(f"{path} {name}: cg steps {its}, max|dH| = {err:.3e}, worst row err / bound {(rowerr / bound).max():.3f}, "
          f"max|H| = {np.abs(Ho).max():.3e}, "
          f"max_i |dH_i| / ((2/eps) S_i) = {(rowerr / ((2.0 / eps) * S)).max():.3e}, "
          f"max|dH| / max|H| = {err / np.abs(Ho).max():.3e}")
    assert np.all(rowerr <= bound), (rowerr / bound).max()


def _run_hvp(cuda_device, prob, cases, V, path, cost="sqeuclidean", max_cg_iters=500, cg_rtol=1e-7):
    import torch
    import log_domain_sinkhorn_updates_b200 as fs
    from helpers import device_inputs
    X, Y, a_d, b_d = device_inputs(prob)
    f_all = np.stack([c[4] for c in cases])
    g_all = np.stack([c[5] for c in cases])
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps, cost=cost)
    out = torch.empty(prob.batch, prob.n, prob.d, device=cuda_device)
    its = fs.fs_hvp_x(h, torch.from_numpy(f_all).to(cuda_device), torch.from_numpy(g_all).to(cuda_device),
                      X, Y, torch.from_numpy(V).to(cuda_device), out, max_cg_iters=max_cg_iters, cg_rtol=cg_rtol)
    fs.fs_sync(h)
    info = fs.fs_get_info(h)
    fs.fs_destroy(h)
    if path != "simt":
        assert info["last_apply_path"] in ("tc", "tc_q2", "tc_2s", "tc_pair")
    assert info["last_hvp_fused"] == (1 if path == "tc" and cost == "sqeuclidean" else 0), info
    return out.cpu().numpy(), its


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("name", list(CASES))
def test_hvp_x_parity(cuda_device, name, path, monkeypatch):
    monkeypatch.setenv("FS_APPLY_SIMT", PATHS[path][0])
    monkeypatch.setenv("FS_HVP_FUSED", PATHS[path][1])
    prob = make_problem(name.split("-")[0], **CASES[name])
    case = _oracle_case(prob, 0)
    rng = np.random.default_rng(200)
    V = rng.standard_normal((1, prob.n, prob.d)).astype(np.float32)
    H, its = _run_hvp(cuda_device, prob, [case], V, path)
    _check_row_bound(path, name, its, H[0], *case[:4], case[4], case[5], prob.eps, V[0])


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("name", list(BATCHED))
def test_hvp_x_batched_parity(cuda_device, name, path, monkeypatch):
    """Every problem of a batch against its own dense oracle HVP; the problems'
    CG solves stop at different steps, and the call's count is the largest."""
    monkeypatch.setenv("FS_APPLY_SIMT", PATHS[path][0])
    monkeypatch.setenv("FS_HVP_FUSED", PATHS[path][1])
    prob = make_problem(name.split("-")[0], **BATCHED[name])
    cases = [_oracle_case(prob, k) for k in range(prob.batch)]
    rng = np.random.default_rng(201)
    V = rng.standard_normal((prob.batch, prob.n, prob.d)).astype(np.float32)
    H, its = _run_hvp(cuda_device, prob, cases, V, path)
    assert 1 <= its <= 500
    for k, case in enumerate(cases):
        _check_row_bound(path, f"{name}[{k}]", its, H[k], *case[:4], case[4], case[5], prob.eps, V[k])


@pytest.mark.parametrize("path", ["tc", "simt"])
def test_hvp_x_long_cg_in_graph_blocks(cuda_device, path, monkeypatch):
    """A CG held to a residual fp32 cannot reach (1e-12) runs to its step limit:
    past the first 64 steps it goes in blocks of 8 that replay one captured CUDA
    graph.  The result must stay within the same bound, and the call must report
    the limit as its step count."""
    monkeypatch.setenv("FS_APPLY_SIMT", PATHS[path][0])
    monkeypatch.setenv("FS_HVP_FUSED", PATHS[path][1])
    prob = make_problem("middim", n=260, m=240, d=16)
    case = _oracle_case(prob, 0)
    rng = np.random.default_rng(202)
    V = rng.standard_normal((1, prob.n, prob.d)).astype(np.float32)
    H, its = _run_hvp(cuda_device, prob, [case], V, path, max_cg_iters=96, cg_rtol=1e-12)
    assert its == 96, its
    _check_row_bound(path, "middim long CG", its, H[0], *case[:4], case[4], case[5], prob.eps, V[0])


COSINE = {
    # the cosine cost: fp32 d = 16 (3xF16, 64-byte rows), bf16 d = 128 (3xF16 at
    # 512-byte rows, the CTA-pair kernels) and a batch of two at d = 32
    "middim-d16": dict(n=260, m=240, d=16),
    "highdim-d128": dict(n=256, m=240),
    "batched-b2": dict(batch=2, n=200, m=180),
}


@pytest.mark.parametrize("path", ["tc_blocked", "simt"])
@pytest.mark.parametrize("name", list(COSINE))
def test_hvp_x_cosine_parity(cuda_device, name, path, monkeypatch):
    """The cosine-cost HVP against the dense oracle (per-pair first and second
    derivatives of the cosine distance).  Same form of bound as above, with
    S_i = sum_j P_ij |D_ij|^2 max_k |v_ik| and D_ij = dC_ij/dx_i: the size of the
    (1/eps) dC_ij D_ij terms the final combination sums (for the squared
    Euclidean cost, |D|^2 = 4 |x - y|^2 and this is the bound above)."""
    monkeypatch.setenv("FS_APPLY_SIMT", PATHS[path][0])
    monkeypatch.setenv("FS_HVP_FUSED", PATHS[path][1])
    prob = make_problem(name.split("-")[0], **COSINE[name])
    cases = [_oracle_case(prob, k, "cosine") for k in range(prob.batch)]
    rng = np.random.default_rng(202)
    V = rng.standard_normal((prob.batch, prob.n, prob.d)).astype(np.float32)
    H, its = _run_hvp(cuda_device, prob, cases, V, path, cost="cosine")
    for k, (Xo, Yo, loga, logb, f32, g32) in enumerate(cases):
        f64, g64 = f32.astype(np.float64), g32.astype(np.float64)
        Ho = dense.hvp_x(Xo, Yo, loga, logb, f64, g64, prob.eps, V[k].astype(np.float64), cost="cosine")
        P = dense.plan(dense.cost_matrix(Xo, Yo, "cosine"), loga, logb, f64, g64, prob.eps)
        D2 = np.sum(dense.cost_grad_x(Xo, Yo, "cosine") ** 2, axis=2)
        S = (P * D2).sum(axis=1) * np.abs(V[k]).max(axis=1)
        bound = 2.0 ** -14 * S / prob.eps + 2.0 ** -10 * np.abs(Ho).max()
        rowerr = np.abs(H[k] - Ho).max(axis=1)
        print(f"{path} cosine {name}[{k}]: cg steps {its}, worst row err / bound {(rowerr / bound).max():.3f}, "
              f"max|dH| / max|H| = {rowerr.max() / np.abs(Ho).max():.3e}, "
              f"max_i |dH_i| / (S_i / eps) = {(rowerr / (S / prob.eps)).max():.3e}")
        assert np.all(rowerr <= bound), (rowerr / bound).max()
