"""Streaming Hessian-vector product of the entropic OT cost with respect to X
(fs_hvp_x; "FlashSinkhorn: IO-aware EOT on GPU", Metodologia section 3) against
the dense oracle (explicit plan, exact linear solve), at potentials the oracle
converged and rounded to float32 (the same bytes on both sides).

Bound: each transport product carries the relative error of the transport
application (about 2^-14 on the tensor-core path, its bf16 splits), the
conjugate-gradient solve stops at a relative residual of 1e-7, and the final
combination subtracts terms of size (2/eps) max|x| |P Y| from each other.  The
test takes |H_gpu - H_oracle| <= 2^-8 max|H_oracle| + 2^-12 (2/eps) S, with
S = max_i sum_j P_ij |x_i - y_j|^2 |v_i| the size of the largest of those terms.
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
}


@pytest.mark.parametrize("path", ["tc", "simt"])
@pytest.mark.parametrize("name", list(CASES))
def test_hvp_x_parity(cuda_device, name, path, monkeypatch):
    import torch
    monkeypatch.setenv("FS_APPLY_SIMT", "1" if path == "simt" else "0")
    import log_domain_sinkhorn_updates_b200 as fs
    from helpers import device_inputs
    prob = make_problem(name, **CASES[name])
    X, Y, a_d, b_d = device_inputs(prob)
    Xo, Yo, loga, logb = oracle.problem_arrays(prob, 0)
    f, g = oracle.solve(Xo, Yo, loga, logb, prob.eps, 400)
    f32, g32 = f.astype(np.float32), g.astype(np.float32)
    rng = np.random.default_rng(200)
    V = rng.standard_normal((prob.n, prob.d)).astype(np.float32)
    h = fs.fs_create(X, Y, a_d, b_d, eps=prob.eps)
    out = torch.empty(1, prob.n, prob.d, device=cuda_device)
    its = fs.fs_hvp_x(h, torch.from_numpy(f32[None]).to(cuda_device), torch.from_numpy(g32[None]).to(cuda_device),
                      X, Y, torch.from_numpy(V[None]).to(cuda_device), out, max_cg_iters=500, cg_rtol=1e-7)
    fs.fs_sync(h)
    H = out.cpu().numpy()[0]
    Ho = dense.hvp_x(Xo, Yo, loga, logb, f32.astype(np.float64), g32.astype(np.float64), prob.eps,
                     V.astype(np.float64))
    P = dense.plan(dense.cost_matrix(Xo, Yo), loga, logb, f32.astype(np.float64), g32.astype(np.float64), prob.eps)
    S = (P * dense.cost_matrix(Xo, Yo)).sum(axis=1) * np.abs(V).max(axis=1)
    bound = 2.0 ** -8 * np.abs(Ho).max() + 2.0 ** -12 * (2.0 / prob.eps) * S.max()
    err = np.abs(H - Ho).max()
    print(f"{path} {name}: cg steps {its}, max|dH| = {err:.3e}, bound {bound:.3e}, max|H| = {np.abs(Ho).max():.3e}")
    assert err <= bound
