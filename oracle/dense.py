"""Dense brute-force entropic OT on a materialised cost matrix (tiny inputs only).

TEST INFRASTRUCTURE ONLY.  An implementation independent of ``oracle.core``
(numpy broadcasting and ``scipy.special.logsumexp`` instead of streamed C),
used to pin it.  Also holds the textbook kernel-domain (scaling) form of
Sinkhorn's algorithm, which reaches the same potentials without any
log-sum-exp, and the closed-form solution of the 2x2 problem.
"""
from __future__ import annotations

import numpy as np
from scipy.special import logsumexp


def cost_matrix(X, Y, cost="sqeuclidean"):
    """C_ij = |x_i - y_j|^2 from the differences (broadcast, n*m*d doubles), or
    for cost="cosine" C_ij = 1 - x_i.y_j / (|x_i| |y_j|) (matrix product of the
    raw vectors, divided by the outer product of their norms)."""
    X = np.asarray(X, dtype=np.float64)
    Y = np.asarray(Y, dtype=np.float64)
    if cost == "cosine":
        nx = np.sqrt(np.sum(X * X, axis=1))
        ny = np.sqrt(np.sum(Y * Y, axis=1))
        return 1.0 - (X @ Y.T) / (nx[:, None] * ny[None, :])
    if cost != "sqeuclidean":
        raise ValueError(f"unknown cost {cost!r}")
    diff = X[:, None, :] - Y[None, :, :]
    return np.einsum("ijk,ijk->ij", diff, diff)


def update_f(C, logb, g, eps):
    return -eps * logsumexp((g[None, :] - C) / eps + logb[None, :], axis=1)


def update_g(C, loga, f, eps):
    return -eps * logsumexp((f[:, None] - C) / eps + loga[:, None], axis=0)


def solve(C, loga, logb, eps, iters, g0=None):
    g = np.zeros(C.shape[1]) if g0 is None else np.array(g0, dtype=np.float64)
    f = np.zeros(C.shape[0])
    for _ in range(iters):
        f = update_f(C, logb, g, eps)
        g = update_g(C, loga, f, eps)
    return f, g


def plan(C, loga, logb, f, g, eps):
    """P_ij = a_i b_j exp((f_i + g_j - C_ij)/eps)."""
    return np.exp(loga[:, None] + logb[None, :] + (f[:, None] + g[None, :] - C) / eps)


def costs(C, loga, logb, f, g, eps):
    P = plan(C, loga, logb, f, g, eps)
    a, b = np.exp(loga), np.exp(logb)
    sum_p = P.sum()
    ab = a[:, None] * b[None, :]
    kl = float(np.sum(P * np.log(P / ab)) - sum_p + 1.0)
    primal = float(np.sum(P * C))
    return dict(dual=float(a @ f + b @ g - eps * (sum_p - 1.0)), primal=primal,
                entropic_primal=primal + eps * kl, sum_p=float(sum_p))


def scaling_sinkhorn(C, a, b, eps, iters):
    """Textbook matrix-scaling Sinkhorn (Cuturi 2013): K = exp(-C/eps),
    u <- a / (K v), v <- b / (K^T u), starting from v = b.

    The plan is diag(u) K diag(v); in the potentials' parametrisation
    P_ij = a_i b_j exp((f_i + g_j - C_ij)/eps) this is f = eps log(u/a),
    g = eps log(v/b).  Only usable where exp(-C/eps) does not underflow.
    """
    K = np.exp(-C / eps)
    v = np.array(b, dtype=np.float64)
    u = np.ones_like(a)
    for _ in range(iters):
        u = a / (K @ v)
        v = b / (K.T @ u)
    return eps * np.log(u / a), eps * np.log(v / b)


def two_by_two_plan(C, a1, b1, eps):
    """Exact entropic-OT plan for n = m = 2.

    With both marginals fixed, the plan has one free entry p = P_11:
    P = [[p, a1-p], [b1-p, 1-a1-b1+p]].  Optimality of the entropic problem
    (P = diag(u) K diag(v)) forces the cross ratio
    P_11 P_22 / (P_12 P_21) = K_11 K_22 / (K_12 K_21) = kappa, a quadratic in p
    whose root inside the feasible interval is the unique optimum.
    """
    kappa = np.exp(-(C[0, 0] + C[1, 1] - C[0, 1] - C[1, 0]) / eps)
    A = 1.0 - kappa
    B = 1.0 - a1 - b1 + kappa * (a1 + b1)
    Cc = -kappa * a1 * b1
    lo, hi = max(0.0, a1 + b1 - 1.0), min(a1, b1)
    if abs(A) < 1e-300:
        roots = [-Cc / B]
    else:
        disc = np.sqrt(B * B - 4 * A * Cc)
        roots = [(-B + disc) / (2 * A), (-B - disc) / (2 * A)]
    p = [r for r in roots if lo - 1e-15 <= r <= hi + 1e-15]
    assert len(p) >= 1, (roots, lo, hi)
    p = p[0]
    return np.array([[p, a1 - p], [b1 - p, 1.0 - a1 - b1 + p]])


def cost_grad_x(X, Y, cost="sqeuclidean"):
    """Per-pair gradients dC_ij/dx_i [n, m, d], written out from the definition of C:
    2 (x_i - y_j) for the squared Euclidean cost; for the cosine cost,
    d/dx (1 - x.y/(|x| |y|)) = -(y^ - (x^.y^) x^) / |x| (x^ = x/|x|, y^ = y/|y|)."""
    X = np.asarray(X, dtype=np.float64)
    Y = np.asarray(Y, dtype=np.float64)
    if cost == "cosine":
        nx = np.linalg.norm(X, axis=1)
        Xh, Yh = X / nx[:, None], Y / np.linalg.norm(Y, axis=1)[:, None]
        s = Xh @ Yh.T
        return -(Yh[None, :, :] - s[:, :, None] * Xh[:, None, :]) / nx[:, None, None]
    return 2.0 * (X[:, None, :] - Y[None, :, :])


def cost_hess_x(X, Y, V, cost="sqeuclidean"):
    """Per-pair Hessian-vector products (d^2 C_ij/dx_i^2) v_i [n, m, d].  Squared
    Euclidean: 2 v_i.  Cosine, differentiating the gradient above once more
    along v (s = x^.y^, |x| = rho):
      [ (y^.v) x^ + s v + (x^.v) y^ - 3 s (x^.v) x^ ] / rho^2."""
    X = np.asarray(X, dtype=np.float64)
    Y = np.asarray(Y, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    n, m = X.shape[0], Y.shape[0]
    if cost == "cosine":
        nx = np.linalg.norm(X, axis=1)
        Xh, Yh = X / nx[:, None], Y / np.linalg.norm(Y, axis=1)[:, None]
        s = Xh @ Yh.T                                  # [n, m]
        yv = V @ Yh.T                                  # y^_j . v_i
        xv = np.sum(Xh * V, axis=1)                    # x^_i . v_i
        H = (yv[:, :, None] * Xh[:, None, :] + s[:, :, None] * V[:, None, :] +
             xv[:, None, None] * Yh[None, :, :] - 3.0 * (s * xv[:, None])[:, :, None] * Xh[:, None, :])
        return H / (nx ** 2)[:, None, None]
    return np.broadcast_to(2.0 * V[:, None, :], (n, m, X.shape[1])).copy()


def hvp_x(X, Y, loga, logb, f, g, eps, V, cost="sqeuclidean"):
    """Hessian-vector product of the entropic OT cost with respect to the positions X
    at optimal potentials (f, g), in direction V [n, d].

    The gradient is G_i = sum_j P_ij D_ij, D_ij = dC_ij/dx_i (2 (x_i - y_j) for
    the squared Euclidean cost).  Moving X along V changes P directly through C
    (dC_ij = D_ij.v_i) and through the potentials, whose response (df, dg) keeps
    both marginals fixed:
        r_i df_i + (P dg)_i   = sum_j P_ij dC_ij
        (P^T df)_j + c_j dg_j = sum_i P_ij dC_ij
    (a singular system: (k, -k) is free and does not change the result).  Then
        dG_i = sum_j P_ij (d^2 C_ij/dx_i^2) v_i + (1/eps) sum_j P_ij (df_i + dg_j - dC_ij) D_ij
    (2 r_i v_i for the first sum at the squared Euclidean cost).  Everything here
    is dense (tiny inputs only): P and the per-pair derivatives materialised,
    the linear system solved by least squares.
    """
    X = np.asarray(X, dtype=np.float64)
    Y = np.asarray(Y, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    P = plan(cost_matrix(X, Y, cost), np.asarray(loga, float), np.asarray(logb, float), np.asarray(f, float),
             np.asarray(g, float), eps)
    n, m = P.shape
    D = cost_grad_x(X, Y, cost)
    dC = np.einsum("ijk,ik->ij", D, V)
    r, c = P.sum(axis=1), P.sum(axis=0)
    A = np.zeros((n + m, n + m))
    A[:n, :n] = np.diag(r)
    A[:n, n:] = P
    A[n:, :n] = P.T
    A[n:, n:] = np.diag(c)
    rhs = np.concatenate([(P * dC).sum(axis=1), (P * dC).sum(axis=0)])
    sol = np.linalg.lstsq(A, rhs, rcond=None)[0]
    df, dg = sol[:n], sol[n:]
    W = P * (df[:, None] + dg[None, :] - dC)
    return np.einsum("ij,ijk->ik", P, cost_hess_x(X, Y, V, cost)) + np.einsum("ij,ijk->ik", W, D) / eps
