"""Pins of the CPU oracle against things other than itself.

The pages print no worked example, so the oracle is pinned to:
  * a library routine (scipy's cdist for the cost matrix),
  * an independent dense brute force (numpy + scipy logsumexp),
  * the textbook matrix-scaling form of Sinkhorn (no log-sum-exp at all),
  * closed forms (n = m = 1; the exact 2x2 entropic plan; the large-eps expansion),
  * exact inequalities (the hard c-transform sandwich), exact marginal identities,
    monotone dual ascent, vanishing duality gap,
  * symmetries (swap, gauge, translation, permutation, scaling).
A planted-mistake test at the end shows each plausible slip fails at least one pin.
"""
import numpy as np
import pytest
from scipy.spatial.distance import cdist

import oracle
from oracle import dense

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rand_problem(n, m, d, seed, uniform=False, scale=1.0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((n, d)) * scale
    Y = rng.standard_normal((m, d)) * scale + 0.3
    if uniform:
        a = np.full(n, 1.0 / n)
        b = np.full(m, 1.0 / m)
    else:
        a = rng.uniform(0.5, 1.5, n)
        a /= a.sum()
        b = rng.uniform(0.5, 1.5, m)
        b /= b.sum()
    return X, Y, np.log(a), np.log(b)


def test_cost_matrix_matches_scipy_cdist():
    X, Y, _, _ = _rand_problem(17, 23, 6, 1)
    C = dense.cost_matrix(X, Y)
    np.testing.assert_allclose(C, cdist(X, Y, "sqeuclidean"), rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("n,m,d", [(37, 53, 5), (1, 9, 3), (64, 1, 2), (40, 40, 128)])
def test_streaming_update_matches_dense(n, m, d):
    X, Y, loga, logb = _rand_problem(n, m, d, 2 + n + m)
    rng = np.random.default_rng(7)
    g = rng.standard_normal(m)
    f0 = rng.standard_normal(n)
    eps = 0.3
    C = dense.cost_matrix(X, Y)
    np.testing.assert_allclose(oracle.update_f(X, Y, logb, g, eps), dense.update_f(C, logb, g, eps),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.update_g(X, Y, loga, f0, eps), dense.update_g(C, loga, f0, eps),
                               rtol=1e-12, atol=1e-12)
    rows = np.array([0, n - 1, n // 2])
    np.testing.assert_allclose(oracle.update_f_rows(rows, X, Y, logb, g, eps),
                               dense.update_f(C, logb, g, eps)[rows], rtol=1e-12, atol=1e-12)


def test_solve_matches_dense_and_plan_stats():
    X, Y, loga, logb = _rand_problem(30, 45, 4, 3)
    eps = 0.2
    f, g = oracle.solve(X, Y, loga, logb, eps, 25)
    C = dense.cost_matrix(X, Y)
    fd, gd = dense.solve(C, loga, logb, eps, 25)
    np.testing.assert_allclose(f, fd, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(g, gd, rtol=1e-11, atol=1e-11)
    r, c = oracle.marginals(X, Y, loga, logb, f, g, eps)
    P = dense.plan(C, loga, logb, f, g, eps)
    np.testing.assert_allclose(r, P.sum(1), rtol=1e-12)
    np.testing.assert_allclose(c, P.sum(0), rtol=1e-12)
    co = oracle.costs(X, Y, loga, logb, f, g, eps)
    cd = dense.costs(C, loga, logb, f, g, eps)
    for k in ("dual", "primal", "entropic_primal", "sum_p"):
        assert abs(co[k] - cd[k]) <= 1e-12 * max(1.0, abs(cd[k])), k
    assert co["max_cost"] == pytest.approx(C.max(), rel=1e-14)
    assert co["min_cost"] == pytest.approx(C.min(), rel=1e-12, abs=1e-14)


@pytest.mark.parametrize("uniform", [True, False])
def test_matches_textbook_scaling_sinkhorn(uniform):
    """Log-domain potentials equal eps*log of the scaling vectors of Cuturi's form."""
    X, Y, loga, logb = _rand_problem(25, 31, 3, 4, uniform=uniform, scale=0.7)
    eps = 0.5
    f, g = oracle.solve(X, Y, loga, logb, eps, 40)
    fs, gs = dense.scaling_sinkhorn(dense.cost_matrix(X, Y), np.exp(loga), np.exp(logb), eps, 40)
    np.testing.assert_allclose(f, fs, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(g, gs, rtol=1e-10, atol=1e-10)


def test_single_point_closed_form():
    """n = m = 1: one update from g gives f = C_11 - g; from g = 0 the solve is at its
    fixed point f = C_11, g = 0 with zero marginal error and dual cost C_11."""
    X = np.array([[0.3, -1.2, 2.0]])
    Y = np.array([[1.1, 0.4, -0.5]])
    C11 = float(((X - Y) ** 2).sum())
    z = np.zeros(1)
    for eps in (0.01, 0.1, 3.0):
        assert oracle.update_f(X, Y, z, np.array([0.7]), eps)[0] == pytest.approx(C11 - 0.7, rel=1e-15)
        f, g = oracle.solve(X, Y, z, z, eps, 5)
        assert f[0] == pytest.approx(C11, rel=1e-15)
        assert g[0] == pytest.approx(0.0, abs=1e-15)
        er, ec = oracle.marginal_error(X, Y, z, z, f, g, eps)
        assert er == pytest.approx(0.0, abs=1e-15) and ec == pytest.approx(0.0, abs=1e-15)
        assert oracle.costs(X, Y, z, z, f, g, eps)["dual"] == pytest.approx(C11, rel=1e-14)


@pytest.mark.parametrize("a1,b1,eps", [(0.5, 0.5, 0.5), (0.3, 0.6, 0.2), (0.8, 0.25, 1.5)])
def test_two_by_two_exact_plan(a1, b1, eps):
    X = np.array([[0.0, 0.0], [1.0, 0.5]])
    Y = np.array([[0.2, -0.3], [0.9, 1.0]])
    loga = np.log([a1, 1 - a1])
    logb = np.log([b1, 1 - b1])
    C = cdist(X, Y, "sqeuclidean")
    P_exact = dense.two_by_two_plan(C, a1, b1, eps)
    f, g = oracle.solve(X, Y, loga, logb, eps, 2000)
    P = dense.plan(C, loga, logb, f, g, eps)
    np.testing.assert_allclose(P, P_exact, rtol=1e-9, atol=1e-12)
    co = oracle.costs(X, Y, loga, logb, f, g, eps)
    ab = np.outer([a1, 1 - a1], [b1, 1 - b1])
    ent = float((P_exact * C).sum() + eps * (P_exact * np.log(P_exact / ab)).sum())
    assert co["dual"] == pytest.approx(ent, rel=1e-9)
    assert co["entropic_primal"] == pytest.approx(ent, rel=1e-9)


@pytest.mark.parametrize("eps", [0.01, 0.1, 1.0])
def test_hard_c_transform_sandwich(eps):
    X, Y, _, logb = _rand_problem(50, 70, 3, 5)
    g = np.random.default_rng(8).standard_normal(70)
    f = oracle.update_f(X, Y, logb, g, eps)
    lo, hi, cm = oracle.minplus_bounds(X, Y, logb, g, eps)
    C = cdist(X, Y, "sqeuclidean")
    np.testing.assert_allclose(lo, (C - g[None, :]).min(1), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(cm, C.max(1), rtol=1e-13)
    assert np.all(f >= lo - 1e-12) and np.all(f <= hi + 1e-12)


def test_large_eps_expansion():
    """f_i = E_b[C_i. - g] - Var_b(C_i. - g)/(2 eps) + O(eps^-2)."""
    X, Y, _, logb = _rand_problem(12, 20, 3, 6)
    g = np.random.default_rng(9).standard_normal(20) * 0.1
    C = cdist(X, Y, "sqeuclidean")
    b = np.exp(logb)
    V = C - g[None, :]
    mean = V @ b
    var = ((V - mean[:, None]) ** 2) @ b
    errs = []
    for eps in (1e2, 1e3):
        f = oracle.update_f(X, Y, logb, g, eps)
        errs.append(np.abs(f - (mean - var / (2 * eps))).max())
    assert errs[1] < errs[0] / 50  # second-order remainder shrinks like eps^-2


def test_marginal_exactness_after_each_update():
    X, Y, loga, logb = _rand_problem(40, 33, 4, 10)
    eps = 0.15
    g = np.random.default_rng(11).standard_normal(33)
    f = oracle.update_f(X, Y, logb, g, eps)
    r, _ = oracle.marginals(X, Y, loga, logb, f, g, eps)
    np.testing.assert_allclose(r, np.exp(loga), rtol=1e-12)
    g2 = oracle.update_g(X, Y, loga, f, eps)
    _, c = oracle.marginals(X, Y, loga, logb, f, g2, eps)
    np.testing.assert_allclose(c, np.exp(logb), rtol=1e-12)


def test_dual_ascent_and_vanishing_gap():
    X, Y, loga, logb = _rand_problem(30, 28, 3, 12)
    eps = 0.1
    f = np.zeros(30)
    g = np.zeros(28)
    duals = [oracle.costs(X, Y, loga, logb, f, g, eps)["dual"]]
    for _ in range(30):
        f = oracle.update_f(X, Y, logb, g, eps)
        duals.append(oracle.costs(X, Y, loga, logb, f, g, eps)["dual"])
        g = oracle.update_g(X, Y, loga, f, eps)
        duals.append(oracle.costs(X, Y, loga, logb, f, g, eps)["dual"])
    dd = np.diff(duals)
    assert np.all(dd >= -1e-12 * np.abs(duals[1:]).max())
    f, g = oracle.solve(X, Y, loga, logb, eps, 3000)
    co = oracle.costs(X, Y, loga, logb, f, g, eps)
    assert abs(co["entropic_primal"] - co["dual"]) < 1e-10
    er, ec = oracle.marginal_error(X, Y, loga, logb, f, g, eps)
    assert er < 1e-10 and ec < 1e-12


def test_symmetries():
    X, Y, loga, logb = _rand_problem(21, 34, 3, 13)
    eps = 0.2
    rng = np.random.default_rng(14)
    g = rng.standard_normal(34)
    f = oracle.update_f(X, Y, logb, g, eps)
    # swap X<->Y: the f-update of (X,Y) is the g-update of (Y,X)
    np.testing.assert_allclose(oracle.update_g(Y, X, logb, g, eps), f, rtol=1e-14, atol=1e-14)
    # gauge: g + c  ->  f - c
    np.testing.assert_allclose(oracle.update_f(X, Y, logb, g + 0.37, eps), f - 0.37, rtol=1e-12, atol=1e-12)
    # translation of both clouds leaves everything unchanged
    t = np.array([3.0, -2.0, 0.5])
    np.testing.assert_allclose(oracle.update_f(X + t, Y + t, logb, g, eps), f, rtol=1e-11, atol=1e-11)
    # permutation equivariance
    p = rng.permutation(21)
    q = rng.permutation(34)
    np.testing.assert_allclose(oracle.update_f(X[p], Y[q], logb[q], g[q], eps), f[p], rtol=1e-13, atol=1e-13)
    # scaling: X,Y * s and eps * s^2  ->  f * s^2
    s = 1.7
    np.testing.assert_allclose(oracle.update_f(X * s, Y * s, logb, g * s * s, eps * s * s), f * s * s,
                               rtol=1e-12, atol=1e-12)
    # full solve with the roles swapped (g-first on (Y,X)) reaches the same fixed point up to gauge
    f1, g1 = oracle.solve(X, Y, loga, logb, eps, 2000)
    g2, f2 = oracle.solve(Y, X, logb, loga, eps, 2000)
    c1 = np.exp(loga) @ f1 - np.exp(logb) @ g1
    c2 = np.exp(loga) @ f2 - np.exp(logb) @ g2
    np.testing.assert_allclose(f1 - c1 / 2, f2 - c2 / 2, atol=1e-9)


# ---- planted mistakes: each one must trip a pin --------------------------------------

def _mutants():
    def sign_of_g(C, logb, g, eps):
        return -eps * dense.logsumexp((-g[None, :] - C) / eps + logb[None, :], axis=1)

    def dropped_logb(C, logb, g, eps):
        return -eps * dense.logsumexp((g[None, :] - C) / eps, axis=1)

    def half_cost(C, logb, g, eps):
        return -eps * dense.logsumexp((g[None, :] - 0.5 * C) / eps + logb[None, :], axis=1)

    def missing_eps_factor(C, logb, g, eps):
        return -dense.logsumexp((g[None, :] - C) / eps + logb[None, :], axis=1)

    return [sign_of_g, dropped_logb, half_cost, missing_eps_factor]


@pytest.mark.parametrize("mutant", _mutants(), ids=lambda f: f.__name__)
def test_planted_mistakes_fail_a_pin(mutant):
    X, Y, loga, logb = _rand_problem(20, 26, 3, 15)
    eps = 0.4
    g = np.random.default_rng(16).standard_normal(26) * 0.2
    C = dense.cost_matrix(X, Y)
    f_bad = mutant(C, logb, g, eps)
    # marginal exactness of the true plan definition
    P = dense.plan(C, loga, logb, f_bad, g, eps)
    marg_ok = np.allclose(P.sum(1), np.exp(loga), rtol=1e-10)
    # agreement with the oracle
    oracle_ok = np.allclose(f_bad, oracle.update_f(X, Y, logb, g, eps), rtol=1e-10, atol=1e-10)
    assert not marg_ok and not oracle_ok


# ---- cosine cost ("cosine distance after normalisation", the second cost the
# method covers per the closing remarks of "FlashSinkhorn: IO-aware EOT on GPU")

def test_cosine_cost_matrix_matches_scipy_cdist():
    X, Y, _, _ = _rand_problem(19, 21, 7, 31)
    np.testing.assert_allclose(dense.cost_matrix(X, Y, "cosine"), cdist(X, Y, "cosine"), rtol=1e-12,
                               atol=1e-13)


@pytest.mark.parametrize("n,m,d", [(37, 53, 5), (1, 9, 3), (40, 40, 128)])
def test_cosine_streaming_matches_dense(n, m, d):
    X, Y, loga, logb = _rand_problem(n, m, d, 40 + n + m)
    rng = np.random.default_rng(8)
    g = 0.1 * rng.standard_normal(m)
    f0 = 0.1 * rng.standard_normal(n)
    eps = 0.05
    C = dense.cost_matrix(X, Y, "cosine")
    np.testing.assert_allclose(oracle.update_f(X, Y, logb, g, eps, cost="cosine"),
                               dense.update_f(C, logb, g, eps), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.update_g(X, Y, loga, f0, eps, cost="cosine"),
                               dense.update_g(C, loga, f0, eps), rtol=1e-12, atol=1e-12)
    rows = np.array([0, n - 1])
    np.testing.assert_allclose(oracle.update_f_rows(rows, X, Y, logb, g, eps, cost="cosine"),
                               dense.update_f(C, logb, g, eps)[rows], rtol=1e-12, atol=1e-12)
    fs, gs = oracle.solve(X, Y, loga, logb, eps, 20, cost="cosine")
    fd, gd = dense.solve(C, loga, logb, eps, 20)
    np.testing.assert_allclose(fs, fd, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(gs, gd, rtol=1e-10, atol=1e-10)
    co = oracle.costs(X, Y, loga, logb, fs, gs, eps, cost="cosine")
    cd = dense.costs(C, loga, logb, fd, gd, eps)
    for key in ("dual", "primal", "entropic_primal", "sum_p"):
        assert abs(co[key] - cd[key]) <= 1e-10 * max(1.0, abs(cd[key])), key
    assert abs(co["max_cost"] - C.max()) <= 1e-14 and abs(co["min_cost"] - C.min()) <= 1e-14


def test_cosine_on_the_sphere_is_half_the_squared_distance():
    """For unit vectors |x - y|^2 = 2 (1 - cos): the cosine solve at eps equals half
    the squared-Euclidean solve at 2 eps (f-update: -eps LSE[(g - C/2)/eps + log b]
    = (1/2)(-2 eps LSE[(2g - C)/(2 eps) + log b]), so every iterate is halved)."""
    X, Y, loga, logb = _rand_problem(30, 25, 4, 55)
    X /= np.linalg.norm(X, axis=1, keepdims=True)
    Y /= np.linalg.norm(Y, axis=1, keepdims=True)
    eps = 0.07
    fc, gc = oracle.solve(X, Y, loga, logb, eps, 15, cost="cosine")
    fq, gq = oracle.solve(X, Y, loga, logb, 2 * eps, 15)
    np.testing.assert_allclose(fc, 0.5 * fq, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(gc, 0.5 * gq, rtol=1e-11, atol=1e-12)


def test_cosine_is_scale_invariant_and_marginal_exact():
    X, Y, loga, logb = _rand_problem(24, 31, 6, 56)
    rng = np.random.default_rng(57)
    sx = rng.uniform(0.2, 5.0, (24, 1))
    sy = rng.uniform(0.2, 5.0, (31, 1))
    eps = 0.05
    f1, g1 = oracle.solve(X, Y, loga, logb, eps, 10, cost="cosine")
    f2, g2 = oracle.solve(X * sx, Y * sy, loga, logb, eps, 10, cost="cosine")
    np.testing.assert_allclose(f1, f2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(g1, g2, rtol=1e-11, atol=1e-12)
    # after the closing g-update the column marginal is exact
    _, c = oracle.marginals(X, Y, loga, logb, f1, g1, eps, cost="cosine")
    np.testing.assert_allclose(c, np.exp(logb), rtol=1e-12)


def test_cosine_rejects_zero_vectors():
    X, Y, loga, logb = _rand_problem(5, 6, 3, 58)
    X[2] = 0.0
    with pytest.raises(ValueError):
        oracle.update_f(X, Y, logb, np.zeros(6), 0.1, cost="cosine")


# ---- transport application (Metodologia section 3 of "FlashSinkhorn: IO-aware
# EOT on GPU": barycentric projection and gradient as plan-weighted averages)

@pytest.mark.parametrize("cost", ["sqeuclidean", "cosine"])
def test_transport_apply_matches_dense_plan(cost):
    X, Y, loga, logb = _rand_problem(23, 31, 4, 70)
    rng = np.random.default_rng(71)
    f = 0.2 * rng.standard_normal(23)
    g = 0.2 * rng.standard_normal(31)
    V = rng.standard_normal((31, 5))
    eps = 0.3
    out, r = oracle.transport_apply(X, Y, loga, logb, f, g, eps, V, cost=cost)
    P = dense.plan(dense.cost_matrix(X, Y, cost), loga, logb, f, g, eps)
    np.testing.assert_allclose(out, P @ V, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(r, P.sum(axis=1), rtol=1e-12)
    # V = 1 gives the row marginal
    ones, _ = oracle.transport_apply(X, Y, loga, logb, f, g, eps, np.ones((31, 1)), cost=cost)
    np.testing.assert_allclose(ones[:, 0], oracle.marginals(X, Y, loga, logb, f, g, eps, cost=cost)[0], rtol=1e-12)


@pytest.mark.parametrize("cost", ["sqeuclidean", "cosine"])
def test_grad_x_matches_finite_differences_of_the_optimal_value(cost):
    """At optimal potentials the entropic OT value (the dual) has gradient
    sum_j P_ij dC_ij/dx_i with respect to x_i (envelope theorem)."""
    rng = np.random.default_rng(72)
    n, m, d, eps = 6, 5, 2, 0.5
    X = rng.standard_normal((n, d))
    Y = rng.standard_normal((m, d))
    a = rng.uniform(0.5, 1.5, n)
    b = rng.uniform(0.5, 1.5, m)
    loga, logb = np.log(a / a.sum()), np.log(b / b.sum())

    def value(Xv):
        f, g = oracle.solve(Xv, Y, loga, logb, eps, 400, cost=cost)
        return oracle.costs(Xv, Y, loga, logb, f, g, eps, cost=cost)["dual"], f, g

    _, f, g = value(X)
    G = oracle.grad_x(X, Y, loga, logb, f, g, eps, cost=cost)
    h = 1e-5
    for i in range(n):
        for k in range(d):
            Xp, Xm = X.copy(), X.copy()
            Xp[i, k] += h
            Xm[i, k] -= h
            fd = (value(Xp)[0] - value(Xm)[0]) / (2 * h)
            assert abs(G[i, k] - fd) <= 1e-8, (i, k, G[i, k], fd)


def test_barycentric_projection_tends_to_the_optimal_assignment():
    """Uniform weights, n = m: as eps -> 0 the plan tends to an optimal permutation
    (here unique), so the barycentric map sends x_i to its assigned y (Hungarian
    algorithm, scipy's linear_sum_assignment)."""
    from scipy.optimize import linear_sum_assignment
    rng = np.random.default_rng(5)
    X = rng.standard_normal((8, 2))
    Y = rng.standard_normal((8, 2)) + 0.2
    loga = logb = np.full(8, -np.log(8))
    f, g = oracle.solve(X, Y, loga, logb, 0.02, 3000)
    T = oracle.barycentric_projection(X, Y, loga, logb, f, g, 0.02)
    _, cols = linear_sum_assignment(dense.cost_matrix(X, Y))
    assert np.abs(T - Y[cols]).max() < 1e-2


@pytest.mark.parametrize("cost", ["sqeuclidean", "cosine"])
def test_grad_y_matches_finite_differences_of_the_optimal_value(cost):
    rng = np.random.default_rng(73)
    n, m, d, eps = 5, 6, 2, 0.4
    X = rng.standard_normal((n, d))
    Y = rng.standard_normal((m, d)) + 0.3
    a = rng.uniform(0.5, 1.5, n)
    b = rng.uniform(0.5, 1.5, m)
    loga, logb = np.log(a / a.sum()), np.log(b / b.sum())

    def value(Yv):
        f, g = oracle.solve(X, Yv, loga, logb, eps, 500, cost=cost)
        return oracle.costs(X, Yv, loga, logb, f, g, eps, cost=cost)["dual"], f, g

    _, f, g = value(Y)
    G = oracle.grad_y(X, Y, loga, logb, f, g, eps, cost=cost)
    h = 1e-5
    for j in range(m):
        for k in range(d):
            Yp, Ym = Y.copy(), Y.copy()
            Yp[j, k] += h
            Ym[j, k] -= h
            fd = (value(Yp)[0] - value(Ym)[0]) / (2 * h)
            assert abs(G[j, k] - fd) <= 1e-8, (j, k, G[j, k], fd)


# ---- streaming HVP (Metodologia section 3: Hessian-vector products of the EOT
# loss as sequences of transport-vector and transport-matrix products)

@pytest.mark.parametrize("cost", ["sqeuclidean", "cosine"])
def test_hvp_x_matches_finite_differences_of_the_gradient(cost):
    """dense.hvp_x against central differences of the gradient at re-converged
    potentials: (G(X + hV) - G(X - hV)) / 2h."""
    rng = np.random.default_rng(74)
    n, m, d, eps = 7, 6, 3, 0.6
    X = rng.standard_normal((n, d))
    Y = rng.standard_normal((m, d)) + 0.2
    a = rng.uniform(0.5, 1.5, n)
    b = rng.uniform(0.5, 1.5, m)
    loga, logb = np.log(a / a.sum()), np.log(b / b.sum())
    V = rng.standard_normal((n, d))

    def grad(Xv):
        f, g = oracle.solve(Xv, Y, loga, logb, eps, 800, cost=cost)
        return oracle.grad_x(Xv, Y, loga, logb, f, g, eps, cost=cost), f, g

    _, f, g = grad(X)
    H = dense.hvp_x(X, Y, loga, logb, f, g, eps, V, cost=cost)
    h = 1e-5
    fd = (grad(X + h * V)[0] - grad(X - h * V)[0]) / (2 * h)
    np.testing.assert_allclose(H, fd, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("cost", ["sqeuclidean", "cosine"])
def test_hvp_x_is_symmetric(cost):
    """<W, H V> = <V, H W>: the Hessian is symmetric."""
    rng = np.random.default_rng(75)
    n, m, d, eps = 6, 8, 2, 0.5
    X = rng.standard_normal((n, d))
    Y = rng.standard_normal((m, d))
    loga, logb = np.full(n, -np.log(n)), np.full(m, -np.log(m))
    f, g = oracle.solve(X, Y, loga, logb, eps, 800, cost=cost)
    V, W = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    assert abs(np.sum(W * dense.hvp_x(X, Y, loga, logb, f, g, eps, V, cost=cost)) -
               np.sum(V * dense.hvp_x(X, Y, loga, logb, f, g, eps, W, cost=cost))) <= 1e-10


@pytest.mark.parametrize("cost", ["sqeuclidean", "cosine"])
def test_per_pair_cost_derivatives_match_finite_differences(cost):
    """dense.cost_grad_x and dense.cost_hess_x (the per-pair first and second
    derivatives the HVP is built from) against central differences of the cost
    matrix itself and of cost_grad_x."""
    rng = np.random.default_rng(76)
    X = rng.standard_normal((4, 3))
    Y = rng.standard_normal((5, 3))
    V = rng.standard_normal((4, 3))
    h = 1e-6
    D = dense.cost_grad_x(X, Y, cost)
    for k in range(3):
        E = np.zeros_like(X)
        E[:, k] = h
        fd = (dense.cost_matrix(X + E, Y, cost) - dense.cost_matrix(X - E, Y, cost)) / (2 * h)
        np.testing.assert_allclose(D[:, :, k], fd, rtol=1e-7, atol=1e-9)
    fdH = (dense.cost_grad_x(X + h * V, Y, cost) - dense.cost_grad_x(X - h * V, Y, cost)) / (2 * h)
    np.testing.assert_allclose(dense.cost_hess_x(X, Y, V, cost), fdH, rtol=1e-6, atol=1e-8)


def test_cosine_gradient_is_tangent_and_scales_inversely():
    """The cosine cost depends on x only through x / |x|: its gradient with
    respect to x_i is orthogonal to x_i, and scaling a point by s > 0 scales its
    gradient by 1 / s (the potentials do not change)."""
    rng = np.random.default_rng(77)
    X = rng.standard_normal((6, 3))
    Y = rng.standard_normal((7, 3))
    loga, logb = np.full(6, -np.log(6)), np.full(7, -np.log(7))
    f, g = oracle.solve(X, Y, loga, logb, 0.3, 500, cost="cosine")
    G = oracle.grad_x(X, Y, loga, logb, f, g, 0.3, cost="cosine")
    assert np.abs(np.sum(G * X, axis=1)).max() <= 1e-13
    s = np.array([0.5, 2.0, 3.0, 1.0, 7.0, 0.25])
    G2 = oracle.grad_x(X * s[:, None], Y, loga, logb, f, g, 0.3, cost="cosine")
    np.testing.assert_allclose(G2, G / s[:, None], rtol=1e-12, atol=1e-15)
