"""ctypes front end of the C oracle (``sinkhorn_oracle.c``).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Every function takes one problem's float64 arrays (X [n,d], Y [m,d], log
weights, potentials) and follows "FlashSinkhorn: IO-aware EOT on GPU",
Metodologia section 1 (the stabilised log-domain updates).  Batched
workloads are handled by the caller, one problem at a time.

``cost`` selects C: "sqeuclidean" (C = |x - y|^2, the page's cost) or
"cosine" (C = 1 - cos(x, y), the cosine distance that the page's closing
remarks name as the other cost the method covers after normalisation).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None
_dp = ctypes.POINTER(ctypes.c_double)
_lp = ctypes.POINTER(ctypes.c_long)


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        L, I, D = ctypes.c_long, ctypes.c_int, ctypes.c_double
        lib.so_update_f.argtypes = [L, L, I, _dp, _dp, _dp, _dp, D, _dp, I]
        lib.so_update_g.argtypes = [L, L, I, _dp, _dp, _dp, _dp, D, _dp, I]
        lib.so_solve.argtypes = [L, L, I, _dp, _dp, _dp, _dp, D, I, _dp, _dp, I]
        lib.so_marginals.argtypes = [L, L, I, _dp, _dp, _dp, _dp, _dp, _dp, D, _dp, _dp, I]
        lib.so_plan_stats.argtypes = [L, L, I, _dp, _dp, _dp, _dp, _dp, _dp, D, _dp, I]
        lib.so_minplus_bounds.argtypes = [L, L, I, _dp, _dp, _dp, _dp, D, _dp, _dp, _dp, I]
        lib.so_update_f_rows.argtypes = [L, _lp, L, I, _dp, _dp, _dp, _dp, D, _dp, I]
        lib.so_transport_apply.argtypes = [L, L, I, _dp, _dp, _dp, _dp, _dp, _dp, D, I, _dp, _dp, _dp, I]
        lib.so_num_threads.argtypes = []
        for name in ("so_update_f", "so_update_g", "so_solve", "so_plan_stats", "so_update_f_rows",
                     "so_transport_apply", "so_num_threads"):
            getattr(lib, name).restype = ctypes.c_int
        lib.so_marginals.restype = None
        lib.so_minplus_bounds.restype = None
        _lib = lib
    return _lib


def _c(a):
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data_as(_dp)


COSTS = {"sqeuclidean": 0, "cosine": 1}


def _cost(cost, *clouds):
    """The C code of ``cost``; the cosine distance is undefined for a zero vector."""
    if cost not in COSTS:
        raise ValueError(f"unknown cost {cost!r}")
    if cost == "cosine":
        for P in clouds:
            if np.any(np.sum(np.asarray(P, dtype=np.float64) ** 2, axis=1) == 0.0):
                raise ValueError("the cosine cost is undefined for a zero vector")
    return COSTS[cost]


def num_threads() -> int:
    """OpenMP threads the oracle runs on (OMP_NUM_THREADS, else all cores)."""
    return int(_load().so_num_threads())


def log_weights(w, count):
    """log of the weights; ``None`` means uniform 1/count."""
    if w is None:
        return np.full(count, -np.log(count))
    return np.log(np.asarray(w, dtype=np.float64))


def problem_arrays(prob, k=0):
    """(X, Y, loga, logb) of problem ``k`` of a drawn workload (duck-typed)."""
    X = np.ascontiguousarray(prob.X[k], dtype=np.float64)
    Y = np.ascontiguousarray(prob.Y[k], dtype=np.float64)
    loga = log_weights(None if prob.a is None else prob.a[k], prob.n)
    logb = log_weights(None if prob.b is None else prob.b[k], prob.m)
    return X, Y, loga, logb


def update_f(X, Y, logb, g, eps, cost="sqeuclidean"):
    """f_i = -eps LSE_j[(g_j - C_ij)/eps + log b_j]  (the f-update of Proposition 1's setting)."""
    ci = _cost(cost, X, Y)
    X, px = _c(X)
    Y, py = _c(Y)
    logb, pb = _c(logb)
    g, pg = _c(g)
    n, d = X.shape
    m = Y.shape[0]
    f = np.empty(n)
    if _load().so_update_f(n, m, d, px, py, pb, pg, float(eps), f.ctypes.data_as(_dp), ci):
        raise MemoryError("oracle update_f")
    return f


def update_g(X, Y, loga, f, eps, cost="sqeuclidean"):
    """g_j = -eps LSE_i[(f_i - C_ij)/eps + log a_i]  (the transposed update)."""
    ci = _cost(cost, X, Y)
    X, px = _c(X)
    Y, py = _c(Y)
    loga, pa = _c(loga)
    f, pf = _c(f)
    n, d = X.shape
    m = Y.shape[0]
    g = np.empty(m)
    if _load().so_update_g(n, m, d, px, py, pa, pf, float(eps), g.ctypes.data_as(_dp), ci):
        raise MemoryError("oracle update_g")
    return g


def update_f_rows(rows, X, Y, logb, g, eps, cost="sqeuclidean"):
    """The f-update at selected rows only (for spot checks at full size)."""
    ci = _cost(cost, np.asarray(X)[np.asarray(rows, dtype=np.int64)], Y)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    X, px = _c(X)
    Y, py = _c(Y)
    logb, pb = _c(logb)
    g, pg = _c(g)
    d = X.shape[1]
    m = Y.shape[0]
    out = np.empty(rows.shape[0])
    if _load().so_update_f_rows(rows.shape[0], rows.ctypes.data_as(_lp), m, d, px, py, pb, pg,
                                float(eps), out.ctypes.data_as(_dp), ci):
        raise MemoryError("oracle update_f_rows")
    return out


def solve(X, Y, loga, logb, eps, iters, g0=None, cost="sqeuclidean"):
    """Alternating Sinkhorn from g0 (default 0): iters x {f <- update_f(g); g <- update_g(f)}."""
    ci = _cost(cost, X, Y)
    X, px = _c(X)
    Y, py = _c(Y)
    loga, pa = _c(loga)
    logb, pb = _c(logb)
    n, d = X.shape
    m = Y.shape[0]
    f = np.zeros(n)
    g = np.zeros(m) if g0 is None else np.array(g0, dtype=np.float64)
    if _load().so_solve(n, m, d, px, py, pa, pb, float(eps), int(iters), f.ctypes.data_as(_dp),
                        g.ctypes.data_as(_dp), ci):
        raise MemoryError("oracle solve")
    return f, g


def marginals(X, Y, loga, logb, f, g, eps, cost="sqeuclidean"):
    """(r, c): row and column sums of P_ij = a_i b_j exp((f_i + g_j - C_ij)/eps)."""
    ci = _cost(cost, X, Y)
    X, px = _c(X)
    Y, py = _c(Y)
    loga, pa = _c(loga)
    logb, pb = _c(logb)
    f, pf = _c(f)
    g, pg = _c(g)
    n, d = X.shape
    m = Y.shape[0]
    r = np.empty(n)
    c = np.empty(m)
    _load().so_marginals(n, m, d, px, py, pa, pb, pf, pg, float(eps), r.ctypes.data_as(_dp),
                         c.ctypes.data_as(_dp), ci)
    return r, c


def marginal_error(X, Y, loga, logb, f, g, eps, cost="sqeuclidean"):
    """(err_row, err_col) = (sum_i |r_i - a_i|, sum_j |c_j - b_j|)."""
    r, c = marginals(X, Y, loga, logb, f, g, eps, cost)
    return float(np.abs(r - np.exp(loga)).sum()), float(np.abs(c - np.exp(logb)).sum())


def plan_stats(X, Y, loga, logb, f, g, eps, cost="sqeuclidean"):
    """sum P, <P,C>, sum P log(P/(a b)), max C, min C -- one pass over all pairs."""
    ci = _cost(cost, X, Y)
    X, px = _c(X)
    Y, py = _c(Y)
    loga, pa = _c(loga)
    logb, pb = _c(logb)
    f, pf = _c(f)
    g, pg = _c(g)
    n, d = X.shape
    m = Y.shape[0]
    out = np.empty(5)
    if _load().so_plan_stats(n, m, d, px, py, pa, pb, pf, pg, float(eps), out.ctypes.data_as(_dp), ci):
        raise MemoryError("oracle plan_stats")
    return dict(sum_p=out[0], primal=out[1], p_log_ratio=out[2], max_cost=out[3], min_cost=out[4])


def costs(X, Y, loga, logb, f, g, eps, cost="sqeuclidean"):
    """Dual and primal objectives of entropic OT at the pair (f, g).

    dual            D = <a,f> + <b,g> - eps (sum_ij P_ij - 1)
    primal          <P, C>                         (transport cost of the plan)
    entropic_primal <P, C> + eps KL(P | a (x) b),  KL(P|Q) = sum P log(P/Q) - sum P + 1
    """
    s = plan_stats(X, Y, loga, logb, f, g, eps, cost)
    a = np.exp(np.asarray(loga, dtype=np.float64))
    b = np.exp(np.asarray(logb, dtype=np.float64))
    dual = float(a @ f + b @ g - eps * (s["sum_p"] - 1.0))
    kl = s["p_log_ratio"] - s["sum_p"] + 1.0
    return dict(dual=dual, primal=float(s["primal"]), entropic_primal=float(s["primal"] + eps * kl),
                sum_p=float(s["sum_p"]), max_cost=float(s["max_cost"]), min_cost=float(s["min_cost"]))


def minplus_bounds(X, Y, logb, g, eps, cost="sqeuclidean"):
    """Per row: (min_j (C_ij - g_j), min_j (C_ij - g_j - eps log b_j), max_j C_ij).

    The soft c-transform (the f-update) lies between the first two for every
    row (hard c-transform sandwich)."""
    ci = _cost(cost, X, Y)
    X, px = _c(X)
    Y, py = _c(Y)
    logb, pb = _c(logb)
    g, pg = _c(g)
    n, d = X.shape
    m = Y.shape[0]
    lo = np.empty(n)
    hi = np.empty(n)
    cm = np.empty(n)
    _load().so_minplus_bounds(n, m, d, px, py, pb, pg, float(eps), lo.ctypes.data_as(_dp),
                              hi.ctypes.data_as(_dp), cm.ctypes.data_as(_dp), ci)
    return lo, hi, cm


os.environ.setdefault("OMP_WAIT_POLICY", "PASSIVE")


def transport_apply(X, Y, loga, logb, f, g, eps, V, cost="sqeuclidean"):
    """(out, r): out_i = sum_j P_ij V_j and r_i = sum_j P_ij for P_ij = a_i b_j exp((f_i + g_j - C_ij)/eps)
    ("FlashSinkhorn: IO-aware EOT on GPU", Metodologia section 3: applying the plan without forming it)."""
    ci = _cost(cost, X, Y)
    X, px = _c(X)
    Y, py = _c(Y)
    loga, pa = _c(loga)
    logb, pb = _c(logb)
    f, pf = _c(f)
    g, pg = _c(g)
    V = np.asarray(V, dtype=np.float64)
    V = V.reshape(V.shape[0], -1)
    V, pv = _c(V)
    n, d = X.shape
    m = Y.shape[0]
    if V.shape[0] != m:
        raise ValueError("V must have one row per column point")
    dv = V.shape[1]
    out = np.empty((n, dv))
    r = np.empty(n)
    _load().so_transport_apply(n, m, d, px, py, pa, pb, pf, pg, float(eps), dv, pv, out.ctypes.data_as(_dp),
                               r.ctypes.data_as(_dp), ci)
    return out, r


def barycentric_projection(X, Y, loga, logb, f, g, eps, cost="sqeuclidean"):
    """T(x_i) = sum_j P_ij y_j / sum_j P_ij (the plan's barycentric map)."""
    out, r = transport_apply(X, Y, loga, logb, f, g, eps, Y, cost)
    return out / r[:, None]


def grad_x(X, Y, loga, logb, f, g, eps, cost="sqeuclidean"):
    """Gradient of the entropic OT cost with respect to the positions X at the
    potentials (f, g): sum_j P_ij dC_ij/dx_i.  At optimal potentials this is the
    gradient of the optimal value (envelope theorem).

    * squared Euclidean, dC/dx = 2 (x - y): 2 (r_i x_i - sum_j P_ij y_j);
    * cosine, C = 1 - x.y / (|x| |y|), dC/dx = -(y^ - (x^.y^) x^) / |x| with
      x^ = x / |x|, y^ = y / |y| (the part of y^ orthogonal to x, over |x|):
      -(b_i - (x^_i.b_i) x^_i) / |x_i| with b_i = sum_j P_ij y^_j, the per-pair
      gradients being linear in y^_j.
    """
    X = np.asarray(X, dtype=np.float64)
    if cost == "cosine":
        Y = np.asarray(Y, dtype=np.float64)
        Yh = Y / np.linalg.norm(Y, axis=1)[:, None]
        bsum, _ = transport_apply(X, Y, loga, logb, f, g, eps, Yh, cost)
        nx = np.linalg.norm(X, axis=1)
        Xh = X / nx[:, None]
        return -(bsum - np.sum(Xh * bsum, axis=1)[:, None] * Xh) / nx[:, None]
    out, r = transport_apply(X, Y, loga, logb, f, g, eps, Y, cost)
    return 2.0 * (r[:, None] * X - out)


def grad_y(X, Y, loga, logb, f, g, eps, cost="sqeuclidean"):
    """Gradient of the entropic OT cost with respect to the positions Y at (f, g):
    grad_x with the roles of the two clouds (and weights, potentials) exchanged,
    both costs being symmetric in x and y (squared Euclidean: 2 (c_j y_j -
    sum_i P_ij x_i))."""
    return grad_x(Y, X, logb, loga, g, f, eps, cost)
