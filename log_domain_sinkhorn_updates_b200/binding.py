"""ctypes binding of the C ABI declared in ``include/flashsinkhorn.h``.

Argument marshalling only: every step of the computation runs in the CUDA
library.  Device arrays are torch CUDA tensors (their data pointers are
passed through); host arrays are numpy arrays.  If the shared library is
missing the import fails loudly -- there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libflashsinkhorn.so")

FS_OK, FS_ERR_INVALID_ARG, FS_ERR_CUDA, FS_ERR_UNSUPPORTED, FS_ERR_NONFINITE, FS_ERR_TIMEOUT, FS_ERR_OOM = range(7)
FS_F32, FS_BF16 = 0, 1
PRECISIONS = {"auto": 0, "bf16": 1, "tf32": 2, "3xtf32": 3, "3xf16": 4, "f32_simt": 5}
PRECISION_NAMES = {v: k for k, v in PRECISIONS.items()}
SCHEDULES = {"alternating": 0, "symmetric": 1}
COSTS = {"sqeuclidean": 0, "cosine": 1}
STATUS_NAMES = {0: "FS_OK", 1: "FS_ERR_INVALID_ARG", 2: "FS_ERR_CUDA", 3: "FS_ERR_UNSUPPORTED",
                4: "FS_ERR_NONFINITE", 5: "FS_ERR_TIMEOUT", 6: "FS_ERR_OOM"}

EXPORTS = ["fs_create", "fs_update_f", "fs_update_g", "fs_solve", "fs_marginal_err", "fs_ot_cost",
           "fs_sync", "fs_get_info", "fs_destroy", "fs_last_error", "fs_solve_host", "fs_kernel_launches",
           "fs_update_f_noalloc", "fs_transport_apply", "fs_barycentric_map", "fs_grad_x",
           "fs_transport_apply_t", "fs_grad_y", "fs_hvp_x", "fs_selftest_wait"]


class FsDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("n", ctypes.c_int), ("m", ctypes.c_int), ("d", ctypes.c_int),
                ("dtype", ctypes.c_int), ("prec", ctypes.c_int), ("eps", ctypes.c_float), ("cost", ctypes.c_int)]


class FsInfo(ctypes.Structure):
    _fields_ = [("prec", ctypes.c_int), ("d_pad", ctypes.c_int), ("row_bytes", ctypes.c_int),
                ("swizzle_bytes", ctypes.c_int), ("stages", ctypes.c_int), ("block_rows", ctypes.c_int),
                ("block_cols", ctypes.c_int), ("splits_f", ctypes.c_int), ("splits_g", ctypes.c_int),
                ("launches_update", ctypes.c_int), ("launches_solve_iter", ctypes.c_int),
                ("device_bytes", ctypes.c_size_t), ("cta_pair", ctypes.c_int), ("last_apply_path", ctypes.c_int),
                ("last_solve_graph", ctypes.c_int), ("last_measure_fused", ctypes.c_int),
                ("last_hvp_fused", ctypes.c_int), ("last_apply_parts", ctypes.c_int)]

    def as_dict(self):
        d = {k: getattr(self, k) for k, _ in self._fields_}
        d["prec"] = PRECISION_NAMES.get(d["prec"], d["prec"])
        d["last_apply_path"] = {0: None, 1: "tc", 2: "simt", 3: "tc_pair", 4: "tc_q2", 5: "lse_vec", 6: "tc_2s"}.get(d["last_apply_path"],
                                                                               d["last_apply_path"])
        d["last_solve_graph"] = {0: None, 1: "graph", 2: "direct"}.get(d["last_solve_graph"], d["last_solve_graph"])
        return d


class FsError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib = None


def lib():
    """The loaded C library (ctypes.CDLL); raises ImportError if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"CUDA extension missing: {LIB_PATH} (run log_domain_sinkhorn_updates_b200/build.py)")
        L = ctypes.CDLL(LIB_PATH)
        vp, dp, fp = ctypes.c_void_p, ctypes.POINTER(ctypes.c_double), ctypes.c_void_p
        L.fs_create.argtypes = [ctypes.POINTER(FsDesc), vp, vp, vp, vp, vp, ctypes.POINTER(ctypes.c_void_p)]
        L.fs_update_f.argtypes = [vp, fp, fp]
        L.fs_update_g.argtypes = [vp, fp, fp]
        L.fs_solve.argtypes = [vp, fp, fp, ctypes.c_int, ctypes.c_int]
        L.fs_marginal_err.argtypes = [vp, fp, fp, dp, dp]
        L.fs_ot_cost.argtypes = [vp, fp, fp, dp, dp]
        L.fs_sync.argtypes = [vp]
        L.fs_get_info.argtypes = [vp, ctypes.POINTER(FsInfo)]
        L.fs_destroy.argtypes = [vp]
        L.fs_last_error.argtypes = [vp]
        L.fs_last_error.restype = ctypes.c_char_p
        L.fs_solve_host.argtypes = [ctypes.POINTER(FsDesc), vp, vp, vp, vp, vp, vp, ctypes.c_int, ctypes.c_int,
                                    dp, dp, dp, dp, vp]
        L.fs_update_f_noalloc.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, vp, vp, vp, vp,
                                          vp, vp]
        L.fs_transport_apply.argtypes = [vp, vp, vp, vp, ctypes.c_int, vp, vp]
        L.fs_barycentric_map.argtypes = [vp, vp, vp, vp, vp]
        L.fs_grad_x.argtypes = [vp, vp, vp, vp, vp, vp]
        L.fs_transport_apply_t.argtypes = [vp, vp, vp, vp, ctypes.c_int, vp, vp]
        L.fs_grad_y.argtypes = [vp, vp, vp, vp, vp, vp]
        L.fs_hvp_x.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.c_int, ctypes.c_double, vp]
        L.fs_selftest_wait.argtypes = [vp, ctypes.c_int]
        L.fs_kernel_launches.argtypes = []
        L.fs_kernel_launches.restype = ctypes.c_ulonglong
        for name in EXPORTS:
            if name not in ("fs_last_error", "fs_kernel_launches"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status, handle=None):
    if status != FS_OK:
        msg = lib().fs_last_error(handle)
        raise FsError(status, msg.decode() if msg else "")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _f32(t):
    import torch
    if t is not None and t.dtype != torch.float32:
        raise ValueError("potentials and weights must be float32")
    return _ptr(t)


def _stream_ptr(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class Handle:
    """Owns an ``fs_handle*``; freed by ``fs_destroy`` (or when collected)."""

    def __init__(self, ptr, desc, stream):
        self.ptr = ptr
        self.desc = desc
        self.stream = stream

    @property
    def batch(self):
        return self.desc.batch

    @property
    def n(self):
        return self.desc.n

    @property
    def m(self):
        return self.desc.m

    def __del__(self):
        try:
            fs_destroy(self)
        except Exception:
            pass


def fs_create(X, Y, a=None, b=None, eps=0.1, prec="auto", stream=None, cost="sqeuclidean") -> Handle:
    """X [batch, n, d] / [n, d], Y likewise (CUDA float32 or bfloat16), a [batch, n], b [batch, m] or None.
    cost: "sqeuclidean" (C = |x - y|^2) or "cosine" (C = 1 - cos(x, y))."""
    import torch
    if X.dim() == 2:
        X, Y = X.unsqueeze(0), Y.unsqueeze(0)
        a = None if a is None else a.reshape(1, -1)
        b = None if b is None else b.reshape(1, -1)
    if X.dtype != Y.dtype:
        raise ValueError("X and Y must share a dtype")
    dtype = {torch.float32: FS_F32, torch.bfloat16: FS_BF16}.get(X.dtype)
    if dtype is None:
        raise ValueError("X, Y must be float32 or bfloat16")
    B, n, d = X.shape
    m = Y.shape[1]
    if Y.shape[0] != B or Y.shape[2] != d:
        raise ValueError("X and Y shapes disagree")
    desc = FsDesc(B, n, m, d, dtype, PRECISIONS[prec] if isinstance(prec, str) else int(prec), float(eps),
                  COSTS[cost])
    out = ctypes.c_void_p()
    st = lib().fs_create(ctypes.byref(desc), _ptr(X), _ptr(Y), _f32(a), _f32(b), _stream_ptr(stream),
                         ctypes.byref(out))
    _check(st)
    return Handle(out, desc, stream)


def fs_update_f(h: Handle, g, f):
    _check(lib().fs_update_f(h.ptr, _f32(g), _f32(f)), h.ptr)


def fs_update_g(h: Handle, f, g):
    _check(lib().fs_update_g(h.ptr, _f32(f), _f32(g)), h.ptr)


def fs_solve(h: Handle, f, g, iters, schedule="alternating"):
    _check(lib().fs_solve(h.ptr, _f32(f), _f32(g), int(iters), SCHEDULES[schedule]), h.ptr)


def fs_marginal_err(h: Handle, f, g, row=True, col=True):
    er = np.zeros(h.batch)
    ec = np.zeros(h.batch)
    dp = ctypes.POINTER(ctypes.c_double)
    _check(lib().fs_marginal_err(h.ptr, _f32(f), _f32(g), er.ctypes.data_as(dp) if row else None,
                                 ec.ctypes.data_as(dp) if col else None), h.ptr)
    return (er if row else None), (ec if col else None)


def fs_ot_cost(h: Handle, f, g):
    dual = np.zeros(h.batch)
    primal = np.zeros(h.batch)
    dp = ctypes.POINTER(ctypes.c_double)
    _check(lib().fs_ot_cost(h.ptr, _f32(f), _f32(g), dual.ctypes.data_as(dp), primal.ctypes.data_as(dp)), h.ptr)
    return dual, primal


def fs_sync(h: Handle):
    _check(lib().fs_sync(h.ptr), h.ptr)


def fs_get_info(h: Handle) -> dict:
    info = FsInfo()
    _check(lib().fs_get_info(h.ptr, ctypes.byref(info)), h.ptr)
    return info.as_dict()


def fs_destroy(h: Handle):
    if h is not None and h.ptr:
        p, h.ptr = h.ptr, None
        lib().fs_destroy(p)


def fs_last_error(h: Handle = None) -> str:
    msg = lib().fs_last_error(h.ptr if h is not None else None)
    return msg.decode() if msg else ""


def fs_update_f_noalloc(X, Y, b, g, f, eps, stream=None):
    """One f-update through the allocation-free entry point: X [n, d], Y [m, d] float32 CUDA
    tensors, b [m] or None (uniform), g [m], output f [n].  Asynchronous on the stream."""
    if X.dim() != 2 or Y.dim() != 2 or X.shape[1] != Y.shape[1]:
        raise ValueError("X [n, d] and Y [m, d] expected")
    n, d = X.shape
    m = Y.shape[0]
    _check(lib().fs_update_f_noalloc(n, m, d, float(eps), _f32(X), _f32(Y), _f32(b), _f32(g), _f32(f),
                                     _stream_ptr(stream)))


def fs_kernel_launches() -> int:
    """Kernels the library has launched in this process (host-side count)."""
    return int(lib().fs_kernel_launches())


def fs_solve_host(X, Y, a, b, g0, eps, iters, dtype="f32", prec="auto", schedule="alternating", stream=None,
                  measure=True, out=None, cost="sqeuclidean"):
    """End-to-end solve from host (numpy) arrays through ``fs_solve_host``.

    X, Y: [batch, n|m, d] float32 (or uint16 bfloat16 bits with dtype="bf16"),
    a, b: float32 or None (uniform), g0: [batch, m] float32 initial g.
    Returns (f, g, err_row, err_col, dual, primal) as numpy arrays.
    """
    X = np.ascontiguousarray(X)
    Y = np.ascontiguousarray(Y)
    if X.ndim == 2:
        X, Y = X[None], Y[None]
    B, n, d = X.shape
    m = Y.shape[1]
    desc = FsDesc(B, n, m, d, FS_BF16 if dtype == "bf16" else FS_F32, PRECISIONS[prec], float(eps), COSTS[cost])
    if out is None:
        f = np.empty((B, n), np.float32)
        g = np.array(g0, dtype=np.float32).reshape(B, m)
    else:
        f, g = out
        g[...] = np.asarray(g0, dtype=np.float32).reshape(B, m)
    res = [np.zeros(B) for _ in range(4)]
    dp = ctypes.POINTER(ctypes.c_double)
    vp = lambda arr: None if arr is None else ctypes.c_void_p(arr.ctypes.data)  # noqa: E731
    rp = [r.ctypes.data_as(dp) if measure else None for r in res]
    st = lib().fs_solve_host(ctypes.byref(desc), vp(X), vp(Y),
                             vp(None if a is None else np.ascontiguousarray(a, np.float32)),
                             vp(None if b is None else np.ascontiguousarray(b, np.float32)),
                             vp(f), vp(g), int(iters), SCHEDULES[schedule], *rp,
                             None if stream is None else ctypes.c_void_p(stream.cuda_stream))
    _check(st)
    return (f, g, *res)


def fs_transport_apply(h: Handle, f, g, V, out, r=None):
    """out[k, i, :] = sum_j P_ij V[k, j, :] (V float32 [batch, m, dv]); r[k, i] = sum_j P_ij if given."""
    import torch
    if V.dtype != torch.float32 or out.dtype != torch.float32:
        raise ValueError("V and out must be float32")
    dv = V.shape[-1]
    _check(lib().fs_transport_apply(h.ptr, _f32(f), _f32(g), _ptr(V), int(dv), _ptr(out), _f32(r)), h.ptr)


def fs_barycentric_map(h: Handle, f, g, Y, out):
    """out[k, i, :] = sum_j P_ij y_j / sum_j P_ij (Y in the handle's dtype, [batch, m, d])."""
    _check(lib().fs_barycentric_map(h.ptr, _f32(f), _f32(g), _ptr(Y), _f32(out)), h.ptr)


def fs_grad_x(h: Handle, f, g, X, Y, grad):
    """grad[k, i, :] = 2 (r_i x_i - sum_j P_ij y_j) (squared Euclidean cost)."""
    _check(lib().fs_grad_x(h.ptr, _f32(f), _f32(g), _ptr(X), _ptr(Y), _f32(grad)), h.ptr)


def fs_transport_apply_t(h: Handle, f, g, U, out, c=None):
    """out[k, j, :] = sum_i P_ij U[k, i, :] (U float32 [batch, n, du]); c[k, j] = sum_i P_ij if given."""
    import torch
    if U.dtype != torch.float32 or out.dtype != torch.float32:
        raise ValueError("U and out must be float32")
    _check(lib().fs_transport_apply_t(h.ptr, _f32(f), _f32(g), _ptr(U), int(U.shape[-1]), _ptr(out), _f32(c)),
           h.ptr)


def fs_grad_y(h: Handle, f, g, X, Y, grad):
    """grad[k, j, :] = 2 (c_j y_j - sum_i P_ij x_i) (squared Euclidean cost)."""
    _check(lib().fs_grad_y(h.ptr, _f32(f), _f32(g), _ptr(X), _ptr(Y), _f32(grad)), h.ptr)


def fs_hvp_x(h: Handle, f, g, X, Y, V, out, max_cg_iters=200, cg_rtol=1e-6) -> int:
    """out = H V, the Hessian of the entropic OT cost with respect to X times V (float32 [n, d]) at
    optimal potentials; returns the conjugate-gradient steps taken."""
    it = ctypes.c_int(0)
    _check(lib().fs_hvp_x(h.ptr, _f32(f), _f32(g), _ptr(X), _ptr(Y), _f32(V), _f32(out), int(max_cg_iters),
                          float(cg_rtol), ctypes.byref(it)), h.ptr)
    return it.value


def fs_selftest_wait(h: Handle, timeout_ms=50) -> int:
    """Run the failure-path self test; returns the library status (FS_ERR_TIMEOUT = 5 expected)."""
    return int(lib().fs_selftest_wait(h.ptr, int(timeout_ms)))
