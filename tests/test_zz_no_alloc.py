"""The allocation-free f-update, fs_update_f_noalloc.

It serves callers that cannot allocate device memory when they need an update
(code running under CUDA graph capture, plug-ins whose host framework owns all
device memory, latency-critical loops): the handle API allocates in fs_create,
this entry point keeps its scratch in a fixed device array inside the library.
Here its result is compared, through the C ABI, with the handle-based
fs_update_f on the same inputs, on two calls in a row (the second call must not
see anything the first left in the shared scratch), within the tolerance of the
single-update parity tests: 1e-4 * max_ij C_ij.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import oracle
from helpers import device_inputs, make_problem


def _tol(prob):
    Xo, Yo, _, logb = oracle.problem_arrays(prob)
    _, _, cmax = oracle.minplus_bounds(Xo, Yo, logb, np.zeros(prob.m), 1.0)
    return 1e-4 * cmax.max()


@pytest.mark.gpu
def test_noalloc_matches_handle_update_on_two_calls(cuda_device):
    import torch

    import log_domain_sinkhorn_updates_b200 as fs
    # fp32, softmax weights, several 128-row/column tiles with ragged tails
    prob = make_problem("middim", n=1000, m=900)
    X, Y, a, b = device_inputs(prob)
    h = fs.fs_create(X, Y, a, b, eps=prob.eps)
    tol = _tol(prob)
    rng = np.random.default_rng(5)
    for call in range(2):
        g = torch.from_numpy((0.5 * rng.standard_normal(prob.m)).astype(np.float32)).to(cuda_device)
        f_ref = torch.empty(1, prob.n, device=cuda_device)
        fs.fs_update_f(h, g[None], f_ref)
        f_na = torch.full((prob.n,), float("nan"), device=cuda_device)
        fs.fs_update_f_noalloc(X[0], Y[0], b[0], g, f_na, prob.eps)
        torch.cuda.synchronize()
        diff = (f_na - f_ref[0]).abs().max().item()
        assert diff <= tol, (call, diff, tol)
    fs.fs_destroy(h)


@pytest.mark.gpu
def test_noalloc_uniform_weights_and_tiny_problem(cuda_device):
    import torch

    import log_domain_sinkhorn_updates_b200 as fs
    prob = make_problem("tiny")  # uniform weights (b = NULL), d = 3
    X, Y, _, _ = device_inputs(prob)
    h = fs.fs_create(X, Y, eps=prob.eps)
    tol = _tol(prob)
    g = torch.zeros(prob.m, device=cuda_device)
    f_ref = torch.empty(1, prob.n, device=cuda_device)
    fs.fs_update_f(h, g[None], f_ref)
    f_na = torch.empty(prob.n, device=cuda_device)
    fs.fs_update_f_noalloc(X[0], Y[0], None, g, f_na, prob.eps)
    torch.cuda.synchronize()
    assert (f_na - f_ref[0]).abs().max().item() <= tol
    fs.fs_destroy(h)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Checked on the host before any device work (runs without a GPU)."""
    from log_domain_sinkhorn_updates_b200 import binding
    L = binding.lib()
    dummy = ctypes.c_void_p(256)
    st = L.fs_update_f_noalloc(600000, 300000, 8, ctypes.c_float(0.1), dummy, dummy, None, dummy, dummy, None)
    assert st == binding.FS_ERR_INVALID_ARG
    assert b"scratch" in L.fs_last_error(None)
    st = L.fs_update_f_noalloc(100, 100, 300, ctypes.c_float(0.1), dummy, dummy, None, dummy, dummy, None)
    assert st == binding.FS_ERR_INVALID_ARG
