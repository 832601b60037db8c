"""The allocation-free f-update, fs_update_f_noalloc.

It serves callers that cannot allocate device memory when they need an update
(plug-ins whose host framework owns all device memory, services with a fixed
memory budget, latency-critical loops): the handle API allocates in fs_create,
this entry point keeps its scratch in a fixed device array inside the library.

Its result is checked, through the C ABI, on two calls in a row (the second
call must not see anything the first left in the shared scratch):

* against the oracle's f-update ("FlashSinkhorn: IO-aware EOT on GPU",
  Metodologia section 1) within the single-update bar with the 4x margin every
  fp32-accurate mode must leave, 1e-4 * max_ij C_ij / 4;
* against the handle-based fs_update_f on the same inputs, within the
  single-update bar 1e-4 * max_ij C_ij.

Clouds far from the origin (a common offset of 100, and a relative offset of 3
per coordinate between X and Y) pin the centring the entry point does before
its fp32 arithmetic.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import oracle
from helpers import device_inputs, make_problem


def _max_cost(X, Y):
    _, _, cmax = oracle.minplus_bounds(X, Y, np.zeros(Y.shape[0]), np.zeros(Y.shape[0]), 1.0)
    return float(cmax.max())


def _shifted(prob, shift_x, shift_y):
    """The recipe's float32 clouds moved by constant offsets (exact float32 sums), as
    (device X, device Y, oracle X, oracle Y)."""
    import torch
    Xf = (prob.X_dev[0] + np.float32(shift_x)).astype(np.float32)
    Yf = (prob.Y_dev[0] + np.float32(shift_y)).astype(np.float32)
    return (torch.from_numpy(Xf).cuda(), torch.from_numpy(Yf).cuda(), Xf.astype(np.float64),
            Yf.astype(np.float64))


@pytest.mark.gpu
@pytest.mark.parametrize("shift_x,shift_y", [(0.0, 0.0), (100.0, 100.0), (0.0, 3.0)])
def test_noalloc_against_oracle_and_handle_update_on_two_calls(cuda_device, shift_x, shift_y):
    import torch

    import log_domain_sinkhorn_updates_b200 as fs
    # fp32, softmax weights, several 128-row/column tiles with ragged tails
    prob = make_problem("middim", n=1000, m=900)
    _, _, _, b = device_inputs(prob)
    X, Y, Xo, Yo = _shifted(prob, shift_x, shift_y)
    logb = np.log(prob.b_dev[0].astype(np.float64))
    h = fs.fs_create(X[None], Y[None], None, b, eps=prob.eps)
    bar = 1e-4 * _max_cost(Xo, Yo)
    rng = np.random.default_rng(5)
    for call in range(2):
        g_np = (0.5 * rng.standard_normal(prob.m)).astype(np.float32)
        g = torch.from_numpy(g_np).to(cuda_device)
        f_ref = torch.empty(1, prob.n, device=cuda_device)
        fs.fs_update_f(h, g[None], f_ref)
        f_na = torch.full((prob.n,), float("nan"), device=cuda_device)
        fs.fs_update_f_noalloc(X, Y, b[0], g, f_na, prob.eps)
        torch.cuda.synchronize()
        fo = oracle.update_f(Xo, Yo, logb, g_np.astype(np.float64), prob.eps)
        f_na_h = f_na.cpu().numpy().astype(np.float64)
        e_oracle = np.abs(f_na_h - fo).max()
        e_handle = (f_na - f_ref[0]).abs().max().item()
        print(f"shift ({shift_x}, {shift_y}) call {call}: max|f - oracle| = {e_oracle:.3e}, "
              f"max|f - handle| = {e_handle:.3e}, bar {bar:.3e}")
        assert e_oracle <= bar / 4, (call, e_oracle, bar)
        assert e_handle <= bar, (call, e_handle, bar)
    fs.fs_destroy(h)


@pytest.mark.gpu
def test_noalloc_uniform_weights_and_tiny_problem(cuda_device):
    import torch

    import log_domain_sinkhorn_updates_b200 as fs
    prob = make_problem("tiny")  # uniform weights (b = NULL), d = 3
    X, Y, _, _ = device_inputs(prob)
    Xo, Yo, _, logb = oracle.problem_arrays(prob)
    h = fs.fs_create(X, Y, eps=prob.eps)
    bar = 1e-4 * _max_cost(Xo, Yo)
    g = torch.zeros(prob.m, device=cuda_device)
    f_ref = torch.empty(1, prob.n, device=cuda_device)
    fs.fs_update_f(h, g[None], f_ref)
    f_na = torch.empty(prob.n, device=cuda_device)
    fs.fs_update_f_noalloc(X[0], Y[0], None, g, f_na, prob.eps)
    torch.cuda.synchronize()
    fo = oracle.update_f(Xo, Yo, logb, np.zeros(prob.m), prob.eps)
    assert np.abs(f_na.cpu().numpy() - fo).max() <= bar / 4
    assert (f_na - f_ref[0]).abs().max().item() <= bar
    fs.fs_destroy(h)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Checked on the host before any device work (runs without a GPU)."""
    from log_domain_sinkhorn_updates_b200 import binding
    L = binding.lib()
    dummy = ctypes.c_void_p(256)
    st = L.fs_update_f_noalloc(600000, 300000, 8, ctypes.c_float(0.1), dummy, dummy, None, dummy, dummy, None)
    assert st == binding.FS_ERR_INVALID_ARG
    assert b"scratch" in L.fs_last_error(None)
    # the largest accepted point count is 982784 floats: n = 982784 - 2 * 128 with m = 128 fits exactly
    st = L.fs_update_f_noalloc(982784 - 2 * 128 + 1, 128, 8, ctypes.c_float(0.1), dummy, dummy, None, dummy, dummy,
                               None)
    assert st == binding.FS_ERR_INVALID_ARG
    st = L.fs_update_f_noalloc(100, 100, 300, ctypes.c_float(0.1), dummy, dummy, None, dummy, dummy, None)
    assert st == binding.FS_ERR_INVALID_ARG
