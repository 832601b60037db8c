"""The seeded input generator: shapes, determinism, dtype casts, distributions."""
import numpy as np
import pytest
import torch

from log_domain_sinkhorn_updates_b200.workloads import WORKLOADS, bf16_round, make_problem


def test_bf16_round_matches_torch_cast():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000) * s for s in (1e-3, 1.0, 1e3)])
    bits, vals = bf16_round(x)
    t = torch.tensor(x.astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(bits, t.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(vals, t.to(torch.float64).numpy())


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_small_draws_have_recipe_shapes_and_are_deterministic(name):
    p = make_problem(name, n=100, m=90, batch=min(WORKLOADS[name]["batch"], 3))
    q = make_problem(name, n=100, m=90, batch=min(WORKLOADS[name]["batch"], 3))
    assert p.X.shape == (p.batch, 100, p.d) and p.Y.shape == (p.batch, 90, p.d)
    assert np.array_equal(p.X, q.X) and np.array_equal(p.Y, q.Y)
    if p.dtype == "bf16":
        assert p.X_dev.dtype == np.uint16
    else:
        assert p.X_dev.dtype == np.float32
        assert np.array_equal(p.X_dev.astype(np.float64), p.X)
    if p.a is not None:
        assert np.all(p.a > 0) and np.allclose(p.a.sum(1), 1.0, atol=1e-6)
        assert np.array_equal(p.a_dev.astype(np.float64), p.a)


def test_distribution_recipes():
    p = make_problem("cloud3d", n=20000, m=20000)
    r = np.linalg.norm(p.X[0], axis=1)
    assert abs(r.mean() - 1.0) < 2e-3 and r.std() < 0.02       # unit sphere + 0.01 noise
    p = make_problem("middim", n=4000, m=4000)
    assert abs(p.Y[0].mean() - 0.5) < 0.01 and abs(p.X[0].var() - 1 / 64) < 1e-3
    p = make_problem("highdim", n=2000, m=2000)
    assert abs(p.Y[0].var() - 1 / 128) < 5e-4 and abs(p.Y[0].mean()) < 5e-3
    p = make_problem("batched", n=500, m=500, batch=4)
    mx = p.X.mean(axis=1)
    my = p.Y.mean(axis=1)
    assert np.abs(mx - my).max() < 0.05                        # shared per-problem mean
    assert mx.std() > 0.5                                       # means differ across problems
