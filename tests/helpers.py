"""Shared test helpers: move a drawn workload to the device, run the oracle per problem."""
import numpy as np

import oracle
from log_domain_sinkhorn_updates_b200.workloads import make_problem


def device_inputs(prob, device="cuda"):
    import torch
    if prob.dtype == "bf16":
        X = torch.from_numpy(prob.X_dev.view(np.int16)).view(torch.bfloat16).to(device)
        Y = torch.from_numpy(prob.Y_dev.view(np.int16)).view(torch.bfloat16).to(device)
    else:
        X = torch.from_numpy(prob.X_dev).to(device)
        Y = torch.from_numpy(prob.Y_dev).to(device)
    a = None if prob.a_dev is None else torch.from_numpy(prob.a_dev).to(device)
    b = None if prob.b_dev is None else torch.from_numpy(prob.b_dev).to(device)
    return X, Y, a, b


def oracle_arrays(prob):
    return [oracle.problem_arrays(prob, k) for k in range(prob.batch)]


def max_cost(prob):
    """Exact max_ij C_ij per problem (oracle, double)."""
    out = []
    for X, Y, _, logb in oracle_arrays(prob):
        _, _, cm = oracle.minplus_bounds(X, Y, logb, np.zeros(Y.shape[0]), 1.0)
        out.append(cm.max())
    return np.array(out)


def smooth_potential(rng, count, scale):
    """A seeded, non-trivial potential to feed an update (input data, not method arithmetic)."""
    return (scale * rng.standard_normal(count)).astype(np.float32)


__all__ = ["device_inputs", "oracle_arrays", "max_cost", "smooth_potential", "make_problem"]
