"""CPU oracle for log-domain Sinkhorn with squared-Euclidean or cosine cost.

TEST INFRASTRUCTURE ONLY: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  It shares no code with
the CUDA library and never imports it.

Two independent implementations live here:

* ``oracle.core``  -- plain C (double, OpenMP over rows), streaming, nothing of
  size n*m stored; the oracle proper, used at every size.
* ``oracle.dense`` -- numpy/scipy brute force on a materialised cost matrix,
  for tiny inputs; used to pin ``oracle.core``.
"""
from .core import (  # noqa: F401
    log_weights, update_f, update_g, update_f_rows, solve, marginals, marginal_error,
    plan_stats, costs, minplus_bounds, num_threads, problem_arrays, COSTS, transport_apply,
    barycentric_projection, grad_x, grad_y,
)
