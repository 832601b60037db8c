"""B200-native (sm_100a) log-domain Sinkhorn for entropic optimal transport.

The CUDA library (``_lib/libflashsinkhorn.so``, C ABI in
``include/flashsinkhorn.h``) does all the work; ``binding`` marshals
arguments to it.  ``workloads`` draws the seeded synthetic point clouds.

The binding is loaded on first attribute access so that ``workloads`` can
be imported on machines without the built library.
"""
import importlib

__all__ = ["fs_create", "fs_update_f", "fs_update_g", "fs_solve", "fs_marginal_err", "fs_ot_cost", "fs_sync",
           "fs_get_info", "fs_destroy", "fs_last_error", "fs_solve_host", "fs_kernel_launches", "fs_update_f_noalloc",
           "fs_transport_apply", "fs_barycentric_map", "fs_grad_x", "fs_transport_apply_t", "fs_grad_y", "fs_hvp_x",
           "fs_selftest_wait",
           "FsError", "Handle"]


def __getattr__(name):
    if name in __all__:
        mod = importlib.import_module(".binding", __name__)
        mod.lib()  # fail loudly here if the CUDA extension is missing
        return getattr(mod, name)
    raise AttributeError(name)
