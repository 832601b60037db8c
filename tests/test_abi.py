"""The C-ABI library: builds, loads, exports every declared symbol, and its host-side
argument checks answer before any device work (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names.update(re.findall(r"^FS_API\s+[\w\s\*]+?\b(fs_\w+)\s*\(", txt, flags=re.M))
    return names


@pytest.fixture(scope="module")
def L():
    from log_domain_sinkhorn_updates_b200 import build, binding
    build.build()
    return binding.lib()


def test_exports_every_declared_symbol(L):
    declared = _declared()
    assert {"fs_create", "fs_update_f", "fs_update_g", "fs_solve", "fs_marginal_err", "fs_ot_cost",
            "fs_destroy", "fs_last_error"} <= declared
    for name in declared:
        assert hasattr(L, name), name
    from log_domain_sinkhorn_updates_b200 import binding
    assert set(binding.EXPORTS) == declared


def test_python_names_match_c_abi():
    import log_domain_sinkhorn_updates_b200 as pkg
    for name in _declared():
        assert callable(getattr(pkg, name))


def test_invalid_arguments_rejected_on_host(L):
    from log_domain_sinkhorn_updates_b200.binding import FsDesc, FS_ERR_INVALID_ARG
    out = ctypes.c_void_p()
    dummy = ctypes.c_void_p(16)
    for desc in [FsDesc(1, 0, 5, 3, 0, 0, 0.1), FsDesc(1, 5, 5, 0, 0, 0, 0.1), FsDesc(0, 5, 5, 3, 0, 0, 0.1),
                 FsDesc(1, 5, 5, 3, 0, 0, 0.0), FsDesc(1, 5, 5, 3, 0, 0, float("nan")),
                 FsDesc(1, 5, 5, 3, 7, 0, 0.1), FsDesc(1, 5, 5, 3, 0, 9, 0.1), FsDesc(1, 5, 5, 3, 0, 0, 0.1, 7)]:
        st = L.fs_create(ctypes.byref(desc), dummy, dummy, None, None, None, ctypes.byref(out))
        assert st == FS_ERR_INVALID_ARG
        assert out.value is None
        assert L.fs_last_error(None)
    st = L.fs_create(ctypes.byref(FsDesc(1, 5, 5, 3, 0, 0, 0.1)), None, dummy, None, None, None, ctypes.byref(out))
    assert st == FS_ERR_INVALID_ARG
    assert L.fs_destroy(None) == 0
    assert L.fs_update_f(None, dummy, dummy) == FS_ERR_INVALID_ARG
    assert L.fs_solve(None, dummy, dummy, 3, 0) == FS_ERR_INVALID_ARG


def test_no_device_is_reported_not_crashed(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    from log_domain_sinkhorn_updates_b200.binding import FsDesc, FS_ERR_CUDA
    out = ctypes.c_void_p()
    dummy = ctypes.c_void_p(16)
    st = L.fs_create(ctypes.byref(FsDesc(1, 5, 5, 3, 0, 0, 0.1)), dummy, dummy, None, None, None, ctypes.byref(out))
    assert st == FS_ERR_CUDA
    assert b"device" in L.fs_last_error(None).lower()


def test_host_solve_rejects_bad_sizes(L):
    from log_domain_sinkhorn_updates_b200 import binding
    with pytest.raises(binding.FsError):
        binding.fs_solve_host(np.zeros((1, 0, 3), np.float32), np.zeros((1, 4, 3), np.float32), None, None,
                              np.zeros((1, 4), np.float32), 0.1, 3)


def _struct_fields(name):
    """Field names, in order, of the typedef struct `name` in include/flashsinkhorn.h."""
    txt = open(os.path.join(ROOT, "include", "flashsinkhorn.h")).read()
    body = re.search(r"typedef struct \{([^{}]*)\}\s*" + name + r"\s*;", txt).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = []
    for decl in body.split(";"):
        decl = decl.strip()
        if decl:
            fields += [v.strip().lstrip("*") for v in decl.split(None, 1)[1].split(",")]
    return fields


@pytest.mark.parametrize("cname,pyname", [("fs_desc", "FsDesc"), ("fs_info", "FsInfo")])
def test_ctypes_structs_match_header(cname, pyname):
    """The binding's ctypes mirrors of the C structs list the header's fields in the
    header's order (a missing or moved field would shift every later one)."""
    from log_domain_sinkhorn_updates_b200 import binding
    assert [f for f, _ in getattr(binding, pyname)._fields_] == _struct_fields(cname)


def test_every_entry_point_rejects_a_null_handle_on_host(L):
    """Every call that takes a handle answers FS_ERR_INVALID_ARG for a null handle (or
    null required pointers) before any device work; the allocation-free update checks
    its sizes and limits on the host too."""
    from log_domain_sinkhorn_updates_b200.binding import FS_ERR_INVALID_ARG, FsInfo
    p = ctypes.c_void_p(16)
    d = ctypes.c_double()
    info = FsInfo()
    i = ctypes.c_int()
    calls = {
        "fs_update_g": (None, p, p),
        "fs_marginal_err": (None, p, p, ctypes.byref(d), ctypes.byref(d)),
        "fs_ot_cost": (None, p, p, ctypes.byref(d), ctypes.byref(d)),
        "fs_sync": (None,),
        "fs_get_info": (None, ctypes.byref(info)),
        "fs_transport_apply": (None, p, p, p, 3, p, p),
        "fs_transport_apply_t": (None, p, p, p, 3, p, p),
        "fs_barycentric_map": (None, p, p, p, p),
        "fs_grad_x": (None, p, p, p, p, p),
        "fs_grad_y": (None, p, p, p, p, p),
        "fs_selftest_wait": (None, 50),
    }
    for name, args in calls.items():
        assert getattr(L, name)(*args) == FS_ERR_INVALID_ARG, name
    # a private ctypes view of the library, so these argtypes leave the binding's alone
    from log_domain_sinkhorn_updates_b200 import binding
    L2 = ctypes.CDLL(binding.LIB_PATH)
    L2.fs_hvp_x.argtypes = [ctypes.c_void_p] * 7 + [ctypes.c_int, ctypes.c_double, ctypes.c_void_p]
    assert L2.fs_hvp_x(None, p, p, p, p, p, p, 10, 1e-6, ctypes.byref(i)) == FS_ERR_INVALID_ARG
    L2.fs_update_f_noalloc.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float] + \
        [ctypes.c_void_p] * 6
    for n, m, dd, eps in [(0, 5, 3, 0.1), (5, 5, 0, 0.1), (5, 5, 3, 0.0), (5, 5, 257, 0.1), (1 << 20, 5, 3, 0.1)]:
        assert L2.fs_update_f_noalloc(n, m, dd, eps, p, p, None, p, p, None) == FS_ERR_INVALID_ARG, (n, m, dd, eps)
    assert L2.fs_update_f_noalloc(5, 5, 3, 0.1, None, p, None, p, p, None) == FS_ERR_INVALID_ARG
