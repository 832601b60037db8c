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
