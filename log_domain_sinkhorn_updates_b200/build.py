"""Build the C-ABI shared library ``_lib/libflashsinkhorn.so`` for sm_100a.

nvcc cross-compiles without a GPU.  Each source compiles to its own object
(in parallel, into ``_build/``), and the objects link into one shared
library.  The library links the CUDA runtime statically and reaches the
driver only through cudaGetDriverEntryPoint (for cuTensorMapEncodeTiled), so
it needs nothing but the NVIDIA driver at run time.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT_DIR = os.path.join(HERE, "_lib")
OBJ_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "libflashsinkhorn.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

SOURCES = ["fs_api.cu", "fs_prep.cu", "fs_lse_tc.cu", "fs_lse_tc2.cu", "fs_lse_simt.cu", "fs_apply.cu", "fs_apply_tc.cu",
           "fs_apply_tc2.cu", "fs_apply_tc_q2.cu", "fs_hvp_tc.cu",
           "fs_hvp.cu", "fs_cosine.cu", "fs_selftest.cu", "fs_noalloc.cu"]
HEADERS = ["fs_internal.cuh", "fs_finish.cuh", "fs_prep.cuh", "fs_tc_common.cuh"]

FLAGS = [
    "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
    "-Xptxas", "-warn-spills",
]


def _deps():
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "flashsinkhorn.h"))
    deps.append(os.path.abspath(__file__))
    return [p for p in deps if os.path.exists(p)]


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _deps())


def _obj_stale(src, obj):
    """An object is rebuilt when its source, any shared header or this script is newer."""
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    shared = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "flashsinkhorn.h"),
                                                          os.path.abspath(__file__)]
    return any(os.path.getmtime(p) > t for p in [src] + shared if os.path.exists(p))


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    os.makedirs(OUT_DIR, exist_ok=True)
    os.makedirs(OBJ_DIR, exist_ok=True)
    inc = ["-I", os.path.join(ROOT, "include"), "-I", CSRC]
    extra = ["-Xptxas", "-v"] if verbose else []
    tag = f".tmp{os.getpid()}"

    def compile_one(src_name):
        src = os.path.join(CSRC, src_name)
        obj = os.path.join(OBJ_DIR, src_name.replace(".cu", ".o"))
        if not force and not _obj_stale(src, obj):
            return obj
        cmd = [NVCC, *extra, *FLAGS, *inc, "-c", src, "-o", obj + tag]
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)
        os.replace(obj + tag, obj)
        return obj

    workers = max(1, min(len(SOURCES), os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=workers) as pool:
        objs = list(pool.map(compile_one, SOURCES))
    tmp = LIB + tag
    subprocess.run([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs, "-o", tmp], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
