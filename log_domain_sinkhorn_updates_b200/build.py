"""Build the C-ABI shared library ``_lib/libflashsinkhorn.so`` for sm_100a.

nvcc cross-compiles without a GPU.  The library links the CUDA runtime
statically and reaches the driver only through cudaGetDriverEntryPoint
(for cuTensorMapEncodeTiled), so it needs nothing but the NVIDIA driver at
run time.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT_DIR = os.path.join(HERE, "_lib")
LIB = os.path.join(OUT_DIR, "libflashsinkhorn.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

SOURCES = ["fs_api.cu", "fs_prep.cu", "fs_lse_tc.cu", "fs_lse_tc2.cu", "fs_lse_simt.cu", "fs_apply.cu", "fs_apply_tc.cu",
           "fs_hvp.cu", "fs_selftest.cu", "fs_noalloc.cu"]
HEADERS = ["fs_internal.cuh", "fs_finish.cuh", "fs_prep.cuh", "fs_tc_common.cuh"]

FLAGS = [
    "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
    "-Xptxas", "-warn-spills",
]


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "flashsinkhorn.h"))
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    os.makedirs(OUT_DIR, exist_ok=True)
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, "-shared", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           *[os.path.join(CSRC, s) for s in SOURCES], "-o", tmp]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
