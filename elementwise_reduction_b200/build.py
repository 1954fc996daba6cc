"""Build libdyt.so (the C-ABI library) in-tree with nvcc for sm_100a.

Run as ``python elementwise_reduction_b200/build.py`` (by path: importing the package
loads the library this script builds).
No GPU is needed to build.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libdyt.so")
SOURCES = [os.path.join(CSRC, f) for f in ("dyt_api.cu", "dyt_inst_f32.cu", "dyt_inst_bf16.cu", "dyt_inst_f16.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("dyt_kernels.cuh", "dyt_math.cuh", "dyt_async.cuh", "dyt_finalize.cuh",
                                                  "dyt_select.cuh", "dyt_select_impl.cuh")] + [
    os.path.join(INCLUDE, "dyt.h")]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-std=c++17", "-O3", "-lineinfo", *ARCH, "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build(force: bool = False, verbose: bool = False, defines=(), out: str | None = None) -> str:
    """Compile libdyt.so if any source is newer than it. Returns its path.

    The translation units (the C ABI, and the kernels of each activation dtype)
    compile in parallel and are linked into one shared library.
    defines: extra -D tuning overrides; out: another output path (for sweeps).
    """
    import concurrent.futures
    import tempfile

    out = out or LIB
    if not force and not defines and os.path.exists(out):
        built = os.path.getmtime(out)
        if all(os.path.getmtime(d) <= built for d in DEPS):
            return out
    with tempfile.TemporaryDirectory() as tmp:
        def compile_one(src: str) -> str:
            obj = os.path.join(tmp, os.path.basename(src) + ".o")
            cmd = [nvcc(), *NVCC_FLAGS, *(["-Xptxas", "-v"] if verbose else []), *[f"-D{d}" for d in defines],
                   "-c", "-o", obj, src]
            subprocess.check_call(cmd)
            return obj

        with concurrent.futures.ThreadPoolExecutor(len(SOURCES)) as pool:
            objs = list(pool.map(compile_one, SOURCES))
        subprocess.check_call([nvcc(), *ARCH, "-shared", "-o", out + ".tmp", *objs, "-lcudart"])
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv))
