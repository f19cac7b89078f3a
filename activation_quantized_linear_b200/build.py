"""Build, in place with nvcc for sm_100a: libconvrot.so (the layer),
libconvrot_debug.so (the same sources with CONVROT_DEBUG=1: device-side
bounds checks and the tests' fault injection, include/convrot_debug.h) and
libconvrot_bench.so (the benchmark's int8 tensor-core rate probe).

Usage: python activation_quantized_linear_b200/build.py [--verbose] [--ptxas-info]
(run as a script: importing the package loads the library it builds)

The library links the CUDA runtime statically and reaches the driver API only
through cudaGetDriverEntryPoint, so it loads on a machine without a GPU (the
host-side argument checks then work; any compute call reports a CUDA error).
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libconvrot.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)
BENCH_SRC = os.path.join(CSRC, "bench")
BENCH_LIB_PATH = os.path.join(PKG_DIR, "libconvrot_bench.so")
DEBUG_LIB_PATH = os.path.join(PKG_DIR, "libconvrot_debug.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def bench_sources() -> list[str]:
    return sorted(glob.glob(os.path.join(BENCH_SRC, "*.cu")))


def needs_rebuild() -> bool:
    libs = (LIB_PATH, BENCH_LIB_PATH, DEBUG_LIB_PATH)
    if not all(os.path.exists(p) for p in libs):
        return True
    t = min(os.path.getmtime(p) for p in libs)
    deps = sources() + bench_sources() + glob.glob(os.path.join(CSRC, "*.h"))
    deps += glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    deps += [os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def _nvcc(srcs: list[str], out: str, verbose: bool, ptxas_info: bool, defines=()) -> None:
    tmp = out + ".tmp"
    cmd = [
        nvcc_path(), *ARCH_FLAGS, "-lineinfo", "-O3", "-std=c++17",
        "-Xcompiler", "-fPIC,-O3", "-shared", "-cudart", "static",
        "-I", INCLUDE, "-I", CSRC, *defines,
        *srcs, "-o", tmp,
    ]
    if ptxas_info:
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd))
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose or ptxas_info:
        sys.stdout.write(res.stdout + res.stderr)
    os.replace(tmp, out)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    if not force and not ptxas_info and not needs_rebuild():
        return LIB_PATH
    _nvcc(sources(), LIB_PATH, verbose, ptxas_info)
    _nvcc(sources(), DEBUG_LIB_PATH, verbose, ptxas_info, defines=("-DCONVROT_DEBUG=1",))
    _nvcc(bench_sources(), BENCH_LIB_PATH, verbose, ptxas_info)
    return LIB_PATH


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv, ptxas_info="--ptxas-info" in sys.argv)
    print(LIB_PATH)
