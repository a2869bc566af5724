"""Build libmoe_route.so in-tree with nvcc for sm_100a.

    python combine_moe_route_08_b200/build.py [--force] [--ptxas-v]

(Run as a script or load it by path: importing the package itself requires
the library to exist already.)

Floating-point flags: no flush-to-zero, IEEE division and square root, and
no FMA contraction, so the bit-exact paths (fp8 scales and codes, the fp32
combine sum) do exactly the operations their comments state.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmoe_route.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "--ftz=false", "--prec-div=true", "--prec-sqrt=true", "--fmad=false",
    "-Xcompiler", "-fPIC,-O2,-Wall",
    "-Xptxas", "-warn-spills",
    "-shared",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def nvcc() -> str:
    for cand in [os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"]:
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          csrc: str = CSRC, out: str = LIB) -> str:
    """Compile every .cu under csrc/ into one shared library (static cudart):
    one nvcc process per source file, in parallel, then one link."""
    if not force and out == LIB and not _stale():
        return out
    import concurrent.futures as cf
    srcs = sorted(glob.glob(os.path.join(csrc, "*.cu")))
    objdir = os.path.join(os.path.dirname(out), "_build", f"obj{os.getpid()}")
    os.makedirs(objdir, exist_ok=True)
    compile_flags = [f for f in NVCC_FLAGS if f != "-shared"]

    def one(src):
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [nvcc(), *compile_flags, *(extra or []), "-I", INCLUDE, "-I", csrc, "-c", "-o", obj, src]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(len(srcs), os.cpu_count() or 4)) as pool:
        objs = list(pool.map(one, srcs))
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run([nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs],
                   check=True)
    os.replace(tmp, out)
    for o in objs:
        os.remove(o)
    os.rmdir(objdir)
    return out


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
    print(LIB)
