"""In-tree build of libmoe.so (the CUDA library behind include/moe.h) for sm_100a.

Each .cu file compiles to an object in parallel; the objects link into one shared library with
the CUDA runtime linked statically, so loading the library needs no GPU driver (symbols can be
inspected on a machine without a GPU; the first CUDA call needs one).
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libmoe.so")
SOURCES = ["api.cu", "repack.cu", "route.cu", "router_tc.cu", "gemm.cu", "decode.cu", "decode_fused.cu", "route_static.cu"]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _deps():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(INCLUDE, "moe.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _deps())


# The decode GEMVs feed 4-bit codes to fp32 FMAs as IEEE subnormals (code * 2^-149, see
# csrc/decode.cu); those FMAs are written as explicit fma.rn.f32 in inline PTX so they keep
# subnormals whatever the compiler flags say, and flush-to-zero builds are refused here as well so
# no other arithmetic silently changes either.
FORBIDDEN_FLAGS = ("-ftz=true", "--ftz=true", "--use_fast_math", "-use_fast_math")


def check_flags(flags) -> None:
    bad = [f for f in flags if f in FORBIDDEN_FLAGS]
    if bad:
        raise ValueError(f"libmoe must be built without flush-to-zero / fast math (got {bad})")


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    check_flags(list(NVCC_FLAGS) + list(extra_flags))
    if not force and up_to_date():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    nvcc = _nvcc()

    def compile_one(src):
        obj = os.path.join(BUILD, os.path.splitext(src)[0] + ".o")
        cmd = [nvcc, *NVCC_FLAGS, *extra_flags, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        if verbose and r.stderr:
            print(r.stderr, file=sys.stderr)
        return obj

    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(compile_one, SOURCES))
    tmp = LIB + ".tmp"
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
           "-Xcompiler", "-fPIC", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
