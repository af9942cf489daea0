"""Build libqlinear.so in-tree with nvcc for sm_100a.

``python -m fp8_linear_layers_b200.build [--verbose]``.  Each ``csrc/*.cu`` is
compiled separately (in parallel, skipped when up to date) and linked into
``fp8_linear_layers_b200/libqlinear.so`` with the CUDA runtime linked
statically, so the library loads on a machine without a GPU (for the symbol
checks) and needs only the driver on a B200.

Flags: ``-gencode arch=compute_100a,code=sm_100a -O3 -lineinfo``; no fast
math (the scales and quotients must be IEEE divisions and subnormals must
survive), no relocatable device code.
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
OBJ_DIR = os.path.join(os.path.dirname(HERE), "_build", "obj")
LIB_PATH = os.path.join(HERE, "libqlinear.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
                     "--expt-relaxed-constexpr", "-I", INCLUDE]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers() -> list[str]:
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _compile(src: str, obj: str, verbose: bool) -> str:
    cmd = [_nvcc(), *NVCC_FLAGS, "-c", src, "-o", obj]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stderr}")
    return r.stderr


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(OBJ_DIR, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    newest_header = max((os.path.getmtime(h) for h in _headers()), default=0.0)
    jobs = []
    objs = []
    for s in srcs:
        o = os.path.join(OBJ_DIR, os.path.basename(s)[:-3] + ".o")
        objs.append(o)
        stale = (force or verbose or not os.path.exists(o)
                 or os.path.getmtime(o) < max(os.path.getmtime(s), newest_header))
        if stale:
            jobs.append((s, o))
    logs = []
    if jobs:
        with concurrent.futures.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
            futs = [ex.submit(_compile, s, o, verbose) for s, o in jobs]
            for f in futs:
                logs.append(f.result())
    need_link = bool(jobs) or not os.path.exists(LIB_PATH) or \
        os.path.getmtime(LIB_PATH) < max(os.path.getmtime(o) for o in objs)
    if need_link:
        tmp = LIB_PATH + f".tmp{os.getpid()}"
        r = subprocess.run([_nvcc(), *ARCH, "-shared", "-cudart", "static", *objs, "-o", tmp],
                           capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr}")
        os.replace(tmp, LIB_PATH)
    if verbose:
        print("\n".join(l for l in logs if l))
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
