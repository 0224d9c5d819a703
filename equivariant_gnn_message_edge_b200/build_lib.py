"""Builds libeqconv.so (sm_100a) in-tree with nvcc.

    python -m equivariant_gnn_message_edge_b200.build_lib [-j JOBS] [--force]

Each .cu under csrc/ is compiled to an object in _build/ (in parallel; objects
newer than every source and header are reused) and linked into
equivariant_gnn_message_edge_b200/libeqconv.so with the static CUDA runtime.

The .cu files under csrc/testing/ are test-only builds of library kernels with
changed constants (see each file's header); each becomes its own small
library lib<name>.so beside libeqconv.so, used only by tests/.
"""
from __future__ import annotations

import argparse
import glob
import os
import re
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libeqconv.so")
TESTING = os.path.join(CSRC, "testing")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-std=c++17", "-O3", "-lineinfo", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC",
              "-Xcompiler", "-fvisibility=hidden", "-I", CSRC, "-I", INCLUDE] + ARCH


def _nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.isabs(c) and os.path.exists(c) or not os.path.isabs(c)):
            return c
    return "nvcc"


_INC = re.compile(r'^\s*#\s*include\s*"([^"]+)"', re.M)


def _deps(path: str, seen=None) -> set:
    """The file and every quoted include it reaches (csrc/ and include/)."""
    seen = set() if seen is None else seen
    if path in seen:
        return seen
    seen.add(path)
    with open(path) as f:
        text = f.read()
    for name in _INC.findall(text):
        for d in (os.path.dirname(path), CSRC, INCLUDE):
            cand = os.path.join(d, name)
            if os.path.exists(cand):
                _deps(cand, seen)
                break
    return seen


def _compile(src: str, force: bool, verbose: bool) -> str:
    obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
    if os.path.dirname(src) == TESTING:
        obj = os.path.join(BUILD, "testing_" + os.path.basename(src)[:-3] + ".o")
    if not force and os.path.exists(obj):
        t = os.path.getmtime(obj)
        if all(t > os.path.getmtime(d) for d in _deps(src)):
            return obj
    cmd = [_nvcc()] + NVCC_FLAGS + ["-c", src, "-o", obj + ".tmp"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    os.replace(obj + ".tmp", obj)
    return obj


def build(jobs: int | None = None, force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    # largest instance files first so the pool stays busy
    srcs.sort(key=lambda s: ("inst" not in s, s), reverse=True)
    jobs = jobs or max(1, os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=jobs) as ex:
        objs = list(ex.map(lambda s: _compile(s, force, verbose), srcs))
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs):
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [_nvcc()] + ARCH + ["-shared", "-o", tmp] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
    build_testing(force, verbose)
    return LIB


def build_testing(force: bool = False, verbose: bool = False) -> list:
    """Test-only libraries: csrc/testing/<name>.cu + the tensor-map encoder ->
    lib<name>.so in the package directory."""
    out = []
    tmap = _compile(os.path.join(CSRC, "eqc_tmap.cu"), False, verbose)
    for src in sorted(glob.glob(os.path.join(TESTING, "*.cu"))):
        obj = _compile(src, force, verbose)
        lib = os.path.join(PKG, "lib" + os.path.basename(src)[:-3] + ".so")
        if force or not os.path.exists(lib) or os.path.getmtime(lib) < max(os.path.getmtime(obj),
                                                                             os.path.getmtime(tmap)):
            tmp = lib + f".tmp{os.getpid()}"
            r = subprocess.run([_nvcc()] + ARCH + ["-shared", "-o", tmp, obj, tmap], capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError(f"link failed ({lib}):\n{r.stdout}\n{r.stderr}")
            os.replace(tmp, lib)
        out.append(lib)
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("-j", "--jobs", type=int, default=None)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    a = ap.parse_args(argv)
    print(build(a.jobs, a.force, a.verbose))


if __name__ == "__main__":
    sys.exit(main())
