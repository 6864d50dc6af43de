"""Build librankcoll.so (sm_100a) in-tree with nvcc.

    python collective_rc_all_b200/build.py [--force] [--verbose-ptxas]

(Run it by path: importing the package loads the library it builds.)

Objects go to collective_rc_all_b200/_build/, the shared library next to
this file.  Each .cu compiles in parallel.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "librankcoll.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
EXPORTS = os.path.join(HERE, "exports.map")  # only the C ABI (rc_*) is exported

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# -fmad=false: no contraction of a*b+c (the fold is adds and one multiply, and
# the results must be bit-identical to one IEEE operation each).
NVFLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-fmad=false", "--expt-relaxed-constexpr",
                  "-Xcompiler", "-fPIC,-O2", "-I", INCLUDE]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    os.makedirs(OBJ, exist_ok=True)
    srcs = _sources()
    hdrs = _headers()
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    jobs = []
    for s in srcs:
        o = os.path.join(OBJ, os.path.basename(s)[:-3] + ".o")
        if force or verbose_ptxas or _stale(o, [s] + hdrs):
            jobs.append([nvcc(), *NVFLAGS, *extra, "-c", s, "-o", o])
    if jobs:
        with cf.ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 4)) as ex:
            results = list(ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), jobs))
        for cmd, r in zip(jobs, results):
            if r.stdout or r.stderr:
                sys.stderr.write(r.stdout + r.stderr)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed: {' '.join(cmd)}")
    objs = [os.path.join(OBJ, os.path.basename(s)[:-3] + ".o") for s in srcs]
    if force or jobs or _stale(LIB, objs + [EXPORTS]):
        tmp = LIB + ".tmp"
        subprocess.run([nvcc(), *ARCH, "-shared", "-Xlinker", f"--version-script={EXPORTS}", "-o", tmp, *objs],
                       check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv))
