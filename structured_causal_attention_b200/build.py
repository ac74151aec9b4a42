"""Build the CUDA library (libhd.so) in-tree for sm_100a with nvcc.

Usage: ``python -m structured_causal_attention_b200.build [--force] [--verbose]``.
Each ``csrc/*.cu`` is compiled to an object in ``_build/`` (in parallel, only
when it or a header changed) and linked into ``libhd.so`` next to this file.
``build(checked=True)`` makes the checked build, ``libhd_checked.so``: the same
sources compiled with ``HD_CHECK_BOUNDS``, whose kernels test every computed
index of a plain load or store against its buffer (objects in
``_build/checked/``). The tests use it; the product path loads ``libhd.so``.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libhd.so")
LIB_CHECKED = os.path.join(HERE, "libhd_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3", "--expt-relaxed-constexpr",
         "-I" + os.path.join(ROOT, "include")]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libhd.so")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False,
          checked: bool = False) -> str:
    nvcc = _nvcc()
    bdir = os.path.join(BUILD, "checked") if checked else BUILD
    lib_path = LIB_CHECKED if checked else LIB
    flags = FLAGS + (["-DHD_CHECK_BOUNDS"] if checked else [])
    os.makedirs(bdir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = _headers()
    objs, jobs = [], []
    for src in sources:
        obj = os.path.join(bdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or _stale(obj, [src] + headers):
            cmd = [nvcc, *ARCH, *flags, "-c", src, "-o", obj]
            if ptxas_verbose:
                cmd += ["-Xptxas", "-v"]
            jobs.append(cmd)

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, r

    failed = []
    if jobs:
        with cf.ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 4)) as ex:
            for cmd, r in ex.map(run, jobs):
                if verbose or ptxas_verbose or r.returncode:
                    sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
                if r.returncode:
                    failed.append(cmd[-3])
    if failed:
        raise RuntimeError("nvcc failed for: " + ", ".join(failed))
    if force or jobs or _stale(lib_path, objs):
        cmd = [nvcc, *ARCH, "-shared", "-o", lib_path + ".tmp", *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode:
            raise RuntimeError("link failed:\n" + r.stdout + r.stderr)
        os.replace(lib_path + ".tmp", lib_path)
    return lib_path


def build_all(force: bool = False, verbose: bool = False) -> None:
    """Both libraries: libhd.so and the checked libhd_checked.so."""
    build(force=force, verbose=verbose)
    build(force=force, verbose=verbose, checked=True)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
          ptxas_verbose="--ptxas" in sys.argv, checked="--checked" in sys.argv)
    print(LIB_CHECKED if "--checked" in sys.argv else LIB)
