"""Build libpace.so in-tree with nvcc for sm_100a.

    python -m bit_recurrent_state_pace_b200.build [--verbose-ptxas]

Compiles every ``csrc/*.cu`` into one shared library next to this file.
No fast-math: the encoder must reproduce IEEE fp32 division and rounding.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libpace.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + [
        os.path.join(ROOT, "include", "pace.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def _run(cmd):
    return subprocess.run(cmd, capture_output=True, text=True)


def build(verbose_ptxas: bool = False, force: bool = False) -> str:
    """Compile every csrc/*.cu to an object in parallel, then link libpace.so."""
    if not force and not needs_build():
        return LIB
    from concurrent.futures import ThreadPoolExecutor
    nvcc = nvcc_path()
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    flags = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
             "-I", os.path.join(ROOT, "include")]
    if verbose_ptxas:
        flags = ["-Xptxas", "-v", *flags]
    srcs = sources()
    objs = [os.path.join(objdir, os.path.basename(f)[:-3] + ".o") for f in srcs]
    with ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        procs = list(ex.map(_run, [[nvcc, *flags, "-c", f, "-o", o] for f, o in zip(srcs, objs)]))
    for proc in procs:
        if proc.returncode != 0:
            sys.stderr.write(proc.stdout + proc.stderr)
            raise RuntimeError("nvcc failed building libpace.so")
        if verbose_ptxas:
            sys.stderr.write(proc.stderr)
    proc = _run([nvcc, *ARCH, "-shared", "-o", LIB + ".tmp", *objs])
    if proc.returncode != 0:
        sys.stderr.write(proc.stdout + proc.stderr)
        raise RuntimeError("linking libpace.so failed")
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(a.verbose_ptxas, force=True if a.force or a.verbose_ptxas else False))
