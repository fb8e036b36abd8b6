"""Builds the CUDA library libss_b200.so in-tree with nvcc for sm_100a.

    python -m selective_state_space_13_b200.build [--force]
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libss_b200.so")
PROBE_LIB = os.path.join(PKG, "libss_probe.so")  # pipe-throughput probes of the benchmark
PROBE_SOURCES = sorted(glob.glob(os.path.join(PKG, "csrc", "probe", "*.cu")))
SOURCES = sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")))
HEADERS = sorted(glob.glob(os.path.join(PKG, "csrc", "*.h")) +
                 glob.glob(os.path.join(PKG, "csrc", "*.cuh")) +
                 glob.glob(os.path.join(ROOT, "include", "*.h")))

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xptxas", "-v"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every csrc/*.cu to an object (in parallel), then link the shared library."""
    if not force and not stale():
        return LIB
    objdir = tempfile.mkdtemp(prefix="ss_build_")
    try:
        def compile_one(src):
            obj = os.path.join(objdir, os.path.basename(src) + ".o")
            cmd = [_nvcc()] + NVCC_FLAGS + ["-I", os.path.join(ROOT, "include"), "-c", "-o", obj,
                                            src]
            res = subprocess.run(cmd, capture_output=True, text=True)
            if res.returncode != 0:
                raise RuntimeError("nvcc failed on %s:\n%s%s" % (src, res.stdout, res.stderr))
            return obj, res.stderr

        with ThreadPoolExecutor(max(1, min(len(SOURCES), os.cpu_count() or 1))) as ex:
            results = list(ex.map(compile_one, SOURCES))
        if verbose:
            for _, log in results:
                sys.stdout.write(log)
        tmp = LIB + ".tmp%d" % os.getpid()
        cmd = [_nvcc()] + ARCH + ["-shared", "-o", tmp] + [obj for obj, _ in results]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("nvcc link failed:\n" + res.stdout + res.stderr)
        os.replace(tmp, LIB)
    finally:
        shutil.rmtree(objdir, ignore_errors=True)
    return LIB


def build_probe(force: bool = False) -> str:
    """Compile the pipe-throughput probes (measurement only) into libss_probe.so."""
    if not force and os.path.exists(PROBE_LIB) and all(
            os.path.getmtime(f) <= os.path.getmtime(PROBE_LIB) for f in PROBE_SOURCES):
        return PROBE_LIB
    tmp = PROBE_LIB + ".tmp%d" % os.getpid()
    cmd = [_nvcc()] + NVCC_FLAGS + ["-shared", "-o", tmp] + PROBE_SOURCES
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed on the probes:\n" + res.stdout + res.stderr)
    os.replace(tmp, PROBE_LIB)
    return PROBE_LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
    print(build_probe(force="--force" in sys.argv))
