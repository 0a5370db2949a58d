"""Builds libfa_b200.so in-tree with nvcc for sm_100a.

Usage: ``python -m exact_attention_104_b200.build [--verbose] [--debug]``.  The
library is rebuilt only when a source under ``csrc/`` or the C header is newer
than it (``force=True`` rebuilds unconditionally).  ``--debug`` builds
``libfa_b200_debug.so`` instead, with the device-side checks of ``-DFA_DEBUG``
(the binding loads it when ``FA_B200_DEBUG=1``).
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
LIB_PATH = os.path.join(PKG_DIR, "libfa_b200.so")
DEBUG_LIB_PATH = os.path.join(PKG_DIR, "libfa_b200_debug.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libfa_b200.so")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def needs_build(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose: bool = False, debug: bool = False, out: str | None = None) -> str:
    """Compile the library; returns its path.  ``debug`` adds -DFA_DEBUG and,
    unless ``out`` names another file, writes libfa_b200_debug.so."""
    path = out or (DEBUG_LIB_PATH if debug else LIB_PATH)
    if not force and not needs_build(path):
        return path
    cmd = [
        _nvcc(), *ARCH_FLAGS, "-lineinfo", "-O3", "-std=c++17", "--expt-relaxed-constexpr",
        "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-I", CSRC,
        "-o", path + ".tmp", os.path.join(CSRC, "fa_api.cu"),
    ]
    if debug:
        cmd.insert(1, "-DFA_DEBUG")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + proc.stdout + proc.stderr)
    if verbose:
        sys.stdout.write(proc.stdout + proc.stderr)
    os.replace(path + ".tmp", path)
    return path


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))
