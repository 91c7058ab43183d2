"""Build libfa.so in-tree with nvcc for sm_100a (B200).

``python -m exact_io_aware_81_b200.build`` compiles ``csrc/fa_api.cu`` (which includes the
kernel headers) into ``exact_io_aware_81_b200/libfa.so``, next to the binding that loads it,
and the debug build ``libfa_debug.so`` (``-DFA_DEBUG_CHECKS``: the kernels check the bounds
of every global-memory index they compute and report a failure through the error word).
The CUDA runtime is linked statically, so the library needs only the NVIDIA driver.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfa.so")
LIB_DEBUG = os.path.join(PKG, "libfa_debug.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cuh")))


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + [os.path.join(INCLUDE, "fa.h")]
    return any(os.path.getmtime(s) > t for s in deps)


def build(force: bool = False, verbose: bool = False, extra=None, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not needs_build(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc_path(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC,
           "-o", tmp, os.path.join(CSRC, "fa_api.cu")]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    if debug:
        cmd += ["-DFA_DEBUG_CHECKS"]
    if extra:
        cmd += list(extra)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stdout.write(res.stdout + res.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    print(build(force="--force" in sys.argv, debug=True))
