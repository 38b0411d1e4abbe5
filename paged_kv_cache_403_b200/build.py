"""Build the native libraries in-tree with nvcc for sm_100a.

* paged_kv_cache_403_b200/libpa.so  -- the C ABI of include/pa.h (kernels + host block manager)
* synthetic/libpa_synth.so          -- device-side synthetic input generator

Each is rebuilt only when a source or header is newer than the library.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
INCLUDE = os.path.join(ROOT, "include")
CSRC = os.path.join(PKG, "csrc")
LIBPA = os.path.join(PKG, "libpa.so")
SYNTH_SRC = os.path.join(ROOT, "synthetic", "csrc", "synth_gen.cu")
LIBSYNTH = os.path.join(ROOT, "synthetic", "libpa_synth.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
              "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _run(cmd: list[str], verbose: bool) -> None:
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)


def build_libpa(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    srcs = [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cu", ".cpp"))]
    deps = srcs + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".hpp", ".cuh"))]
    deps += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    if force or _stale(LIBPA, deps):
        tmp = LIBPA + ".tmp"
        _run([_nvcc(), *ARCH, *NVCC_FLAGS, *(extra or []), "-I", INCLUDE, "-I", CSRC, "-o", tmp, *srcs],
             verbose)
        os.replace(tmp, LIBPA)
    return LIBPA


def build_synth(force: bool = False, verbose: bool = False) -> str:
    if force or _stale(LIBSYNTH, [SYNTH_SRC]):
        tmp = LIBSYNTH + ".tmp"
        _run([_nvcc(), *ARCH, *NVCC_FLAGS, "-o", tmp, SYNTH_SRC], verbose)
        os.replace(tmp, LIBSYNTH)
    return LIBSYNTH


def build_all(force: bool = False, verbose: bool = False) -> None:
    build_libpa(force, verbose)
    build_synth(force, verbose)


if __name__ == "__main__":
    build_all(force="--force" in sys.argv, verbose=True)
