"""Build libfdllm.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m block_kv_cache_b200.build [--force]

The shared object lands next to this file, where the binding loads it from.
Rebuilds only when a source or header is newer than the library.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libfdllm.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA library cannot be built")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


# Instrumented build: kernels record per-CTA event clocks (csrc/timeline.cuh),
# readable through fdl_timeline_<file>(); a separate library, loaded only when
# FDLLM_LIB names it.
LIB_TIMELINE = os.path.join(HERE, "libfdllm_timeline.so")


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          timeline: bool = False) -> str:
    lib = LIB_TIMELINE if timeline else LIB
    if not force and not timeline and not _stale():
        return LIB
    tmp = lib + ".tmp"
    flags = ["-DFDL_TIMELINE"] if timeline else []
    cmd = [_nvcc(), *NVCC_FLAGS, *flags, *(extra or []), "-I", INCLUDE, "-I", CSRC, *sources(),
           "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, file=sys.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    extra = [a for a in sys.argv[1:] if a not in ("--force", "-v", "--timeline")]
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, extra=extra,
                timeline="--timeline" in sys.argv))
