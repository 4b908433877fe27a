"""Build libqknorm.so (the CUDA library behind include/qknorm.h) in-tree.

nvcc cross-compiles for sm_100a without a GPU:

    python -m attention_normalization_b200.build [--force] [--ptxas-verbose]

The CUDA runtime is linked statically, so the library does not depend on which
libcudart the host process (e.g. PyTorch) has loaded; both talk to the same
driver context.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PKG, "libqknorm.so")
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libqknorm.so")


def _inputs() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def is_stale() -> bool:
    if not os.path.exists(LIBRARY):
        return True
    t = os.path.getmtime(LIBRARY)
    return any(os.path.getmtime(p) > t for p in _inputs())


def build(force: bool = False, ptxas_verbose: bool = False, quiet: bool = False) -> str:
    if not force and not is_stale():
        return LIBRARY
    tmp = LIBRARY + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
           "-Xcompiler", "-fPIC,-Wall", "-shared", "-cudart", "static",
           "-I", INCLUDE, "-I", CSRC,
           os.path.join(CSRC, "qknorm_api.cu"), os.path.join(CSRC, "qkv_gemm.cu"), os.path.join(CSRC, "qknorm_tp.cu"),
           os.path.join(CSRC, "qknorm_host.cu"), "-o", tmp]
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libqknorm.so")
    if ptxas_verbose or (r.stderr.strip() and not quiet):
        sys.stderr.write(r.stderr)
    os.replace(tmp, LIBRARY)
    return LIBRARY


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    a = ap.parse_args(argv)
    print(build(force=a.force, ptxas_verbose=a.ptxas_verbose))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
