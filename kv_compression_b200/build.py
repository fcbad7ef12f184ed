"""Build liblca.so (the C-ABI library) in-tree for sm_100a with nvcc."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "liblca.so")
# The range-checked debug build: every guarded index is checked and a failure is
# reported through the device error word (LCA_ERR_DEVICE_CHECK), never a trap.
LIB_CHECKED = os.path.join(HERE, "liblca_checked.so")
SOURCES = ["lca_capi.cu"]
HEADERS = ["checks.cuh", "ptx.cuh", "tc_kernel.cuh", "pair_kernel.cuh", "simt_kernel.cuh", "combine_kernel.cuh",
           "condense_kernel.cuh", "paged_kernel.cuh",
           "gqa_kernel.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale(out: str, deps: list[str]) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra: tuple[str, ...] = (),
          out: str = LIB) -> str:
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "lca.h")]
    if not force and not extra and not _stale(out, deps):
        return out
    cmd = [_nvcc(), *NVCC_FLAGS, *extra, f"-I{INCLUDE}", "-o", out,
           *[os.path.join(CSRC, f) for f in SOURCES]]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    return out


def build_checked(force: bool = False, verbose: bool = False) -> str:
    """The debug library with every kernel index range-checked (-DLCA_CHECKS)."""
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "lca.h")]
    if not force and not _stale(LIB_CHECKED, deps):
        return LIB_CHECKED
    return build(force=True, verbose=verbose, extra=("-DLCA_CHECKS",), out=LIB_CHECKED)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
    print(build_checked(force="--force" in sys.argv, verbose=True))
