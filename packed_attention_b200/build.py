"""Build libmfattn.so in-tree for sm_100a with nvcc.

Run ``python -m packed_attention_b200.build`` (or call :func:`build`). The
library is linked against the static CUDA runtime so it does not depend on
which libcudart the host process already loaded. ``build(checked=True)``
builds libmfattn_checked.so from the same sources with -DMF_CHECKED: the
kernels then range-check every global index they compute and report a bad
one as MF_ERR_BOUNDS instead of accessing it.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmfattn.so")
CHECKED_LIB = os.path.join(HERE, "libmfattn_checked.so")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return [os.path.join(CSRC, "mf_attn.cu"), os.path.join(CSRC, "static_scratch.cu"),
            os.path.join(CSRC, "plan.cpp")]


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = glob.glob(os.path.join(CSRC, "*")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = CHECKED_LIB if checked else LIB
    if not force and not _stale(lib):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, *(["-DMF_CHECKED"] if checked else []),
           *(["-Xptxas", "-v"] if verbose else []), "-o", tmp, *sources()]
    subprocess.check_call(cmd, cwd=HERE)
    os.replace(tmp, lib)
    return lib


def build_all(force: bool = False) -> None:
    """The product library and its checked twin."""
    build(force=force)
    build(force=force, checked=True)


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv))
    print(build(force=True, checked=True))
