"""Build libfa.so (the CUDA library) in-tree with nvcc for sm_100a.

Usage: ``python -m exact_io_aware_96_b200.build`` (or ``__graft_entry__.build()``).
The CUDA runtime is linked statically; the driver API is reached through
cudaGetDriverEntryPoint, so the library needs no libcuda at link time.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libfa.so")
SOURCES = [os.path.join(CSRC, "fa_api.cu")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


LIB_CHECK = os.path.join(HERE, "libfa_check.so")


def build(verbose: bool = False, extra: list[str] | None = None, check: bool = False) -> str:
    """Build libfa.so, or with check=True libfa_check.so: the same sources
    compiled with FA_CHECK=1 (device-side index and bounds checks)."""
    out = LIB_CHECK if check else LIB
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared",
           "-I" + INCLUDE, "-I" + CSRC, "-o", out + ".tmp", *(["-DFA_CHECK=1"] if check else []), *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    if extra:
        cmd[1:1] = extra
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    os.replace(out + ".tmp", out)
    if verbose:
        sys.stdout.write(res.stdout + res.stderr)
    return out


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, check="--check" in sys.argv))
