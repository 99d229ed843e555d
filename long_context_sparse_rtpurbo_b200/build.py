"""Builds librtp.so (sm_100a) in-tree with nvcc."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-shared", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    return "nvcc"


def build(verbose: bool = False, extra_flags=(), out_name: str = "librtp.so") -> str:
    """Compiles csrc/rtp_api.cu into ``out_name`` (librtp_trace.so with -DRTP_TRACE records
    per-CTA phase timestamps of the decode kernel in the workspace)."""
    out = os.path.join(HERE, out_name)
    src = os.path.join(HERE, "csrc", "rtp_api.cu")
    cmd = [nvcc(), *NVCC_FLAGS, *extra_flags, "-o", out, src]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    return out


def build_checks(verbose: bool = False) -> str:
    """librtp_checks.so: the library with -DRTP_CHECKS (bounds checks of data-dependent indices
    that record RTP_ECHECK instead of touching memory outside a buffer), for debugging runs
    selected with RTP_LIBRARY_PATH."""
    return build(verbose, ["-DRTP_CHECKS"], "librtp_checks.so")


if __name__ == "__main__":
    print(build(verbose=True))
