"""Build libssscan.so (sm_100a) in-tree with nvcc.

    python -m selective_state_space_ss_b200.build [--verbose-ptxas]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libssscan.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return [os.path.join(CSRC, "ss_scan.cu")]


def deps():
    return (sources() + glob.glob(os.path.join(CSRC, "*.cuh"))
            + [os.path.join(ROOT, "include", "ss_scan.h"), os.path.abspath(__file__)])


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in deps())


def build(force: bool = False, ptxas_verbose: bool = False, out: str | None = None,
          defines=()) -> str:
    """Compile libssscan.so (or `out`, with extra -D `defines`, for tuning builds)."""
    target = out or LIB
    if out is None and not force and not stale():
        return LIB
    tmp = target + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
           "-shared", "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-o", tmp,
           *[f"-D{d}" for d in defines], *sources()]
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, target)
    return target


CHECKED_LIB = os.path.join(PKG, "libssscan_checked.so")


def build_checked(force: bool = False) -> str:
    """Compile the checked build (SS_BOUNDS_CHECK: every global index the kernels
    form is compared with its tensor's extent; a miss is skipped and reported by
    ss_last_device_error as SS_ERR_BOUNDS).  Same C ABI; for tests."""
    if not force and os.path.exists(CHECKED_LIB) and not any(
            os.path.getmtime(p) > os.path.getmtime(CHECKED_LIB) for p in deps()):
        return CHECKED_LIB
    return build(out=CHECKED_LIB, defines=["SS_BOUNDS_CHECK"])


def build_probe() -> str:
    """Compile the standalone issue-rate probe (probe_rates.cu) next to the library."""
    out = os.path.join(PKG, "probe_rates")
    src = os.path.join(CSRC, "probe_rates.cu")
    if not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        subprocess.check_call([NVCC, *ARCH, "-O3", "-o", out, src])
    return out


if __name__ == "__main__":
    build_probe()
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    if "--checked" in sys.argv:
        build_checked(force=True)
    print(LIB)
