"""Build libssscan.so (sm_100a) in-tree with nvcc.

    python -m selective_state_space_ss_b200.build [--verbose-ptxas]
"""
from __future__ import annotations

import glob
import hashlib
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


def source_hash(defines=()) -> str:
    """Hash of every source the library is built from, and the -D flags."""
    h = hashlib.sha256(" ".join(defines).encode())
    for p in sorted(deps()):
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode() + b"\0" + f.read())
    return h.hexdigest()


def _stale(target: str, defines=()) -> bool:
    # by content, not by time stamps (a copied tree may carry any mtimes): the
    # hash of the sources a library was built from sits beside it in <lib>.src
    try:
        with open(target + ".src") as f:
            return not os.path.exists(target) or f.read().strip() != source_hash(defines)
    except OSError:
        return True


def stale() -> bool:
    return _stale(LIB)


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
    with open(target + ".src", "w") as f:
        f.write(source_hash(defines))
    return target


CHECKED_LIB = os.path.join(PKG, "libssscan_checked.so")


def build_checked(force: bool = False) -> str:
    """Compile the checked build (SS_BOUNDS_CHECK: every global index the kernels
    form is compared with its tensor's extent; a miss is skipped and reported by
    ss_last_device_error as SS_ERR_BOUNDS).  Same C ABI; for tests."""
    if not force and not _stale(CHECKED_LIB, ["SS_BOUNDS_CHECK"]):
        return CHECKED_LIB
    return build(out=CHECKED_LIB, defines=["SS_BOUNDS_CHECK"])


def build_probe() -> str:
    """Compile the standalone issue-rate probe (probe_rates.cu) next to the library."""
    out = os.path.join(PKG, "probe_rates")
    src = os.path.join(CSRC, "probe_rates.cu")
    with open(src, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()
    try:
        with open(out + ".src") as f:
            fresh = os.path.exists(out) and f.read().strip() == h
    except OSError:
        fresh = False
    if not fresh:
        subprocess.check_call([NVCC, *ARCH, "-O3", "-o", out, src])
        with open(out + ".src", "w") as f:
            f.write(h)
    return out


if __name__ == "__main__":
    build_probe()
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    if "--checked" in sys.argv:
        build_checked(force=True)
    print(LIB)
