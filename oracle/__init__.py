"""fp64 CPU oracle for the S6 selective-scan forward (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package.  The product path (the CUDA library and
its binding) never imports, links or runs anything here, and this package
imports nothing from the product.

The arithmetic lives in ``ss_oracle.c`` (plain serial recurrence in double,
threads over channels); this module only compiles it with gcc and marshals
numpy arrays.  See the C file's header for the passages it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ss_oracle.c")
_LIB = os.path.join(_HERE, "libssoracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile ss_oracle.c into libssoracle.so (gcc, -O2, no fast-math)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
             "-ffp-contract=off", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            vp, i64 = ctypes.c_void_p, ctypes.c_int64
            lib.oracle_scan_fwd.argtypes = [
                vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int, ctypes.c_int,
                i64, i64, i64, ctypes.c_int, vp, i64, vp, vp, vp, vp, vp, ctypes.c_int, ctypes.c_int,
                ctypes.c_int]
            lib.oracle_scan_fwd.restype = ctypes.c_int
            lib.oracle_scan_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int,
                                            ctypes.c_int, i64, i64, i64, ctypes.c_int, vp, vp,
                                            vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int]
            lib.oracle_scan_bwd.restype = ctypes.c_int
            lib.oracle_softplus.argtypes = [ctypes.c_double]
            lib.oracle_softplus.restype = ctypes.c_double
            lib.oracle_silu.argtypes = [ctypes.c_double]
            lib.oracle_silu.restype = ctypes.c_double
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _stored(a, name):
    """Return (contiguous array, dtype code).  bf16 travels as uint16 bits."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, F32
    if a.dtype == np.uint16:
        return a, BF16
    raise TypeError(f"{name}: expected float32 or uint16 (bf16 bits), got {a.dtype}")


def scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None,
             softplus=True, channels=None, nthreads=None, h0=None, conv_weight=None,
             conv_bias=None, zoh=False):
    """Serial fp64 selective scan.

    u, delta, z: [batch, dim, L]; B, C: [batch, N, L]; all float32 or all
    bf16 bits (uint16).  A: [dim, N] float32; D, delta_bias: [dim] float32.
    channels: optional 1-D int array of flat channel ids (b*dim + d); then
    only those rows are computed.  h0: optional [batch, dim, N] initial state
    (widened to float64; the scan starts from zero without it).
    conv_weight: optional [dim, W] float32 taps of the causal depthwise
    convolution; u then holds the convolution's input x and the scan runs on
    SiLU(conv(x) + conv_bias).  conv_bias: optional [dim] float32.
    zoh: exact zero-order hold, B_bar = expm1(Delta A) / A * B (Delta B where
    A = 0), instead of the simplified Delta B.
    Returns (y, last_state) as float64 with
    shapes [batch, dim, L] / [batch, dim, N], or [len(channels), L] /
    [len(channels), N] when channels is given.
    """
    u, dt = _stored(u, "u")
    delta, dt2 = _stored(delta, "delta")
    B, dt3 = _stored(B, "B")
    C, dt4 = _stored(C, "C")
    if len({dt, dt2, dt3, dt4}) != 1:
        raise TypeError("u, delta, B, C must share one stored dtype")
    if z is not None:
        z, dt5 = _stored(z, "z")
        if dt5 != dt:
            raise TypeError("z must share the stored dtype of u")
    batch, dim, L = u.shape
    N = B.shape[1]
    if delta.shape != u.shape or B.shape != (batch, N, L) or C.shape != B.shape:
        raise ValueError("shape mismatch")
    if z is not None and z.shape != u.shape:
        raise ValueError("z shape mismatch")
    A = np.ascontiguousarray(A, dtype=np.float32)
    if A.shape != (dim, N):
        raise ValueError("A must be [dim, N]")
    D = None if D is None else np.ascontiguousarray(D, dtype=np.float32)
    delta_bias = None if delta_bias is None else np.ascontiguousarray(delta_bias, dtype=np.float32)
    if h0 is not None:
        h0 = np.ascontiguousarray(h0, dtype=np.float64)
        if h0.shape != (batch, dim, N):
            raise ValueError("h0 must be [batch, dim, N]")
    conv_w = conv_b = None
    width = 0
    if conv_weight is not None:
        conv_w = np.ascontiguousarray(conv_weight, dtype=np.float32)
        if conv_w.ndim != 2 or conv_w.shape[0] != dim:
            raise ValueError("conv_weight must be [dim, W]")
        width = conv_w.shape[1]
        if conv_bias is not None:
            conv_b = np.ascontiguousarray(conv_bias, dtype=np.float32)
            if conv_b.shape != (dim,):
                raise ValueError("conv_bias must be [dim]")
    if channels is not None:
        channels = np.ascontiguousarray(channels, dtype=np.int64)
        nch = channels.size
        y = np.empty((nch, L), np.float64)
        h = np.empty((nch, N), np.float64)
    else:
        nch = batch * dim
        y = np.empty((batch, dim, L), np.float64)
        h = np.empty((batch, dim, N), np.float64)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load().oracle_scan_fwd(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(delta_bias), int(bool(softplus)), dt, batch, dim, L, N,
        _ptr(channels), nch, _ptr(y), _ptr(h), _ptr(h0), _ptr(conv_w), _ptr(conv_b), width,
        int(bool(zoh)), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_scan_fwd rejected its arguments")
    return y, h


def scan_step(state, u, delta, A, B, C, D=None, z=None, delta_bias=None,
              softplus=True, nthreads=None):
    """One recurrent (decode) step: the scan over a single token started from
    the carried state.

    state: [batch, dim, N] (any float dtype, widened to float64); u, delta, z:
    [batch, dim]; B, C: [batch, N]; the rest as in scan_fwd.  Returns
    (y [batch, dim], new_state [batch, dim, N]) as float64.
    """
    y, h = scan_fwd(np.asarray(u)[..., None], np.asarray(delta)[..., None], A,
                    np.asarray(B)[..., None], np.asarray(C)[..., None], D=D,
                    z=None if z is None else np.asarray(z)[..., None],
                    delta_bias=delta_bias, softplus=softplus, nthreads=nthreads,
                    h0=state)
    return y[..., 0], h


def scan_bwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True, dy=None,
             dlast=None, nthreads=None):
    """Reverse-mode gradients of the scan (simplified B_bar, zero initial state).

    Inputs as scan_fwd; dy: [batch, dim, L] gradient of the loss with respect
    to y; dlast: optional [batch, dim, N] gradient with respect to the final
    state.  Returns a dict of float64 arrays: du, ddelta, dz (None without z),
    dA [dim, N], dB, dC [batch, N, L], dD, ddelta_bias [dim].
    """
    u, dt = _stored(u, "u")
    delta, _ = _stored(delta, "delta")
    B, _ = _stored(B, "B")
    C, _ = _stored(C, "C")
    if z is not None:
        z, _ = _stored(z, "z")
    batch, dim, L = u.shape
    N = B.shape[1]
    A = np.ascontiguousarray(A, dtype=np.float32)
    D = None if D is None else np.ascontiguousarray(D, dtype=np.float32)
    delta_bias = None if delta_bias is None else np.ascontiguousarray(delta_bias, dtype=np.float32)
    dy = np.ascontiguousarray(dy, dtype=np.float64)
    if dy.shape != (batch, dim, L):
        raise ValueError("dy must be [batch, dim, L]")
    if dlast is not None:
        dlast = np.ascontiguousarray(dlast, dtype=np.float64)
        if dlast.shape != (batch, dim, N):
            raise ValueError("dlast must be [batch, dim, N]")
    out = {"du": np.empty((batch, dim, L)), "ddelta": np.empty((batch, dim, L)),
           "dz": np.empty((batch, dim, L)) if z is not None else None,
           "dA": np.empty((dim, N)), "dB": np.empty((batch, N, L)), "dC": np.empty((batch, N, L)),
           "dD": np.empty(dim), "ddelta_bias": np.empty(dim)}
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load().oracle_scan_bwd(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
        int(bool(softplus)), dt, batch, dim, L, N, _ptr(dy), _ptr(dlast), _ptr(out["du"]),
        _ptr(out["ddelta"]), _ptr(out["dz"]), _ptr(out["dA"]), _ptr(out["dB"]), _ptr(out["dC"]),
        _ptr(out["dD"]), _ptr(out["ddelta_bias"]), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_scan_bwd rejected its arguments")
    return out


def softplus(x: float) -> float:
    return _load().oracle_softplus(float(x))


def silu(z: float) -> float:
    return _load().oracle_silu(float(z))
