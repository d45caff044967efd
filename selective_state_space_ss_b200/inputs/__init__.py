"""Seeded synthetic inputs for the selective-scan forward.

This module is the only thing the CUDA path and the fp64 oracle share: it
draws the input tensors (host numpy arrays) that both sides then consume.
It holds none of the scan's arithmetic.

Workload recipe (shapes and distributions of the selective-SSM layer inputs
described in "从Transformer的痛点说起 ... Mamba", sec. 4.2 and 6.2):
  u, z, B, C ~ N(0, 1);  delta ~ N(0, 0.5) (0.5 read as the std);
  dt ~ log-uniform[dt_min, dt_max] per channel, delta_bias = log(expm1(dt))
  (the inverse of softplus, so that softplus(bias) = dt);
  A[d, n] = -(n + 1)               for the integer-spectrum workload, else
  A[d, n] = -(n + 1) * (1 + 0.1 U) with U ~ U(0, 1);
  D[d] ~ N(0, 1).
Activations use the layout [batch, dim, L] and B, C use [batch, N, L], L fastest.

A carried state (initial state of a continued scan, or the state a decode step
advances) is drawn as N(0, 1) fp32 [batch, dim, N]: the magnitude of a state
after many steps of unit-variance inputs with Delta*B*u of order 0.01-1.
Decode-step workloads are Workload objects with seqlen = 1 (one token per
channel); their tensors drop the L axis.

The short convolution's taps [dim, W] and bias [dim] are U(-1/sqrt(W),
1/sqrt(W)), the default initialisation of a depthwise Conv1d of width W; its
input x takes the place of u (N(0, 1)).
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssgen.c")
_LIB = os.path.join(_HERE, "libssgen.so")
_lock = threading.Lock()
_lib = None

# stream ids: one independent counter-based stream per tensor
STREAM = {"u": 1, "delta": 2, "z": 3, "B": 4, "C": 5, "A": 6, "D": 7, "dt": 8, "h0": 9,
          "conv_w": 10, "conv_b": 11}


def build(force: bool = False) -> str:
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp,
                               _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u64, i64, d = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double
            lib.ssgen_fill.argtypes = [u64, u64, u64, i64, d, d, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_void_p, ctypes.c_int]
            lib.ssgen_fill.restype = ctypes.c_int
            lib.ssgen_normal_at.argtypes = [u64, u64]
            lib.ssgen_normal_at.restype = d
            lib.ssgen_uniform_at.argtypes = [u64, u64]
            lib.ssgen_uniform_at.restype = d
            lib.ssgen_stream_key.argtypes = [u64, u64]
            lib.ssgen_stream_key.restype = u64
            _lib = lib
    return _lib


_OUT = {"f32": (0, np.float32), "bf16": (1, np.uint16), "f64": (2, np.float64)}


def fill(seed: int, stream: int, shape, *, kind: str = "normal", mean: float = 0.0,
         scale: float = 1.0, out: str = "f32", offset: int = 0, nthreads: int | None = None):
    """Draw mean + scale * X element by element, X ~ N(0,1) or U(0,1).

    Element j of the flat result is draw number offset + j of the stream, so
    any slice can be regenerated on its own.  out: 'f32', 'bf16' (uint16 bit
    patterns, round-to-nearest-even) or 'f64'.
    """
    code, dt = _OUT[out]
    arr = np.empty(shape, dtype=dt)
    n = arr.size
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load().ssgen_fill(seed & (2**64 - 1), stream, offset, n, mean, scale,
                            0 if kind == "normal" else 1, code, arr.ctypes.data, nthreads)
    if rc != 0:
        raise ValueError("ssgen_fill rejected its arguments")
    return arr


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    dim: int
    seqlen: int
    dstate: int
    dtype: str            # 'f32' or 'bf16' for u, delta, z, B, C
    dt_min: float = 1e-3
    dt_max: float = 1e-1
    a_jitter: bool = True  # False: A[d,n] = -(n+1) exactly
    with_z: bool = True
    with_D: bool = True
    with_bias: bool = True
    softplus: bool = True

    @property
    def elements(self) -> int:
        return self.batch * self.dim * self.seqlen

    def algorithmic_bytes(self) -> int:
        """Bytes a fused scan must move: inputs once, y and the final state once."""
        es = 4 if self.dtype == "f32" else 2
        n_act = 2 + (1 if self.with_z else 0)
        rd = (n_act * self.elements + 2 * self.batch * self.dstate * self.seqlen) * es
        rd += self.dim * self.dstate * 4 + self.dim * 4 * ((1 if self.with_D else 0) + (1 if self.with_bias else 0))
        wr = self.elements * 4 + self.batch * self.dim * self.dstate * 4
        return rd + wr

    def exps(self) -> int:
        return self.elements * self.dstate


# The five named workloads (sizes of the pages' configurations).
WORKLOADS = {
    "b2_l1024_d512_n16_f32": Workload("b2_l1024_d512_n16_f32", 2, 512, 1024, 16, "f32", a_jitter=False),
    "b8_l2048_d1536_n16_bf16": Workload("b8_l2048_d1536_n16_bf16", 8, 1536, 2048, 16, "bf16"),
    "b4_l8192_d5120_n16_bf16": Workload("b4_l8192_d5120_n16_bf16", 4, 5120, 8192, 16, "bf16"),
    "b1_l1048576_d1536_n16_bf16": Workload("b1_l1048576_d1536_n16_bf16", 1, 1536, 1 << 20, 16, "bf16",
                                           dt_min=1e-4, dt_max=1e-2),
}
for _n in (16, 32, 64, 128):
    _w = Workload(f"b16_l4096_d2048_n{_n}_bf16", 16, 2048, 4096, _n, "bf16")
    WORKLOADS[_w.name] = _w


def make_inputs(w: Workload, seed: int = 1234, nthreads: int | None = None) -> dict:
    """Host inputs for workload w.  Activations/B/C as float32 or bf16 bits."""
    out = "f32" if w.dtype == "f32" else "bf16"
    B_, D_, L_, N_ = w.batch, w.dim, w.seqlen, w.dstate
    kw = dict(out=out, nthreads=nthreads)
    x = {
        "u": fill(seed, STREAM["u"], (B_, D_, L_), **kw),
        "delta": fill(seed, STREAM["delta"], (B_, D_, L_), scale=0.5, **kw),
        "B": fill(seed, STREAM["B"], (B_, N_, L_), **kw),
        "C": fill(seed, STREAM["C"], (B_, N_, L_), **kw),
        "z": fill(seed, STREAM["z"], (B_, D_, L_), **kw) if w.with_z else None,
    }
    n1 = np.arange(1, N_ + 1, dtype=np.float64)[None, :]
    if w.a_jitter:
        jit = fill(seed, STREAM["A"], (D_, N_), kind="uniform", out="f64")
        A = -(n1 * (1.0 + 0.1 * jit))
    else:
        A = -np.repeat(n1, D_, axis=0)
    x["A"] = np.ascontiguousarray(A, dtype=np.float32)
    x["D"] = fill(seed, STREAM["D"], (D_,), out="f32") if w.with_D else None
    if w.with_bias:
        lo, hi = np.log(w.dt_min), np.log(w.dt_max)
        dt = np.exp(lo + (hi - lo) * fill(seed, STREAM["dt"], (D_,), kind="uniform", out="f64"))
        x["delta_bias"] = np.log(np.expm1(dt)).astype(np.float32)
    else:
        x["delta_bias"] = None
    return x


def make_row_inputs(w: Workload, seed: int, b: int, dims, nthreads: int | None = None) -> dict:
    """Channels `dims` of batch row b of make_inputs(w, seed), and nothing else.

    Returns the inputs of a workload with batch 1 and dim len(dims): every
    tensor holds exactly the values make_inputs draws for those channels (the
    streams are counter-based, so each row is drawn at its own offset), which
    lets a timing sample of a very long sequence skip the other channels."""
    dims = np.asarray(dims, dtype=np.int64)
    out = "f32" if w.dtype == "f32" else "bf16"
    D_, L_, N_ = w.dim, w.seqlen, w.dstate
    k = len(dims)

    def rows(name, scale=1.0):
        dt = _OUT[out][1]
        arr = np.empty((1, k, L_), dtype=dt)
        for i, d in enumerate(dims):
            arr[0, i] = fill(seed, STREAM[name], (L_,), scale=scale, out=out,
                             offset=int((b * D_ + d) * L_), nthreads=nthreads)
        return arr

    x = {"u": rows("u"), "delta": rows("delta", 0.5), "z": rows("z") if w.with_z else None}
    for name in ("B", "C"):
        x[name] = fill(seed, STREAM[name], (1, N_, L_), out=out, offset=b * N_ * L_,
                       nthreads=nthreads)
    full = make_inputs(dataclasses.replace(w, batch=1, seqlen=1), seed=seed, nthreads=nthreads)
    x["A"] = np.ascontiguousarray(full["A"][dims])
    x["D"] = None if full["D"] is None else np.ascontiguousarray(full["D"][dims])
    x["delta_bias"] = (None if full["delta_bias"] is None
                       else np.ascontiguousarray(full["delta_bias"][dims]))
    return x


def make_state(batch: int, dim: int, dstate: int, seed: int = 1234, scale: float = 1.0,
               nthreads: int | None = None) -> np.ndarray:
    """A carried state [batch, dim, dstate] float32, N(0, scale^2)."""
    return fill(seed, STREAM["h0"], (batch, dim, dstate), scale=scale, nthreads=nthreads)


def make_step_inputs(w: Workload, seed: int = 1234, nthreads: int | None = None) -> dict:
    """Inputs of one decode step: make_inputs at seqlen 1 with the L axis
    dropped (u, delta, z [batch, dim]; B, C [batch, N]) plus the carried
    state [batch, dim, N] under key "state"."""
    if w.seqlen != 1:
        raise ValueError("a decode-step workload has seqlen 1")
    x = make_inputs(w, seed=seed, nthreads=nthreads)
    for k in ("u", "delta", "z", "B", "C"):
        if x[k] is not None:
            x[k] = np.ascontiguousarray(x[k][..., 0])
    x["state"] = make_state(w.batch, w.dim, w.dstate, seed=seed, nthreads=nthreads)
    return x


def step_bytes(w: Workload) -> int:
    """Bytes one decode step must move: the state read and written once, the
    token's inputs, B and C, A, D and the bias, and y."""
    es = 4 if w.dtype == "f32" else 2
    ch = w.batch * w.dim
    n_act = 2 + (1 if w.with_z else 0)
    rd = ch * w.dstate * 4 + n_act * ch * es + 2 * w.batch * w.dstate * es
    rd += w.dim * w.dstate * 4 + w.dim * 4 * ((1 if w.with_D else 0) + (1 if w.with_bias else 0))
    wr = ch * w.dstate * 4 + ch * 4
    return rd + wr


# Decode-step workloads: a batch of sequences advancing one token through one
# layer of a Mamba-6.9B-wide model (d_model 4096, expand 2: dim 8192).
STEP_WORKLOADS = {
    "step_b128_d8192_n16_bf16": Workload("step_b128_d8192_n16_bf16", 128, 8192, 1, 16, "bf16"),
    "step_b128_d8192_n16_f32": Workload("step_b128_d8192_n16_f32", 128, 8192, 1, 16, "f32"),
}


def make_conv(dim: int, width: int, seed: int = 1234) -> tuple[np.ndarray, np.ndarray]:
    """Taps [dim, width] and bias [dim] of the short depthwise convolution."""
    r = 1.0 / np.sqrt(width)
    w = fill(seed, STREAM["conv_w"], (dim, width), kind="uniform", mean=-r, scale=2 * r)
    b = fill(seed, STREAM["conv_b"], (dim,), kind="uniform", mean=-r, scale=2 * r)
    return w, b
