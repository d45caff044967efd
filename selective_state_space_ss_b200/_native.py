"""ctypes binding of libssscan.so (the C ABI in include/ss_scan.h).

Argument marshalling only: every step of the scan runs in the CUDA library.
PyTorch provides device memory and the stream.  There is no CPU fallback; if
the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

# SSSCAN_LIBRARY may point at another build of the same library (tuning runs).
_LIB_PATH = os.environ.get("SSSCAN_LIBRARY") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "libssscan.so")
_lock = threading.Lock()
_lib = None

SS_OK, SS_ERR_INVALID_ARG, SS_ERR_UNSUPPORTED, SS_ERR_CUDA, SS_ERR_TIMEOUT, SS_ERR_BOUNDS = range(6)
SS_F32, SS_BF16 = 0, 1

EXPORTED = ("ss_scan_fwd", "ss_scan_workspace_bytes", "ss_status_string",
            "ss_last_device_error", "ss_debug_inject", "ss_scan_fwd_noalloc",
            "ss_scan_fwd_from_state", "ss_scan_step", "ss_scan_fwd_conv", "ss_scan_fwd_zoh",
            "ss_scan_bwd", "ss_scan_bwd_workspace_bytes", "ss_scan_fwd_train",
            "ss_debug_pointwise", "ss_debug_fwd_kernels")

# bytes of the library's static scratch array (SS_NOALLOC_SCRATCH_BYTES)
SS_NOALLOC_SCRATCH_BYTES = 4 << 20

# test hooks (include/ss_scan_debug.h)
(SS_DEBUG_CLEAR, SS_DEBUG_FORCE_WORKERS, SS_DEBUG_SKIP_PUBLISH, SS_DEBUG_SPIN_LIMIT,
 SS_DEBUG_STEP_SIMPLE, SS_DEBUG_FORCE_SEGMENTS) = range(6)
# pointwise functions ss_debug_pointwise evaluates (include/ss_scan_debug.h)
(SS_PW_SOFTPLUS, SS_PW_SILU, SS_PW_SOFTPLUS2, SS_PW_SILU2, SS_PW_EXP2_NEG_FMA, SS_PW_RCP_1_2,
 SS_PW_EX2) = range(7)


class SSError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {ss_status_string(status)}")


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libssscan.so once; raise if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build it with `python -m selective_state_space_ss_b200.build` "
                "(nvcc, sm_100a).  There is no CPU fallback.")
        lib = ctypes.CDLL(_LIB_PATH)
        vp, i64, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        lib.ss_scan_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ci, vp, vp,
                                    i64, i64, i64, ci, ci, vp, ctypes.c_size_t, vp]
        lib.ss_scan_fwd.restype = ci
        lib.ss_scan_workspace_bytes.argtypes = [i64, i64, i64, ci]
        lib.ss_scan_workspace_bytes.restype = ctypes.c_size_t
        lib.ss_status_string.argtypes = [ci]
        lib.ss_status_string.restype = ctypes.c_char_p
        lib.ss_last_device_error.argtypes = [vp]
        lib.ss_last_device_error.restype = ci
        lib.ss_debug_inject.argtypes = [ci, ctypes.c_longlong]
        lib.ss_debug_inject.restype = ci
        lib.ss_scan_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ci, vp, vp,
                                            i64, i64, i64, ci, ci, vp]
        lib.ss_scan_fwd_noalloc.restype = ci
        lib.ss_scan_fwd_from_state.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ci, vp, vp, vp,
                                               i64, i64, i64, ci, ci, vp, ctypes.c_size_t, vp]
        lib.ss_scan_fwd_from_state.restype = ci
        lib.ss_scan_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ci, vp, vp, i64, i64, ci, ci, vp]
        lib.ss_scan_fwd_conv.argtypes = [vp, vp, vp, ci, vp, vp, vp, vp, vp, vp, vp, ci, vp, vp,
                                         i64, i64, i64, ci, ci, vp, ctypes.c_size_t, vp]
        lib.ss_scan_fwd_conv.restype = ci
        lib.ss_scan_fwd_zoh.argtypes = lib.ss_scan_fwd.argtypes
        lib.ss_scan_fwd_zoh.restype = ci
        lib.ss_scan_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ci, vp, vp, vp, vp, vp, vp, vp,
                                    vp, vp, vp, vp, i64, i64, i64, ci, ci, vp, ctypes.c_size_t, vp]
        lib.ss_scan_fwd_train.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ci, vp, vp, vp,
                                          i64, i64, i64, ci, ci, vp, ctypes.c_size_t, vp]
        lib.ss_scan_fwd_train.restype = ci
        lib.ss_scan_bwd.restype = ci
        lib.ss_scan_bwd_workspace_bytes.argtypes = [i64, i64, i64, ci]
        lib.ss_scan_bwd_workspace_bytes.restype = ctypes.c_size_t
        lib.ss_scan_step.restype = ci
        lib.ss_debug_pointwise.argtypes = [ci, vp, vp, i64, vp]
        lib.ss_debug_pointwise.restype = ci
        lib.ss_debug_fwd_kernels.argtypes = [i64, i64, i64, ci, ci]
        lib.ss_debug_fwd_kernels.restype = ci
        _lib = lib
        return lib


def ss_status_string(status: int) -> str:
    return load_library().ss_status_string(int(status)).decode()


def ss_scan_workspace_bytes(batch: int, dim: int, seqlen: int, dstate: int) -> int:
    n = load_library().ss_scan_workspace_bytes(batch, dim, seqlen, dstate)
    if n == ctypes.c_size_t(-1).value:
        raise SSError(SS_ERR_INVALID_ARG, "ss_scan_workspace_bytes")
    return n


def _stream_handle(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def ss_last_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    return load_library().ss_last_device_error(_stream_handle(stream, None))


def ss_debug_inject(what: int, value: int = 0) -> None:
    """Test hook for the next ss_scan_fwd / ss_scan_step call (include/ss_scan_debug.h)."""
    st = load_library().ss_debug_inject(int(what), int(value))
    if st != SS_OK:
        raise SSError(st, "ss_debug_inject")


def ss_debug_fwd_kernels(batch: int, dim: int, seqlen: int, dstate: int, in_dtype: int) -> int:
    """Kernels one ss_scan_fwd call launches for this shape (include/ss_scan_debug.h)."""
    n = load_library().ss_debug_fwd_kernels(batch, dim, seqlen, dstate, int(in_dtype))
    if n < 1:
        raise SSError(SS_ERR_INVALID_ARG, "ss_debug_fwd_kernels")
    return n


def ss_debug_pointwise(fn: int, x, stream=None):
    """Evaluate one of the kernels' pointwise functions on a CUDA float32 tensor
    (test hook, include/ss_scan_debug.h); returns a new tensor."""
    if x.device.type != "cuda" or x.dtype != torch.float32:
        raise ValueError("x must be a float32 CUDA tensor")
    x = x.contiguous()
    y = torch.empty_like(x)
    st = load_library().ss_debug_pointwise(int(fn), x.data_ptr(), y.data_ptr(), x.numel(),
                                           _stream_handle(stream, x.device))
    if st != SS_OK:
        raise SSError(st, "ss_debug_pointwise")
    return y


def _ptr(t):
    return None if t is None else t.data_ptr()


def _check_dev(name, t, device, dtypes, shape=None):
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or t.device != device:
        raise ValueError(f"{name} must be a tensor on {device}")
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")


def _fwd_operands(u, delta, A, B, C, D, z, delta_bias):
    device = u.device
    if device.type != "cuda":
        raise ValueError("the scan runs on CUDA tensors only (no CPU fallback)")
    if u.dim() != 3 or B.dim() != 3:
        raise ValueError("u must be [batch, dim, L] and B [batch, N, L]")
    batch, dim, L = u.shape
    N = B.shape[1]
    in_types = (torch.float32, torch.bfloat16)
    for name, t in (("u", u), ("delta", delta), ("z", z)):
        _check_dev(name, t, device, in_types, (batch, dim, L))
    for name, t in (("B", B), ("C", C)):
        _check_dev(name, t, device, in_types, (batch, N, L))
    if len({t.dtype for t in (u, delta, B, C, z) if t is not None}) != 1:
        raise ValueError("u, delta, B, C and z must share one dtype")
    _check_dev("A", A, device, (torch.float32,), (dim, N))
    _check_dev("D", D, device, (torch.float32,), (dim,))
    _check_dev("delta_bias", delta_bias, device, (torch.float32,), (dim,))
    return device, batch, dim, L, N


def _fwd_call(name, initial_state, u, delta, A, B, C, D, z, delta_bias, softplus, y_out,
              last_state_out, return_last_state, workspace, stream):
    lib = load_library()
    device, batch, dim, L, N = _fwd_operands(u, delta, A, B, C, D, z, delta_bias)
    if y_out is None:
        y_out = torch.empty((batch, dim, L), dtype=torch.float32, device=device)
    _check_dev("y_out", y_out, device, (torch.float32,), (batch, dim, L))
    if last_state_out is None and return_last_state:
        last_state_out = torch.empty((batch, dim, N), dtype=torch.float32, device=device)
    _check_dev("last_state_out", last_state_out, device, (torch.float32,), (batch, dim, N))
    need = ss_scan_workspace_bytes(batch, dim, L, N)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    dt = SS_F32 if u.dtype == torch.float32 else SS_BF16
    head = (_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
            int(bool(softplus)))
    tail = (_ptr(y_out), _ptr(last_state_out), batch, dim, L, N, dt, _ptr(workspace), ws_bytes,
            _stream_handle(stream, device))
    if name == "ss_scan_fwd":
        st = lib.ss_scan_fwd(*head, *tail)
    elif name == "ss_scan_fwd_zoh":
        st = lib.ss_scan_fwd_zoh(*head, *tail)
    elif name == "ss_scan_fwd_train":
        ck = initial_state
        nk = (L + 15) // 16
        _check_dev("checkpoints", ck, device, (torch.float32,), (batch, nk, dim, N))
        st = lib.ss_scan_fwd_train(*head, tail[0], tail[1], _ptr(ck), *tail[2:])
    elif name == "ss_scan_fwd_conv":
        cw, cb = initial_state
        _check_dev("conv_weight", cw, device, (torch.float32,))
        _check_dev("conv_bias", cb, device, (torch.float32,), (dim,))
        if cw.dim() != 2 or cw.shape[0] != dim:
            raise ValueError("conv_weight must be [dim, W]")
        st = lib.ss_scan_fwd_conv(_ptr(u), _ptr(cw), _ptr(cb), cw.shape[1], _ptr(delta), _ptr(A),
                                  _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
                                  int(bool(softplus)), *tail)
    else:
        _check_dev("initial_state", initial_state, device, (torch.float32,), (batch, dim, N))
        st = lib.ss_scan_fwd_from_state(*head, _ptr(initial_state), *tail)
    if st != SS_OK:
        raise SSError(st, name)
    return y_out, last_state_out


def ss_scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                y_out=None, last_state_out=None, return_last_state=True,
                workspace=None, stream=None):
    """Fused selective-scan forward on the GPU.

    u, delta, z: [batch, dim, L]; B, C: [batch, N, L]; one dtype, float32 or
    bfloat16.  A: [dim, N] float32; D, delta_bias: [dim] float32 (optional).
    Returns (y [batch, dim, L] float32, last_state [batch, dim, N] float32 or
    None).  Output and workspace tensors are allocated with torch when not
    given; the library itself allocates nothing.
    """
    return _fwd_call("ss_scan_fwd", None, u, delta, A, B, C, D, z, delta_bias, softplus, y_out,
                     last_state_out, return_last_state, workspace, stream)


def ss_scan_fwd_from_state(initial_state, u, delta, A, B, C, D=None, z=None, delta_bias=None,
                           softplus=True, y_out=None, last_state_out=None,
                           return_last_state=True, workspace=None, stream=None):
    """ss_scan_fwd started from initial_state [batch, dim, N] float32 (None:
    zero).  last_state_out may be initial_state itself (in-place advance)."""
    return _fwd_call("ss_scan_fwd_from_state", initial_state, u, delta, A, B, C, D, z,
                     delta_bias, softplus, y_out, last_state_out, return_last_state, workspace,
                     stream)


def ss_scan_fwd_zoh(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                    y_out=None, last_state_out=None, return_last_state=True, workspace=None,
                    stream=None):
    """ss_scan_fwd with the exact zero-order-hold B_bar = (exp(Delta A) - 1) / A * B."""
    return _fwd_call("ss_scan_fwd_zoh", None, u, delta, A, B, C, D, z, delta_bias, softplus, y_out,
                     last_state_out, return_last_state, workspace, stream)


def ss_scan_fwd_conv(x, conv_weight, delta, A, B, C, D=None, z=None, delta_bias=None,
                     conv_bias=None, softplus=True, y_out=None, last_state_out=None,
                     return_last_state=True, workspace=None, stream=None):
    """ss_scan_fwd with u = SiLU(causal depthwise conv1d(x) + conv_bias) formed
    in the kernel.  x: [batch, dim, L] (float32 or bfloat16); conv_weight:
    [dim, W] float32 with W in 1..4 (tap W-1 meets the current token);
    conv_bias: [dim] float32 (optional)."""
    return _fwd_call("ss_scan_fwd_conv", (conv_weight, conv_bias), x, delta, A, B, C, D, z,
                     delta_bias, softplus, y_out, last_state_out, return_last_state, workspace,
                     stream)


def ss_scan_bwd_workspace_bytes(batch: int, dim: int, seqlen: int, dstate: int) -> int:
    n = load_library().ss_scan_bwd_workspace_bytes(batch, dim, seqlen, dstate)
    if n == ctypes.c_size_t(-1).value:
        raise SSError(SS_ERR_INVALID_ARG, "ss_scan_bwd_workspace_bytes")
    return n


def ss_scan_fwd_train(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                      y_out=None, last_state_out=None, checkpoints=None, return_last_state=True,
                      workspace=None, stream=None):
    """ss_scan_fwd that also writes the state at every 16-step chunk start.

    Returns (y, last_state, checkpoints); checkpoints [batch, ceil(L/16), dim,
    N] float32 (allocated with torch when not given) feed ss_scan_bwd.
    """
    batch, dim, L = u.shape
    N = B.shape[1]
    if checkpoints is None:
        checkpoints = torch.empty((batch, (L + 15) // 16, dim, N), dtype=torch.float32,
                                  device=u.device)
    y, h = _fwd_call("ss_scan_fwd_train", checkpoints, u, delta, A, B, C, D, z, delta_bias,
                     softplus, y_out, last_state_out, return_last_state, workspace, stream)
    return y, h, checkpoints


def ss_scan_bwd(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None, softplus=True,
                dlast_state=None, checkpoints=None, workspace=None, stream=None):
    """Gradients of ss_scan_fwd for an upstream dy [batch, dim, L] float32.

    Returns a dict of float32 tensors: du, ddelta, dz (None without z), dA
    [dim, N], dB, dC [batch, N, L], dD (None without D), ddelta_bias (None
    without delta_bias).  The states are recomputed, not stored; checkpoints
    from ss_scan_fwd_train (optional) spare the call its own forward pass.
    """
    lib = load_library()
    device, batch, dim, L, N = _fwd_operands(u, delta, A, B, C, D, z, delta_bias)
    _check_dev("dy", dy, device, (torch.float32,), (batch, dim, L))
    _check_dev("dlast_state", dlast_state, device, (torch.float32,), (batch, dim, N))
    f32 = dict(dtype=torch.float32, device=device)
    g = {"du": torch.empty((batch, dim, L), **f32), "ddelta": torch.empty((batch, dim, L), **f32),
         "dz": torch.empty((batch, dim, L), **f32) if z is not None else None,
         "dA": torch.empty((dim, N), **f32), "dB": torch.empty((batch, N, L), **f32),
         "dC": torch.empty((batch, N, L), **f32),
         "dD": torch.empty((dim,), **f32) if D is not None else None,
         "ddelta_bias": torch.empty((dim,), **f32) if delta_bias is not None else None}
    _check_dev("checkpoints", checkpoints, device, (torch.float32,), (batch, (L + 15) // 16, dim, N))
    if workspace is None and checkpoints is None:
        need = ss_scan_bwd_workspace_bytes(batch, dim, L, N)
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    dt = SS_F32 if u.dtype == torch.float32 else SS_BF16
    st = lib.ss_scan_bwd(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                         _ptr(delta_bias), int(bool(softplus)), _ptr(dy), _ptr(dlast_state),
                         _ptr(checkpoints), _ptr(g["du"]), _ptr(g["ddelta"]), _ptr(g["dA"]), _ptr(g["dB"]),
                         _ptr(g["dC"]), _ptr(g["dD"]), _ptr(g["dz"]), _ptr(g["ddelta_bias"]),
                         batch, dim, L, N, dt, _ptr(workspace), ws_bytes,
                         _stream_handle(stream, device))
    if st != SS_OK:
        raise SSError(st, "ss_scan_bwd")
    return g


def ss_scan_step(state, u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                 y_out=None, stream=None):
    """One recurrent (decode) step; advances state [batch, dim, N] float32 in place.

    u, delta, z: [batch, dim]; B, C: [batch, N]; float32 or bfloat16.
    Returns y [batch, dim] float32.
    """
    lib = load_library()
    device = state.device
    if device.type != "cuda":
        raise ValueError("ss_scan_step runs on CUDA tensors only (no CPU fallback)")
    if state.dim() != 3:
        raise ValueError("state must be [batch, dim, N]")
    batch, dim, N = state.shape
    _check_dev("state", state, device, (torch.float32,), (batch, dim, N))
    in_types = (torch.float32, torch.bfloat16)
    for name, t in (("u", u), ("delta", delta), ("z", z)):
        _check_dev(name, t, device, in_types, (batch, dim))
    for name, t in (("B", B), ("C", C)):
        _check_dev(name, t, device, in_types, (batch, N))
    if len({t.dtype for t in (u, delta, B, C, z) if t is not None}) != 1:
        raise ValueError("u, delta, B, C and z must share one dtype")
    _check_dev("A", A, device, (torch.float32,), (dim, N))
    _check_dev("D", D, device, (torch.float32,), (dim,))
    _check_dev("delta_bias", delta_bias, device, (torch.float32,), (dim,))
    if y_out is None:
        y_out = torch.empty((batch, dim), dtype=torch.float32, device=device)
    _check_dev("y_out", y_out, device, (torch.float32,), (batch, dim))
    dt = SS_F32 if u.dtype == torch.float32 else SS_BF16
    st = lib.ss_scan_step(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                          _ptr(delta_bias), int(bool(softplus)), _ptr(state), _ptr(y_out),
                          batch, dim, N, dt, _stream_handle(stream, device))
    if st != SS_OK:
        raise SSError(st, "ss_scan_step")
    return y_out


def ss_scan_fwd_noalloc(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                        y_out=None, last_state_out=None, stream=None):
    """ss_scan_fwd without a workspace: the library's static scratch array is used.

    For callers that cannot allocate device memory where they call the scan.
    The library allocates nothing; y_out and last_state_out must then be given
    (they are allocated with torch here only when missing).  Raises SSError
    with SS_ERR_UNSUPPORTED when the problem needs more scratch than
    SS_NOALLOC_SCRATCH_BYTES.  Overlapping calls on the GPU race on the array.
    """
    lib = load_library()
    device = u.device
    if device.type != "cuda":
        raise ValueError("ss_scan_fwd_noalloc runs on CUDA tensors only (no CPU fallback)")
    batch, dim, L = u.shape
    N = B.shape[1]
    in_types = (torch.float32, torch.bfloat16)
    for name, t in (("u", u), ("delta", delta), ("z", z)):
        _check_dev(name, t, device, in_types, (batch, dim, L))
    for name, t in (("B", B), ("C", C)):
        _check_dev(name, t, device, in_types, (batch, N, L))
    if len({t.dtype for t in (u, delta, B, C, z) if t is not None}) != 1:
        raise ValueError("u, delta, B, C and z must share one dtype")
    _check_dev("A", A, device, (torch.float32,), (dim, N))
    _check_dev("D", D, device, (torch.float32,), (dim,))
    _check_dev("delta_bias", delta_bias, device, (torch.float32,), (dim,))
    if y_out is None:
        y_out = torch.empty((batch, dim, L), dtype=torch.float32, device=device)
    _check_dev("y_out", y_out, device, (torch.float32,), (batch, dim, L))
    _check_dev("last_state_out", last_state_out, device, (torch.float32,), (batch, dim, N))
    dt = SS_F32 if u.dtype == torch.float32 else SS_BF16
    st = lib.ss_scan_fwd_noalloc(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                                 _ptr(delta_bias), int(bool(softplus)), _ptr(y_out),
                                 _ptr(last_state_out), batch, dim, L, N, dt,
                                 _stream_handle(stream, device))
    if st != SS_OK:
        raise SSError(st, "ss_scan_fwd_noalloc")
    return y_out, last_state_out
