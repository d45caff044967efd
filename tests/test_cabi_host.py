"""C-ABI checks that need no GPU: the library loads, exports every function the
header declares, and rejects bad arguments on the host before any launch.

Every call below fails host-side validation, so no CUDA call is made; the
pointers are fake addresses that are never dereferenced.
"""
import ctypes
import os
import re

import pytest

from selective_state_space_ss_b200 import build as B
from selective_state_space_ss_b200 import _native as N

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return N.load_library()


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(ss_[a-z0-9_]+)\s*\(", text))
    return names


def test_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert {"ss_scan_fwd", "ss_scan_workspace_bytes", "ss_status_string", "ss_last_device_error"} <= declared
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert set(N.EXPORTED) <= declared


def test_debug_inject_rejects_unknown_code(lib):
    assert lib.ss_debug_inject(99, 0) == N.SS_ERR_INVALID_ARG
    assert lib.ss_debug_inject(N.SS_DEBUG_CLEAR, 0) == N.SS_OK


def test_status_strings(lib):
    for s in range(6):
        assert N.ss_status_string(s).startswith("SS_")
    assert "unknown" in N.ss_status_string(99)


def _call(lib, **over):
    a = dict(u=0x10000, delta=0x20000, A=0x30000, B=0x40000, C=0x50000, D=None, z=None,
             bias=None, sp=1, y=0x60000, h=None, batch=1, dim=1, L=8, N=16, dt=N.SS_F32,
             ws=None, wsb=0)
    a.update(over)
    return lib.ss_scan_fwd(a["u"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"], a["bias"],
                           a["sp"], a["y"], a["h"], a["batch"], a["dim"], a["L"], a["N"], a["dt"],
                           a["ws"], a["wsb"], None)


@pytest.mark.parametrize("field", ["u", "delta", "A", "B", "C", "y"])
def test_null_required_pointer(lib, field):
    assert _call(lib, **{field: None}) == N.SS_ERR_INVALID_ARG


@pytest.mark.parametrize("over", [dict(batch=0), dict(dim=0), dict(L=0), dict(batch=-1),
                                  dict(L=1 << 62, dim=1 << 10)])
def test_bad_sizes(lib, over):
    assert _call(lib, **over) == N.SS_ERR_INVALID_ARG


@pytest.mark.parametrize("n", [0, 1, 8, 17, 24, 256])
def test_unsupported_dstate(lib, n):
    assert _call(lib, N=n) == N.SS_ERR_UNSUPPORTED


def test_unsupported_dtype(lib):
    assert _call(lib, dt=7) == N.SS_ERR_UNSUPPORTED


@pytest.mark.parametrize("field,addr,dt", [("u", 0x10002, N.SS_F32), ("B", 0x40001, N.SS_BF16),
                                           ("A", 0x30002, N.SS_F32), ("y", 0x60002, N.SS_BF16)])
def test_misaligned(lib, field, addr, dt):
    assert _call(lib, **{field: addr, "dt": dt}) == N.SS_ERR_INVALID_ARG


def _call_state(lib, **over):
    a = dict(u=0x10000, delta=0x20000, A=0x30000, B=0x40000, C=0x50000, D=None, z=None,
             bias=None, sp=1, h0=0x70000, y=0x60000, h=None, batch=1, dim=1, L=8, N=16,
             dt=N.SS_F32, ws=None, wsb=0)
    a.update(over)
    return lib.ss_scan_fwd_from_state(a["u"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"],
                                      a["bias"], a["sp"], a["h0"], a["y"], a["h"], a["batch"],
                                      a["dim"], a["L"], a["N"], a["dt"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("over,status", [
    (dict(u=None), N.SS_ERR_INVALID_ARG), (dict(y=None), N.SS_ERR_INVALID_ARG),
    (dict(h0=0x70002), N.SS_ERR_INVALID_ARG), (dict(L=0), N.SS_ERR_INVALID_ARG),
    (dict(N=24), N.SS_ERR_UNSUPPORTED), (dict(dt=5), N.SS_ERR_UNSUPPORTED)])
def test_from_state_rejections(lib, over, status):
    assert _call_state(lib, **over) == status


def _call_step(lib, **over):
    a = dict(u=0x10000, delta=0x20000, A=0x30000, B=0x40000, C=0x50000, D=None, z=None,
             bias=None, sp=1, state=0x70000, y=0x60000, batch=1, dim=1, N=16, dt=N.SS_F32)
    a.update(over)
    return lib.ss_scan_step(a["u"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"], a["bias"],
                            a["sp"], a["state"], a["y"], a["batch"], a["dim"], a["N"], a["dt"], None)


@pytest.mark.parametrize("field", ["u", "delta", "A", "B", "C", "state", "y"])
def test_step_null_required_pointer(lib, field):
    assert _call_step(lib, **{field: None}) == N.SS_ERR_INVALID_ARG


@pytest.mark.parametrize("over,status", [
    (dict(batch=0), N.SS_ERR_INVALID_ARG), (dict(dim=-3), N.SS_ERR_INVALID_ARG),
    (dict(batch=1 << 40, dim=1 << 20), N.SS_ERR_INVALID_ARG),
    (dict(dim=1 << 28), N.SS_ERR_INVALID_ARG),
    (dict(N=8), N.SS_ERR_UNSUPPORTED), (dict(N=256), N.SS_ERR_UNSUPPORTED),
    (dict(dt=2), N.SS_ERR_UNSUPPORTED), (dict(state=0x70002), N.SS_ERR_INVALID_ARG),
    (dict(u=0x10001, dt=N.SS_BF16), N.SS_ERR_INVALID_ARG), (dict(D=0x80002), N.SS_ERR_INVALID_ARG)])
def test_step_rejections(lib, over, status):
    assert _call_step(lib, **over) == status


def _call_conv(lib, **over):
    a = dict(x=0x10000, cw=0x90000, cb=None, W=4, delta=0x20000, A=0x30000, B=0x40000,
             C=0x50000, D=None, z=None, bias=None, sp=1, y=0x60000, h=None, batch=1, dim=1, L=8,
             N=16, dt=N.SS_F32, ws=None, wsb=0)
    a.update(over)
    return lib.ss_scan_fwd_conv(a["x"], a["cw"], a["cb"], a["W"], a["delta"], a["A"], a["B"],
                                a["C"], a["D"], a["z"], a["bias"], a["sp"], a["y"], a["h"],
                                a["batch"], a["dim"], a["L"], a["N"], a["dt"], a["ws"], a["wsb"],
                                None)


@pytest.mark.parametrize("over,status", [
    (dict(cw=None), N.SS_ERR_INVALID_ARG), (dict(x=None), N.SS_ERR_INVALID_ARG),
    (dict(W=0), N.SS_ERR_UNSUPPORTED), (dict(W=5), N.SS_ERR_UNSUPPORTED),
    (dict(cw=0x90002), N.SS_ERR_INVALID_ARG), (dict(cb=0x90006), N.SS_ERR_INVALID_ARG),
    (dict(N=48), N.SS_ERR_UNSUPPORTED)])
def test_conv_rejections(lib, over, status):
    assert _call_conv(lib, **over) == status


@pytest.mark.parametrize("over", [dict(u=None), dict(N=8), dict(L=0), dict(y=0x60002)])
def test_zoh_rejections(lib, over):
    a = dict(u=0x10000, delta=0x20000, A=0x30000, B=0x40000, C=0x50000, D=None, z=None,
             bias=None, sp=1, y=0x60000, h=None, batch=1, dim=1, L=8, N=16, dt=N.SS_F32,
             ws=None, wsb=0)
    a.update(over)
    st = lib.ss_scan_fwd_zoh(a["u"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"], a["bias"],
                             a["sp"], a["y"], a["h"], a["batch"], a["dim"], a["L"], a["N"], a["dt"],
                             a["ws"], a["wsb"], None)
    assert st in (N.SS_ERR_INVALID_ARG, N.SS_ERR_UNSUPPORTED)


def _call_bwd(lib, **over):
    a = dict(u=0x10000, delta=0x20000, A=0x30000, B=0x40000, C=0x50000, D=None, z=None,
             bias=None, sp=1, dy=0x60000, dl=None, ck=None, du=0x70000, dd=0x80000, dA=0x90000,
             dB=0xa0000, dC=0xb0000, dD=None, dz=None, db=None, batch=1, dim=1, L=8, N=16,
             dt=N.SS_F32, ws=0x100000, wsb=1 << 20)
    a.update(over)
    return lib.ss_scan_bwd(a["u"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"], a["bias"],
                           a["sp"], a["dy"], a["dl"], a["ck"], a["du"], a["dd"], a["dA"], a["dB"], a["dC"],
                           a["dD"], a["dz"], a["db"], a["batch"], a["dim"], a["L"], a["N"], a["dt"],
                           a["ws"], a["wsb"], None)


@pytest.mark.parametrize("over,status", [
    (dict(dy=None), N.SS_ERR_INVALID_ARG), (dict(du=None), N.SS_ERR_INVALID_ARG),
    (dict(dB=None), N.SS_ERR_INVALID_ARG), (dict(z=0x110000), N.SS_ERR_INVALID_ARG),
    (dict(ws=None), N.SS_ERR_INVALID_ARG), (dict(ws=0x100010), N.SS_ERR_INVALID_ARG),
    (dict(N=12), N.SS_ERR_UNSUPPORTED), (dict(dt=3), N.SS_ERR_UNSUPPORTED),
    (dict(L=0), N.SS_ERR_INVALID_ARG), (dict(dA=0x90002), N.SS_ERR_INVALID_ARG),
    (dict(ck=0x120008), N.SS_ERR_INVALID_ARG)])
def test_bwd_rejections(lib, over, status):
    assert _call_bwd(lib, **over) == status


@pytest.mark.parametrize("ck", [None, 0x70008])
def test_fwd_train_rejects_bad_checkpoints(lib, ck):
    assert lib.ss_scan_fwd_train(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, None, None, None, 1,
                                 0x60000, None, ck, 1, 1, 8, 16, N.SS_F32, None, 0,
                                 None) == N.SS_ERR_INVALID_ARG


def test_bwd_workspace_query(lib):
    assert lib.ss_scan_bwd_workspace_bytes(0, 1, 1, 16) == ctypes.c_size_t(-1).value
    assert lib.ss_scan_bwd_workspace_bytes(1, 1, 1, 24) == ctypes.c_size_t(-1).value
    # the checkpoint array: 4 bytes x batch x ceil(L/16) x dim x dstate, 256-aligned
    n = lib.ss_scan_bwd_workspace_bytes(8, 1536, 2048, 16)
    assert n == 8 * 128 * 1536 * 16 * 4
    assert lib.ss_scan_bwd_workspace_bytes(1, 3, 17, 16) == 512  # 2 chunks x 3 x 16 x 4 = 384


def test_workspace_query_rejects_bad_sizes(lib):
    # (valid sizes need the device's SM count, so they are covered by the GPU tests)
    with pytest.raises(N.SSError):
        N.ss_scan_workspace_bytes(8, 1536, 2048, 17)
    assert lib.ss_scan_workspace_bytes(0, 1, 1, 16) == ctypes.c_size_t(-1).value
    assert lib.ss_scan_workspace_bytes(1, 1, 0, 16) == ctypes.c_size_t(-1).value


def test_binding_refuses_cpu_tensors():
    import torch

    x = torch.zeros(1, 2, 8)
    with pytest.raises(ValueError):
        N.ss_scan_fwd(x, x, torch.zeros(2, 16), torch.zeros(1, 16, 8), torch.zeros(1, 16, 8))
    with pytest.raises(ValueError):
        N.ss_scan_fwd_from_state(torch.zeros(1, 2, 16), x, x, torch.zeros(2, 16),
                                 torch.zeros(1, 16, 8), torch.zeros(1, 16, 8))
    t = torch.zeros(1, 2)
    with pytest.raises(ValueError):
        N.ss_scan_step(torch.zeros(1, 2, 16), t, t, torch.zeros(2, 16), torch.zeros(1, 16),
                       torch.zeros(1, 16))
    B = torch.zeros(1, 16, 8)
    with pytest.raises(ValueError):
        N.ss_scan_fwd_zoh(x, x, torch.zeros(2, 16), B, B)
    with pytest.raises(ValueError):
        N.ss_scan_fwd_conv(x, torch.zeros(2, 4), x, torch.zeros(2, 16), B, B)
    with pytest.raises(ValueError):
        N.ss_scan_fwd_train(x, x, torch.zeros(2, 16), B, B)
    with pytest.raises(ValueError):
        N.ss_scan_bwd(x, x, torch.zeros(2, 16), B, B, torch.zeros(1, 2, 8))


def test_built_libraries_match_their_sources(lib):
    # each library records the hash of the sources (and -D flags) it was built
    # from; a build is redone exactly when that hash changes
    assert B.source_hash() == B.source_hash()
    assert B.source_hash() != B.source_hash(["SS_BOUNDS_CHECK"])
    assert not B.stale(), "libssscan.so is older than its sources"
    with open(B.LIB + ".src") as f:
        assert f.read().strip() == B.source_hash()
