"""ss_scan_fwd_noalloc: the scan for callers that cannot allocate device memory
where they call it (for example inside a framework that owns every device
allocation).  Its scratch is the library's static device array, so the test
checks it through the C ABI against ss_scan_fwd, whose workspace the caller
allocates, and against the fp64 oracle: same inputs, results within the
parity tolerance, on two calls in a row (the array keeps the previous call's
contents).  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import selective_state_space_ss_b200 as ss  # noqa: E402
from selective_state_space_ss_b200 import _native as N  # noqa: E402
from selective_state_space_ss_b200 import inputs as I  # noqa: E402
from tests.helpers import TOL, rel_err, to_device  # noqa: E402


def _noalloc_cabi(xd, y, h):
    """Call the C symbol directly with device pointers (no workspace argument)."""
    lib = N.load_library()
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    batch, dim, L = xd["u"].shape
    n = xd["B"].shape[1]
    dt = N.SS_F32 if xd["u"].dtype == torch.float32 else N.SS_BF16
    return lib.ss_scan_fwd_noalloc(p(xd["u"]), p(xd["delta"]), p(xd["A"]), p(xd["B"]), p(xd["C"]),
                                   p(xd["D"]), p(xd["z"]), p(xd["delta_bias"]), 1, p(y), p(h),
                                   batch, dim, L, n, dt, torch.cuda.current_stream().cuda_stream)


def _reference(xd):
    return ss.ss_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"], z=xd["z"],
                          delta_bias=xd["delta_bias"], softplus=True)


@pytest.mark.parametrize("shape,dtype,workers", [
    ((4, 5120, 256, 16), "bf16", 0),   # 640 channel groups: the balanced schedule, scratch in use
    ((3, 200, 777, 32), "bf16", 5),    # forced split of 7 groups: carries on a small problem
    ((2, 64, 301, 16), "f32", 3),      # element-wise load path (1204-byte rows) with a split
    ((2, 96, 200, 64), "bf16", 0),     # few channel groups: sequence segments, scratch in use
    ((1, 64, 70000, 16), "f32", 0),    # long segments with the carry-in correction
])
def test_noalloc_matches_workspace_entry_point(shape, dtype, workers):
    ss.ss_debug_inject(ss.SS_DEBUG_CLEAR)
    b, d, L, n = shape
    w = I.Workload("noalloc", b, d, L, n, dtype)
    x = I.make_inputs(w, seed=77)
    xd = to_device(x)
    yo, ho = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"],
                             x["delta_bias"])
    if workers:
        ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, workers)
    need = ss.ss_scan_workspace_bytes(b, d, L, n)
    assert need <= N.SS_NOALLOC_SCRATCH_BYTES
    if shape[1] == 5120 or shape[2] >= 200:
        assert need > 0  # this case really runs a kernel that uses scratch
    y_ref, h_ref = _reference(xd)
    torch.cuda.synchronize()
    assert ss.ss_last_device_error() == ss.SS_OK
    for call in range(2):  # two calls in a row share the static array
        if workers:
            ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, workers)
        y = torch.full_like(y_ref, float("nan"))
        h = torch.full_like(h_ref, float("nan"))
        assert _noalloc_cabi(xd, y, h) == N.SS_OK
        assert ss.ss_last_device_error() == ss.SS_OK
        assert rel_err(y.cpu().numpy(), y_ref.cpu().numpy()) <= TOL[dtype], f"call {call}"
        assert rel_err(h.cpu().numpy(), h_ref.cpu().numpy()) <= TOL[dtype], f"call {call}"
        assert rel_err(y.cpu().numpy(), yo) <= TOL[dtype], f"call {call} vs oracle"
        assert rel_err(h.cpu().numpy(), ho) <= TOL[dtype], f"call {call} vs oracle"


def test_noalloc_rejects_problems_beyond_its_scratch():
    ss.ss_debug_inject(ss.SS_DEBUG_CLEAR)
    # 640 channel groups at N = 64 shared by 600 CTAs: 600 carries of
    # 32 x 64 fp32 states (~4.9 MB) do not fit the static array
    b, d, L, n = 20, 1024, 64, 64
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, 600)
    try:
        assert ss.ss_scan_workspace_bytes(b, d, L, n) > N.SS_NOALLOC_SCRATCH_BYTES
        w = I.Workload("noalloc_big", b, d, L, n, "bf16")
        xd = to_device(I.make_inputs(w, seed=5))
        y = torch.zeros(b, d, L, device="cuda")
        h = torch.zeros(b, d, n, device="cuda")
        assert _noalloc_cabi(xd, y, h) == N.SS_ERR_UNSUPPORTED
        torch.cuda.synchronize()
        assert torch.count_nonzero(y).item() == 0  # nothing was launched
    finally:
        ss.ss_debug_inject(ss.SS_DEBUG_CLEAR)
