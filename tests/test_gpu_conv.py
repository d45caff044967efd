"""GPU-vs-oracle parity for ss_scan_fwd_conv: the scan whose input is the
SiLU of the block's causal depthwise convolution, formed inside the kernel.

Tolerances as for the forward (fp32 1e-5, bf16 2e-3, relative to the largest
reference value; the final state likewise).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import selective_state_space_ss_b200 as ss  # noqa: E402
from selective_state_space_ss_b200 import inputs as I  # noqa: E402
from tests.helpers import TOL, rel_err, to_device  # noqa: E402


def _run(w, x, cw, cb, softplus=True, workspace=None, channels=None):
    xd = to_device(x)
    cwd = torch.from_numpy(cw).cuda()
    cbd = None if cb is None else torch.from_numpy(cb).cuda()
    y, h = ss.ss_scan_fwd_conv(xd["u"], cwd, xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                               z=xd["z"], delta_bias=xd["delta_bias"], conv_bias=cbd,
                               softplus=softplus, workspace=workspace)
    assert ss.ss_last_device_error() == ss.SS_OK
    yr, hr = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"],
                             x["delta_bias"], softplus=softplus, conv_weight=cw, conv_bias=cb,
                             channels=channels)
    y = y.cpu().numpy().reshape(-1, w.seqlen)
    h = h.cpu().numpy().reshape(-1, w.dstate)
    if channels is not None:
        y, h = y[channels], h[channels]
    tol = TOL[w.dtype]
    ey, eh = rel_err(y, yr.reshape(-1, w.seqlen)), rel_err(h, hr.reshape(-1, w.dstate))
    assert ey <= tol, f"{w.name}: y rel err {ey:.3e} > {tol}"
    assert eh <= tol, f"{w.name}: last_state rel err {eh:.3e} > {tol}"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [16, 32, 64, 128])
@pytest.mark.parametrize("L", [1, 3, 33, 1000, 2049])
def test_conv_small_shapes(dtype, N, L):
    # 3 x 37 channels: the time-split kernel for N <= 32, partial tiles, ragged
    # tails; odd L takes the element-wise loads
    w = I.Workload(f"conv_{dtype}_{N}_{L}", 3, 37, L, N, dtype)
    x = I.make_inputs(w, seed=L + N)
    cw, cb = I.make_conv(37, 4, seed=L)
    _run(w, x, cw, cb)


@pytest.mark.parametrize("width", [1, 2, 3, 4])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_conv_widths_channel_parallel(width, dtype):
    # enough channel groups for the channel-parallel kernel
    w = I.Workload(f"convw_{dtype}_{width}", 4, 1280, 256, 16, dtype)
    x = I.make_inputs(w, seed=width)
    cw, cb = I.make_conv(1280, width, seed=width + 10)
    _run(w, x, cw, cb)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_conv_without_bias_gate_skip(dtype):
    import dataclasses
    w = dataclasses.replace(I.Workload(f"convbare_{dtype}", 2, 300, 517, 32, dtype),
                            with_z=False, with_D=False)
    x = I.make_inputs(w, seed=3)
    cw, _ = I.make_conv(300, 4, seed=4)
    _run(w, x, cw, None)


@pytest.mark.parametrize("workers", [3, 7])
@pytest.mark.parametrize("N", [16, 64])
def test_conv_balanced_schedule(workers, N):
    # ranges that start inside a channel group: the halo of such a piece comes
    # from its own staged x rows, not from an earlier chunk
    w = I.Workload(f"convbal_{N}_{workers}", 5, 40, 1000, N, "bf16")
    x = I.make_inputs(w, seed=workers)
    cw, cb = I.make_conv(40, 4, seed=workers)
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, workers)
    need = ss.ss_scan_workspace_bytes(w.batch, w.dim, w.seqlen, w.dstate)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, workers)
    _run(w, x, cw, cb, workspace=ws)


def test_conv_full_workload_sampled():
    # the bench-sized workload with the convolution on, sampled channels
    w = I.WORKLOADS["b8_l2048_d1536_n16_bf16"]
    x = I.make_inputs(w, seed=77)
    cw, cb = I.make_conv(w.dim, 4, seed=78)
    ch = np.random.default_rng(0).choice(w.batch * w.dim, 256, replace=False)
    _run(w, x, cw, cb, channels=ch)


def test_conv_rejects_bad_width():
    w = I.Workload("convbad", 1, 8, 16, 16, "f32")
    x = to_device(I.make_inputs(w, seed=1))
    for width in (5, 8):
        cw = torch.zeros(8, width, device="cuda")
        with pytest.raises(ss.SSError):
            ss.ss_scan_fwd_conv(x["u"], cw, x["delta"], x["A"], x["B"], x["C"])
