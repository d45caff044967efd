"""GPU-vs-oracle parity for ss_scan_fwd_zoh: the exact zero-order-hold input
matrix B_bar = (exp(Delta A) - 1) / A * B.

Tolerances as for the forward (fp32 1e-5, bf16 2e-3, relative to the largest
reference value; the final state likewise).  Both branches of the kernel's
(exp(x) - 1)/x are covered: small |Delta A| (series), large (quotient), the
boundary between them, and A = 0.
"""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import selective_state_space_ss_b200 as ss  # noqa: E402
from selective_state_space_ss_b200 import inputs as I  # noqa: E402
from tests.helpers import TOL, rel_err, to_device  # noqa: E402


def _run(w, x, softplus=True, workspace=None, channels=None):
    xd = to_device(x)
    y, h = ss.ss_scan_fwd_zoh(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"], z=xd["z"],
                              delta_bias=xd["delta_bias"], softplus=softplus, workspace=workspace)
    assert ss.ss_last_device_error() == ss.SS_OK
    yr, hr = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"],
                             x["delta_bias"], softplus=softplus, zoh=True, channels=channels)
    y = y.cpu().numpy().reshape(-1, w.seqlen)
    h = h.cpu().numpy().reshape(-1, w.dstate)
    if channels is not None:
        y, h = y[channels], h[channels]
    tol = TOL[w.dtype]
    ey, eh = rel_err(y, yr.reshape(-1, w.seqlen)), rel_err(h, hr.reshape(-1, w.dstate))
    assert ey <= tol, f"{w.name}: y rel err {ey:.3e} > {tol}"
    assert eh <= tol, f"{w.name}: last_state rel err {eh:.3e} > {tol}"
    return y


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [16, 32, 64, 128])
@pytest.mark.parametrize("L", [1, 7, 300, 2049])
def test_zoh_small_shapes(dtype, N, L):
    w = I.Workload(f"zoh_{dtype}_{N}_{L}", 3, 37, L, N, dtype)
    _run(w, I.make_inputs(w, seed=L * 3 + N))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dt_range", [(1e-4, 1e-2), (1e-3, 1e-1), (0.05, 2.0)])
def test_zoh_delta_regimes_channel_parallel(dtype, dt_range):
    # small Delta A: the series branch; large: the quotient branch; the middle
    # range crosses the boundary between them
    w = I.Workload(f"zohr_{dtype}_{dt_range[0]}", 4, 1280, 300, 16, dtype, dt_min=dt_range[0],
                   dt_max=dt_range[1])
    _run(w, I.make_inputs(w, seed=11))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_zoh_a_zero_states(dtype):
    # A = 0 on some states: B_bar = Delta B there, no division by zero
    w = I.Workload(f"zoh0_{dtype}", 2, 200, 400, 32, dtype)
    x = I.make_inputs(w, seed=13)
    x["A"][:, ::5] = 0.0
    _run(w, x)


def test_zoh_boundary_of_the_series():
    # Delta A x log2(e) swept through the series/quotient switch: Delta fixed
    # per channel, softplus off, A chosen so |x2| covers 0.2 .. 0.3
    w = dataclasses.replace(I.Workload("zohb", 1, 512, 256, 16, "f32"), with_bias=False,
                            softplus=False)
    x = I.make_inputs(w, seed=17)
    x["delta"] = np.full((1, 512, 256), 0.1, np.float32)
    x2 = np.linspace(-0.3, -0.2, 512 * 16).reshape(512, 16)
    x["A"] = (x2 / 0.1 / np.log2(np.e)).astype(np.float32)
    _run(w, x, softplus=False)


@pytest.mark.parametrize("workers", [3, 7])
def test_zoh_balanced_schedule(workers):
    w = I.Workload(f"zohbal_{workers}", 5, 40, 1000, 64, "bf16")
    x = I.make_inputs(w, seed=workers)
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, workers)
    need = ss.ss_scan_workspace_bytes(w.batch, w.dim, w.seqlen, w.dstate)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, workers)
    _run(w, x, workspace=ws)


def test_zoh_full_workload_sampled():
    w = I.WORKLOADS["b8_l2048_d1536_n16_bf16"]
    x = I.make_inputs(w, seed=79)
    ch = np.random.default_rng(1).choice(w.batch * w.dim, 256, replace=False)
    _run(w, x, channels=ch)
