"""GPU-vs-oracle parity for ss_scan_fwd (through the C ABI).

Tolerances: fp32 inputs max|y - y_ref| <= 1e-5 max|y_ref|; bf16 inputs (fp32
state and accumulation) <= 2e-3 max|y_ref|; the final state under the same
relative rule against max|h_ref|.  Both sides read identical seeded inputs.
"""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
from selective_state_space_ss_b200 import inputs as I  # noqa: E402
from tests.helpers import TOL, rel_err, run_gpu, to_device  # noqa: E402


def _parity(w: I.Workload, seed=1, channels=None, softplus=None):
    x = I.make_inputs(w, seed=seed)
    sp = w.softplus if softplus is None else softplus
    xd = to_device(x)
    y, h = run_gpu(xd, softplus=sp)
    torch.cuda.synchronize()
    y = y.cpu().numpy().reshape(-1, w.seqlen)
    h = h.cpu().numpy().reshape(-1, w.dstate)
    yr, hr = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"],
                             x["delta_bias"], softplus=sp, channels=channels)
    yr = yr.reshape(-1, w.seqlen)
    hr = hr.reshape(-1, w.dstate)
    if channels is not None:
        y, h = y[channels], h[channels]
    tol = TOL[w.dtype]
    ey, eh = rel_err(y, yr), rel_err(h, hr)
    assert ey <= tol, f"{w.name}: y rel err {ey:.3e} > {tol}"
    assert eh <= tol, f"{w.name}: last_state rel err {eh:.3e} > {tol}"
    return ey, eh


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [16, 32, 64, 128])
@pytest.mark.parametrize("L", [1, 2, 7, 8, 33, 1000, 4097])
def test_small_shapes(dtype, N, L):
    # odd batch*dim, a partial channel tile, ragged tails, single-step sequences
    w = I.Workload(f"small_{dtype}_N{N}_L{L}", 3, 37, L, N, dtype)
    _parity(w, seed=L * 131 + N)


@pytest.mark.parametrize("variant", ["no_z", "no_D", "no_bias", "no_softplus", "bare"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_optional_inputs(variant, dtype):
    base = I.Workload("opt", 2, 70, 300, 16, dtype)
    kw = {"no_z": dict(with_z=False), "no_D": dict(with_D=False),
          "no_bias": dict(with_bias=False), "no_softplus": dict(softplus=False),
          "bare": dict(with_z=False, with_D=False, with_bias=False, softplus=False)}[variant]
    w = dataclasses.replace(base, name=f"opt_{variant}_{dtype}", **kw)
    if not w.softplus:
        # without the softplus Delta = delta + bias must stay positive and small
        x = I.make_inputs(w, seed=5)
        dl = np.abs(I.bf16_to_f32(x["delta"]) if dtype == "bf16" else x["delta"]) * 0.02 + 1e-3
        x["delta"] = (dl.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16) if dtype == "bf16" \
            else dl.astype(np.float32)
        if x["delta_bias"] is not None:
            x["delta_bias"] = np.full_like(x["delta_bias"], 1e-3)
        xd = to_device(x)
        y, h = run_gpu(xd, softplus=False)
        yr, hr = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"],
                                 x["delta_bias"], softplus=False)
        assert rel_err(y.cpu().numpy(), yr) <= TOL[dtype]
        assert rel_err(h.cpu().numpy(), hr) <= TOL[dtype]
    else:
        _parity(w, seed=5)


@pytest.mark.parametrize("name", ["b2_l1024_d512_n16_f32", "b8_l2048_d1536_n16_bf16"])
def test_full_config_all_channels(name):
    _parity(I.WORKLOADS[name], seed=1234)


@pytest.mark.parametrize("name", ["b4_l8192_d5120_n16_bf16", "b16_l4096_d2048_n16_bf16",
                                  "b16_l4096_d2048_n32_bf16", "b16_l4096_d2048_n64_bf16",
                                  "b16_l4096_d2048_n128_bf16"])
def test_full_config_sampled_channels(name):
    w = I.WORKLOADS[name]
    rng = np.random.default_rng(42)
    nch = w.batch * w.dim
    channels = np.unique(np.concatenate([[0, nch - 1, w.dim - 1, w.dim],
                                         rng.choice(nch, 60, replace=False)]))
    _parity(w, seed=1234, channels=channels)


def test_long_sequence_sampled_channels():
    w = I.WORKLOADS["b1_l1048576_d1536_n16_bf16"]
    rng = np.random.default_rng(43)
    channels = np.unique(np.concatenate([[0, 1535], rng.choice(w.dim, 14, replace=False)]))
    _parity(w, seed=1234, channels=channels)


def test_index_plumbing_distinct_values():
    """A[d,n] = -(1 + d + 100 n) 1e-3 and distinct D, bias: the final state and y must
    land at the right (b, d, n) with no tolerance beyond fp32 rounding."""
    w = I.Workload("plumb", 3, 45, 64, 16, "f32", with_z=False)
    x = I.make_inputs(w, seed=9)
    d_idx = np.arange(w.dim)[:, None]
    n_idx = np.arange(w.dstate)[None, :]
    x["A"] = (-(1 + d_idx + 100 * n_idx) * 1e-3).astype(np.float32)
    x["D"] = (10.0 + np.arange(w.dim)).astype(np.float32)
    x["delta_bias"] = (-3.0 + 0.01 * np.arange(w.dim)).astype(np.float32)
    xd = to_device(x)
    y, h = run_gpu(xd)
    yr, hr = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"])
    y, h = y.cpu().numpy(), h.cpu().numpy()
    # per-element relative check: any misplaced index is off by O(1)
    assert np.max(np.abs(h - hr) / (np.abs(hr) + 1e-3)) < 1e-4
    assert np.max(np.abs(y - yr) / (np.abs(yr) + 1e-2)) < 1e-4


def test_deterministic():
    w = I.Workload("det", 2, 100, 777, 32, "bf16")
    xd = to_device(I.make_inputs(w, seed=3))
    y1, h1 = run_gpu(xd)
    y2, h2 = run_gpu(xd)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(h1, h2)


def test_hold_and_reset_limits_on_gpu():
    """Delta -> 0 keeps the state bitwise; Delta -> large with A <= -1 resets it."""
    w = I.Workload("lim", 1, 40, 96, 16, "f32")
    x = I.make_inputs(w, seed=2)
    x["delta"][:, :, 48:] = -120.0  # e^(-120 + bias) underflows to 0 in fp32: Delta = 0, exact hold
    xd = to_device(x)
    y, h = run_gpu(xd)
    x48 = {k: (np.ascontiguousarray(v[:, :, :48]) if (v is not None and v.ndim == 3) else v)
           for k, v in x.items()}
    y48, h48 = run_gpu(to_device(x48))
    assert torch.equal(h, h48)
    x["delta"][:, :, :] = 60.0
    x["A"] = np.minimum(x["A"], -1.0).astype(np.float32)
    y, h = run_gpu(to_device(x))
    yr, hr = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"])
    assert rel_err(y.cpu().numpy(), yr) <= TOL["f32"]
    assert rel_err(h.cpu().numpy(), hr) <= TOL["f32"]


def test_unaligned_fallback_path():
    """Row starts off 16-byte boundaries (L odd, offset views) take the element-wise path."""
    w = I.Workload("unal", 2, 33, 129, 16, "bf16")
    x = I.make_inputs(w, seed=4)
    xd = to_device(x)
    # shift every activation tensor by one element inside a larger buffer
    for k in ("u", "delta", "z"):
        big = torch.empty(xd[k].numel() + 1, dtype=xd[k].dtype, device="cuda")
        big[1:].copy_(xd[k].reshape(-1))
        xd[k] = big[1:].view(xd[k].shape)
    y, h = run_gpu(xd)
    yr, hr = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"])
    assert rel_err(y.cpu().numpy(), yr) <= TOL["bf16"]
    assert rel_err(h.cpu().numpy(), hr) <= TOL["bf16"]


def test_device_error_word_clear():
    from selective_state_space_ss_b200 import SS_OK, ss_last_device_error

    w = I.Workload("err", 1, 8, 40, 16, "f32")
    run_gpu(to_device(I.make_inputs(w, seed=1)))
    assert ss_last_device_error() == SS_OK


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L", [7, 100, 1001, 2048])
def test_wide_shapes_channel_parallel_path(dtype, L):
    """Enough channel groups (5 x ceil(1000/32) = 160) to fill the SMs, so N = 16
    runs the channel-parallel kernel rather than the time split: partial last
    channel tile, ragged tails, odd L (element-wise loads)."""
    w = I.Workload(f"wide_{dtype}_L{L}", 5, 1000, L, 16, dtype)
    rng = np.random.default_rng(L)
    channels = np.unique(np.concatenate([[0, 999, 1000, 4999], rng.choice(5000, 300, replace=False)]))
    _parity(w, seed=L + 7, channels=channels)
