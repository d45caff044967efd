"""GPU-vs-oracle parity for sequences cut into segments (through the C ABI).

With fewer channel groups than resident CTA slots, ss_scan_fwd scans segments
of each sequence at once, each from a zero state, and a second kernel adds the
carry-in sum_n C_t[n] prod(A_bar)[n] h_in[n] ("Mamba 选择性机制", sec. 3.1:
the recurrence composes with the associative operator).  These tests force the
segment count on problems the oracle checks in full, and cover what the
correction must get right: the carried state through many segments, no decay
(A = 0: the term is never dropped), Delta of either sign (softplus off), an
initial state (only segment 0 starts from it, and it may alias the final state),
the fused convolution and the exact zero-order hold, ragged last segments, and
the plain unsegmented path on the same small shapes.

Tolerances as for the forward: max|x - x_ref| <= 1e-5 (fp32 inputs) or 2e-3
(bf16 inputs) times max|x_ref|, for y and the final state.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import selective_state_space_ss_b200 as ss  # noqa: E402
from selective_state_space_ss_b200 import inputs as I  # noqa: E402
from tests.helpers import TOL, rel_err, to_device  # noqa: E402


def _fwd(xd, segments, softplus=True, h0=None, **kw):
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_SEGMENTS, segments)
    args = (xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"])
    opt = dict(D=xd["D"], z=xd["z"], delta_bias=xd["delta_bias"], softplus=softplus, **kw)
    if h0 is not None:
        y, h = ss.ss_scan_fwd_from_state(h0, *args, **opt)
    else:
        y, h = ss.ss_scan_fwd(*args, **opt)
    torch.cuda.synchronize()
    assert ss.ss_last_device_error() == ss.SS_OK
    return y.cpu().numpy(), h.cpu().numpy()


def _ref(x, softplus=True, h0=None):
    return oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"],
                           x["delta_bias"], softplus=softplus, h0=h0)


def _check(w, y, h, yr, hr):
    tol = TOL[w.dtype]
    ey, eh = rel_err(y, yr), rel_err(h, hr)
    assert ey <= tol, f"{w.name}: y rel err {ey:.3e} > {tol}"
    assert eh <= tol, f"{w.name}: last_state rel err {eh:.3e} > {tol}"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [16, 32, 64, 128])
@pytest.mark.parametrize("segments", [1, 2, 3, 7, 40])
def test_forced_segments(dtype, N, segments):
    # L = 1234: 39 chunks of 32 steps, so 40 requested segments become 39 of
    # one chunk, and 7 become 7 with a short last one
    w = I.Workload(f"seg_{dtype}_N{N}_S{segments}", 2, 45, 1234, N, dtype)
    x = I.make_inputs(w, seed=N + segments)
    y, h = _fwd(to_device(x), segments)
    _check(w, y, h, *_ref(x))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L", [1, 31, 33, 95, 4097])
def test_segments_ragged_lengths(dtype, L):
    w = I.Workload(f"segL_{dtype}_{L}", 1, 70, L, 16, dtype)
    x = I.make_inputs(w, seed=L)
    y, h = _fwd(to_device(x), 5)
    _check(w, y, h, *_ref(x))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_segments_without_decay(dtype):
    # A = 0 for half the states: their carry-in weight stays 1 over the whole
    # segment, so the correction may never drop them
    w = I.Workload(f"segA0_{dtype}", 1, 40, 3000, 16, dtype)
    x = I.make_inputs(w, seed=3)
    x["A"][:, ::2] = 0.0
    y, h = _fwd(to_device(x), 6)
    _check(w, y, h, *_ref(x))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_segments_softplus_off(dtype):
    # Delta = delta + bias of either sign: the weights do not fall monotonically
    w = I.Workload(f"segsp_{dtype}", 1, 40, 2000, 16, dtype)
    x = I.make_inputs(w, seed=4)
    dl = I.bf16_to_f32(x["delta"]) if dtype == "bf16" else x["delta"]
    dl = (dl * 0.01).astype(np.float32)
    x["delta"] = (dl.view(np.uint32) >> 16).astype(np.uint16) if dtype == "bf16" else dl
    x["delta_bias"] = np.full_like(x["delta_bias"], 2e-3)
    y, h = _fwd(to_device(x), 5, softplus=False)
    _check(w, y, h, *_ref(x, softplus=False))


def test_segments_long_memory():
    # dt in [1e-4, 1e-2] as in the million-step workload: most carry-in terms
    # live for thousands of steps, across several segments
    w = I.Workload("seglong", 1, 64, 65536, 16, "bf16", dt_min=1e-4, dt_max=1e-2)
    x = I.make_inputs(w, seed=8)
    y, h = _fwd(to_device(x), 16)
    _check(w, y, h, *_ref(x))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("alias", [False, True])
def test_segments_from_state(dtype, alias):
    # only segment 0 starts from h0; with alias the final state overwrites h0
    w = I.Workload(f"segh0_{dtype}_{alias}", 2, 33, 1500, 32, dtype)
    x = I.make_inputs(w, seed=11)
    h0 = I.make_state(2, 33, 32, seed=12)
    h0d = torch.from_numpy(h0).cuda()
    kw = dict(last_state_out=h0d) if alias else {}
    y, h = _fwd(to_device(x), 4, h0=h0d, **kw)
    _check(w, y, h, *_ref(x, h0=h0))
    if alias:
        np.testing.assert_array_equal(h, h0d.cpu().numpy())


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_segments_conv(dtype):
    w = I.Workload(f"segconv_{dtype}", 1, 50, 1000, 16, dtype)
    x = I.make_inputs(w, seed=13)
    cw, cb = I.make_conv(w.dim, 4, seed=14)
    xd = to_device(x)
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_SEGMENTS, 6)
    y, h = ss.ss_scan_fwd_conv(xd["u"], torch.from_numpy(cw).cuda(), xd["delta"], xd["A"], xd["B"],
                               xd["C"], D=xd["D"], z=xd["z"], delta_bias=xd["delta_bias"],
                               conv_bias=torch.from_numpy(cb).cuda())
    yr, hr = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"],
                             x["delta_bias"], conv_weight=cw, conv_bias=cb)
    _check(w, y.cpu().numpy(), h.cpu().numpy(), yr, hr)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_segments_zoh(dtype):
    w = I.Workload(f"segzoh_{dtype}", 1, 50, 1000, 16, dtype)
    x = I.make_inputs(w, seed=15)
    xd = to_device(x)
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_SEGMENTS, 6)
    y, h = ss.ss_scan_fwd_zoh(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"], z=xd["z"],
                              delta_bias=xd["delta_bias"])
    yr, hr = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"],
                             x["delta_bias"], zoh=True)
    _check(w, y.cpu().numpy(), h.cpu().numpy(), yr, hr)


def test_training_forward_is_never_segmented():
    # the checkpoints must hold true states: a segment request is ignored
    w = I.Workload("segtrain", 1, 40, 700, 16, "f32")
    x = I.make_inputs(w, seed=16)
    xd = to_device(x)
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_SEGMENTS, 5)
    y, h, ck = ss.ss_scan_fwd_train(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                                    z=xd["z"], delta_bias=xd["delta_bias"])
    ss.ss_debug_inject(ss.SS_DEBUG_CLEAR)
    _check(w, y.cpu().numpy(), h.cpu().numpy(), *_ref(x))
    # checkpoint k is the state before step 16 k: the final state of a scan over 16 k steps
    for k in (1, 20, 43):
        xs = {kk: (np.ascontiguousarray(v[:, :, :16 * k]) if (v is not None and v.ndim == 3) else v)
              for kk, v in x.items()}
        _, hk = _ref(xs)
        assert rel_err(ck[:, k].cpu().numpy(), hk) <= TOL["f32"]


def test_auto_segments_on_few_channels():
    # one batch row of 64 channels over 70000 steps: the default plan segments
    # the sequence (shorter ones take the time split)
    w = I.Workload("segauto", 1, 64, 70000, 16, "bf16", dt_min=1e-4, dt_max=1e-2)
    x = I.make_inputs(w, seed=17)
    y, h = _fwd(to_device(x), 0)
    _check(w, y, h, *_ref(x))


def test_kernels_per_call():
    # the million-token shape is cut into segments (scan + correction); the
    # B8 L2048 D1536 shape fills the GPU with channel groups (one kernel)
    assert ss.ss_debug_fwd_kernels(1, 1536, 1 << 20, 16, ss.SS_BF16) == 2
    assert ss.ss_debug_fwd_kernels(8, 1536, 2048, 16, ss.SS_BF16) == 1
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_SEGMENTS, 4)
    assert ss.ss_debug_fwd_kernels(1, 64, 4096, 16, ss.SS_F32) == 2
    ss.ss_debug_inject(ss.SS_DEBUG_CLEAR)
    with pytest.raises(ss.SSError):
        ss.ss_debug_fwd_kernels(1, 64, 4096, 24, ss.SS_F32)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("drop", ["z", "D", "bias"])
def test_segments_optional_inputs(dtype, drop):
    # the correction gates by SiLU(z) only when z is given, and reads no D or bias
    w = I.Workload(f"segopt_{dtype}_{drop}", 1, 70, 3000, 16, dtype)
    x = I.make_inputs(w, seed=31)
    key = {"z": "z", "D": "D", "bias": "delta_bias"}[drop]
    x[key] = None
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_SEGMENTS, 5)
    xd = to_device(x)
    y, h = ss.ss_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"], z=xd["z"],
                          delta_bias=xd["delta_bias"])
    torch.cuda.synchronize()
    assert ss.ss_last_device_error() == ss.SS_OK
    yr, hr = _ref(x)
    _check(w, y.cpu().numpy(), h.cpu().numpy(), yr, hr)
