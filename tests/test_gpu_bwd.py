"""GPU-vs-oracle parity for ss_scan_bwd (gradients with recomputation).

Every gradient is compared with the fp64 oracle's reverse-mode sweep
element by element, relative to its largest reference value.  Tolerance:
TOL_BWD (see the design notes: fp32 recomputation of the states, fp32
adjoint, and atomically ordered sums over channels, steps and batch rows).
"""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import selective_state_space_ss_b200 as ss  # noqa: E402
from selective_state_space_ss_b200 import inputs as I  # noqa: E402
from tests.helpers import rel_err, to_device  # noqa: E402

TOL_BWD = {"f32": 1e-4, "bf16": 1e-4}
NAMES = ("du", "ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias")


def _dy(w, seed):
    return I.fill(seed, 12, (w.batch, w.dim, w.seqlen))


def _run(w, x, dy, dlast=None, softplus=True, ckpt=False):
    xd = to_device(x)
    checkpoints = None
    if ckpt:  # the training forward writes the checkpoints the backward starts from
        _, _, checkpoints = ss.ss_scan_fwd_train(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"],
                                                 D=xd["D"], z=xd["z"], delta_bias=xd["delta_bias"],
                                                 softplus=softplus)
    g = ss.ss_scan_bwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], torch.from_numpy(dy).cuda(),
                       D=xd["D"], z=xd["z"], delta_bias=xd["delta_bias"], softplus=softplus,
                       dlast_state=None if dlast is None else torch.from_numpy(dlast).cuda(),
                       checkpoints=checkpoints)
    assert ss.ss_last_device_error() == ss.SS_OK
    r = oracle.scan_bwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"],
                        softplus=softplus, dy=dy.astype(np.float64),
                        dlast=None if dlast is None else dlast.astype(np.float64))
    errs = {}
    for k in NAMES:
        if g[k] is None or r[k] is None:
            assert (g[k] is None) == (r[k] is None or (k == "dD" and x["D"] is None)
                                      or (k == "ddelta_bias" and x["delta_bias"] is None)), k
            continue
        errs[k] = rel_err(g[k].cpu().numpy(), r[k])
    bad = {k: v for k, v in errs.items() if v > TOL_BWD[w.dtype]}
    assert not bad, f"{w.name}: {bad} (all: {errs})"
    return errs


@pytest.mark.parametrize("ckpt", [False, True])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [16, 32, 64, 128])
@pytest.mark.parametrize("L", [1, 15, 16, 17, 300])
def test_bwd_small_shapes(dtype, N, L, ckpt):
    # 2 x 37 channels: the forward's time-split kernel writes the checkpoints
    # for N <= 32, the channel-parallel one for N >= 64
    w = I.Workload(f"bwd_{dtype}_{N}_{L}", 2, 37, L, N, dtype)
    x = I.make_inputs(w, seed=L + N)
    _run(w, x, _dy(w, L), ckpt=ckpt)


@pytest.mark.parametrize("workers", [0, 3])
@pytest.mark.parametrize("N", [16, 64])
def test_bwd_checkpoints_from_wide_forward(workers, N):
    # enough channel groups for the channel-parallel forward (and, forced, its
    # balanced schedule) to write the checkpoints
    w = I.Workload(f"bwdck_{N}_{workers}", 4, 1280, 200, N, "bf16")
    x = I.make_inputs(w, seed=workers + N)
    if workers:
        ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, workers)
    _run(w, x, _dy(w, 3), ckpt=True)


@pytest.mark.parametrize("N,batch,dim", [(16, 2, 37), (16, 4, 1280), (128, 2, 40)])
def test_fwd_train_checkpoints_are_states(N, batch, dim):
    # checkpoint k holds the state before step 16 k: the oracle's final state of
    # the first 16 k steps; y is that of the plain forward
    L = 150
    w = I.Workload("ckstates", batch, dim, L, N, "f32")
    x = I.make_inputs(w, seed=N + dim)
    xd = to_device(x)
    y, h, ck = ss.ss_scan_fwd_train(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                                    z=xd["z"], delta_bias=xd["delta_bias"])
    # the training forward (never segmented, one channel per lane) agrees with
    # the plain forward to fp32 rounding
    y0, h0 = ss.ss_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"], z=xd["z"],
                            delta_bias=xd["delta_bias"])
    torch.cuda.synchronize()
    assert rel_err(y.cpu().numpy(), y0.cpu().numpy()) <= 1e-6
    assert rel_err(h.cpu().numpy(), h0.cpu().numpy()) <= 1e-6
    ck = ck.cpu().numpy()
    assert ck.shape == (batch, 10, dim, N)
    assert np.all(ck[:, 0] == 0.0)
    for k in (1, 4, 9):
        cut = {kk: (np.ascontiguousarray(v[:, :, :16 * k]) if kk in ("u", "delta", "z", "B", "C") else v)
               for kk, v in x.items()}
        _, hr = oracle.scan_fwd(cut["u"], cut["delta"], cut["A"], cut["B"], cut["C"], cut["D"],
                                cut["z"], cut["delta_bias"])
        assert rel_err(ck[:, k], hr) <= 1e-5


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bwd_with_final_state_gradient(dtype):
    w = I.Workload(f"bwdlast_{dtype}", 3, 50, 200, 16, dtype)
    x = I.make_inputs(w, seed=5)
    dlast = I.fill(6, 13, (3, 50, 16))
    _run(w, x, _dy(w, 7), dlast=dlast)


@pytest.mark.parametrize("variant", ["no_z", "no_D", "no_bias", "no_softplus", "bare"])
def test_bwd_optional_inputs(variant):
    kw = {"no_z": dict(with_z=False), "no_D": dict(with_D=False),
          "no_bias": dict(with_bias=False), "no_softplus": dict(softplus=False),
          "bare": dict(with_z=False, with_D=False, with_bias=False, softplus=False)}[variant]
    w = dataclasses.replace(I.Workload("bwdopt", 2, 70, 130, 32, "f32"), **kw)
    x = I.make_inputs(w, seed=9)
    if not w.softplus:  # Delta = delta + bias must stay positive and small
        x["delta"] = (np.abs(x["delta"]) * 0.02 + 1e-3).astype(np.float32)
        if x["delta_bias"] is not None:
            x["delta_bias"] = np.full_like(x["delta_bias"], 1e-3)
    _run(w, x, _dy(w, 10), softplus=w.softplus)


def test_bwd_medium_workload():
    # several CTAs per batch row (the sums over channels cross CTAs), 64 chunks
    w = I.Workload("bwdmed", 2, 512, 1024, 16, "bf16")
    x = I.make_inputs(w, seed=11)
    _run(w, x, _dy(w, 12))


@pytest.mark.parametrize("ckpt", [False, True])
def test_bwd_full_workload(ckpt):
    # the bench workload, every gradient element
    w = I.WORKLOADS["b8_l2048_d1536_n16_bf16"]
    x = I.make_inputs(w, seed=31)
    _run(w, x, _dy(w, 32), ckpt=ckpt)


def test_bwd_workspace_too_small():
    w = I.Workload("bwdws", 1, 32, 64, 16, "f32")
    xd = to_device(I.make_inputs(w, seed=1))
    dy = torch.zeros(1, 32, 64, device="cuda")
    need = ss.ss_scan_bwd_workspace_bytes(1, 32, 64, 16)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ss.SSError):
        ss.ss_scan_bwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], dy, workspace=ws)
