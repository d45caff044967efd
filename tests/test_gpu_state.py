"""GPU-vs-oracle parity for the carried state: ss_scan_fwd_from_state (a scan
started from an initial state) and ss_scan_step (one recurrent decode step
that advances the state in place), both through the C ABI.

Tolerances as for the forward: fp32 inputs 1e-5, bf16 inputs 2e-3, relative to
the largest reference value; the state under the same rule against max|h_ref|.
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


def _from_state(xd, h0, softplus=True, **kw):
    return ss.ss_scan_fwd_from_state(h0, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                                     z=xd["z"], delta_bias=xd["delta_bias"], softplus=softplus, **kw)


def _oracle_from_state(x, h0, softplus=True):
    return oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"],
                           x["delta_bias"], softplus=softplus, h0=h0)


def _check(w, got_y, got_h, ref_y, ref_h):
    tol = TOL[w.dtype]
    ey = rel_err(got_y.cpu().numpy(), ref_y)
    eh = rel_err(got_h.cpu().numpy(), ref_h)
    assert ey <= tol, f"{w.name}: y rel err {ey:.3e} > {tol}"
    assert eh <= tol, f"{w.name}: state rel err {eh:.3e} > {tol}"


# ------------------------------------------------ scan from a carried state --

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [16, 32, 64, 128])
@pytest.mark.parametrize("L", [1, 7, 300, 2049])
def test_from_state_small_shapes(dtype, N, L):
    w = I.Workload(f"h0_{dtype}_N{N}_L{L}", 3, 37, L, N, dtype)
    x = I.make_inputs(w, seed=L + 7 * N)
    h0 = I.make_state(w.batch, w.dim, N, seed=L + N)
    xd = to_device(x)
    y, h = _from_state(xd, torch.from_numpy(h0).cuda())
    yr, hr = _oracle_from_state(x, h0)
    _check(w, y, h, yr, hr)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [16, 64])
def test_from_state_time_split_mode(dtype, N):
    # one batch row of 24 channels: too few channel groups to fill the GPU, so
    # N = 16 takes the time-split kernel
    w = I.Workload(f"h0split_{dtype}_{N}", 1, 24, 3000, N, dtype)
    x = I.make_inputs(w, seed=31)
    h0 = I.make_state(1, 24, N, seed=32)
    y, h = _from_state(to_device(x), torch.from_numpy(h0).cuda())
    yr, hr = _oracle_from_state(x, h0)
    _check(w, y, h, yr, hr)


@pytest.mark.parametrize("workers", [2, 3, 7])
@pytest.mark.parametrize("N", [16, 128])
def test_from_state_balanced_schedule(workers, N):
    # forced worker counts: ranges start and end inside channel groups, so the
    # initial state must be read only by the piece that starts a group
    w = I.Workload(f"h0bal_{N}_{workers}", 5, 40, 1000, N, "bf16")
    x = I.make_inputs(w, seed=workers)
    h0 = I.make_state(5, 40, N, seed=workers + 1)
    xd = to_device(x)
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, workers)
    need = ss.ss_scan_workspace_bytes(w.batch, w.dim, w.seqlen, w.dstate)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    y, h = _from_state(xd, torch.from_numpy(h0).cuda(), workspace=ws)
    assert ss.ss_last_device_error() == ss.SS_OK
    yr, hr = _oracle_from_state(x, h0)
    _check(w, y, h, yr, hr)


@pytest.mark.parametrize("workers", [0, 3])
def test_from_state_in_place(workers):
    # last_state_out is the initial-state buffer itself
    w = I.Workload("h0inplace", 4, 70, 513, 32, "bf16")
    x = I.make_inputs(w, seed=41)
    h0 = I.make_state(4, 70, 32, seed=42)
    state = torch.from_numpy(h0).cuda()
    if workers:
        ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, workers)
    y, h = _from_state(to_device(x), state, last_state_out=state)
    assert h.data_ptr() == state.data_ptr()
    assert ss.ss_last_device_error() == ss.SS_OK
    yr, hr = _oracle_from_state(x, h0)
    _check(w, y, state, yr, hr)


def test_from_state_none_is_zero_state():
    w = I.Workload("h0none", 2, 50, 200, 16, "f32")
    x = I.make_inputs(w, seed=3)
    xd = to_device(x)
    y0, h0 = ss.ss_scan_fwd(xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"], z=xd["z"],
                            delta_bias=xd["delta_bias"])
    y1, h1 = _from_state(xd, None)
    assert torch.equal(y0, y1) and torch.equal(h0, h1)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_sequence_in_pieces_matches_one_scan(dtype):
    # a prompt fed in three pieces, the state carried in place between calls
    w = I.Workload(f"pieces_{dtype}", 2, 96, 1500, 16, dtype)
    x = I.make_inputs(w, seed=51)
    cuts = [0, 512, 1001, 1500]
    state = torch.zeros(2, 96, 16, device="cuda")
    ys = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        part = {k: (np.ascontiguousarray(v[:, :, a:b]) if k in ("u", "delta", "z", "B", "C") else v)
                for k, v in x.items()}
        y, _ = _from_state(to_device(part), state, last_state_out=state)
        ys.append(y)
    yr, hr = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"])
    _check(w, torch.cat(ys, dim=2), state, yr, hr)


# ------------------------------------------------------- one decode step ----

def _step_gpu(xd, state, softplus=True, **kw):
    return ss.ss_scan_step(state, xd["u"], xd["delta"], xd["A"], xd["B"], xd["C"], D=xd["D"],
                           z=xd["z"], delta_bias=xd["delta_bias"], softplus=softplus, **kw)


def _step_oracle(x, softplus=True):
    return oracle.scan_step(x["state"], x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"],
                            x["delta_bias"], softplus=softplus)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [16, 32, 64, 128])
@pytest.mark.parametrize("batch,dim", [(1, 1), (3, 37), (2, 1000), (7, 513)])
def test_step_shapes(dtype, N, batch, dim):
    w = I.Workload(f"step_{dtype}_{N}_{batch}x{dim}", batch, dim, 1, N, dtype)
    x = I.make_step_inputs(w, seed=batch * 1000 + dim + N)
    xd = to_device(x)
    y = _step_gpu(xd, xd["state"])
    yr, hr = _step_oracle(x)
    _check(w, y, xd["state"], yr, hr)


@pytest.mark.parametrize("simple", [False, True])
@pytest.mark.parametrize("variant", ["no_z", "no_D", "no_bias", "no_softplus", "bare"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_step_optional_inputs(variant, dtype, simple):
    # dim 304: rows of 16-byte multiples, so the bulk-copy pipeline applies
    # unless the plain-load kernel is forced
    kw = {"no_z": dict(with_z=False), "no_D": dict(with_D=False),
          "no_bias": dict(with_bias=False), "no_softplus": dict(softplus=False),
          "bare": dict(with_z=False, with_D=False, with_bias=False, softplus=False)}[variant]
    w = dataclasses.replace(I.Workload("stepopt", 4, 304, 1, 32, dtype), **kw)
    x = I.make_step_inputs(w, seed=9)
    if not w.softplus:  # without the softplus Delta = delta + bias must stay positive and small
        dl = np.abs(I.bf16_to_f32(x["delta"]) if dtype == "bf16" else x["delta"]) * 0.02 + 1e-3
        x["delta"] = (dl.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16) \
            if dtype == "bf16" else dl.astype(np.float32)
        if x["delta_bias"] is not None:
            x["delta_bias"] = np.full_like(x["delta_bias"], 1e-3)
    xd = to_device(x)
    if simple:
        ss.ss_debug_inject(ss.SS_DEBUG_STEP_SIMPLE, 1)
    y = _step_gpu(xd, xd["state"], softplus=w.softplus)
    yr, hr = _step_oracle(x, softplus=w.softplus)
    _check(w, y, xd["state"], yr, hr)


@pytest.mark.parametrize("simple", [False, True])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [16, 32, 64, 128])
@pytest.mark.parametrize("batch,dim", [(1, 8), (3, 1000), (5, 4104), (300, 40)])
def test_step_both_kernels(dtype, N, batch, dim, simple):
    # shapes the bulk-copy pipeline takes: one partial tile, ragged last tiles,
    # many short rows (several tiles per CTA, channel tiles changing mid-range)
    w = I.Workload(f"steppipe_{dtype}_{N}_{batch}x{dim}", batch, dim, 1, N, dtype)
    x = I.make_step_inputs(w, seed=dim + N + batch)
    xd = to_device(x)
    if simple:
        ss.ss_debug_inject(ss.SS_DEBUG_STEP_SIMPLE, 1)
    y = _step_gpu(xd, xd["state"])
    yr, hr = _step_oracle(x)
    _check(w, y, xd["state"], yr, hr)


def test_step_batch_beyond_grid_rows():
    # more batch rows than one grid dimension holds: the kernel walks the rest
    w = I.Workload("stepbig", 70000, 3, 1, 16, "bf16")
    x = I.make_step_inputs(w, seed=13)
    xd = to_device(x)
    y = _step_gpu(xd, xd["state"])
    yr, hr = _step_oracle(x)
    _check(w, y, xd["state"], yr, hr)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_step_unaligned_views(dtype):
    # state and B/C that start off a vector boundary take element-wise loads
    w = I.Workload(f"stepun_{dtype}", 3, 50, 1, 16, dtype)
    x = I.make_step_inputs(w, seed=17)
    xd = to_device(x)
    st_buf = torch.zeros(xd["state"].numel() + 1, device="cuda")
    state = st_buf[1:].view_as(xd["state"])
    state.copy_(xd["state"])
    views = {}
    for k in ("B", "C"):
        buf = torch.zeros(xd[k].numel() + 1, dtype=xd[k].dtype, device="cuda")
        views[k] = buf[1:].view_as(xd[k])
        views[k].copy_(xd[k])
    xd2 = dict(xd, **views)
    y = _step_gpu(xd2, state)
    yr, hr = _step_oracle(x)
    _check(w, y, state, yr, hr)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_step_chain_matches_scan(dtype):
    # a prompt scanned with the fused kernel, then tokens generated one step at
    # a time, against the oracle's scan over the whole sequence
    P, S = 300, 40
    w = I.Workload(f"chain_{dtype}", 2, 80, P + S, 16, dtype)
    x = I.make_inputs(w, seed=61)
    xd = to_device(x)
    cut = lambda k, a, b: xd[k][:, :, a:b].contiguous()
    y_p, state = ss.ss_scan_fwd(cut("u", 0, P), cut("delta", 0, P), xd["A"], cut("B", 0, P),
                                cut("C", 0, P), D=xd["D"], z=cut("z", 0, P), delta_bias=xd["delta_bias"])
    ys = [y_p]
    for t in range(P, P + S):
        tok = {k: xd[k][:, :, t].contiguous() for k in ("u", "delta", "z", "B", "C")}
        y = ss.ss_scan_step(state, tok["u"], tok["delta"], xd["A"], tok["B"], tok["C"], D=xd["D"],
                            z=tok["z"], delta_bias=xd["delta_bias"])
        ys.append(y[..., None])
    yr, hr = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"])
    _check(w, torch.cat(ys, dim=2), state, yr, hr)


@pytest.mark.parametrize("name", sorted(I.STEP_WORKLOADS))
def test_step_full_workloads(name):
    w = I.STEP_WORKLOADS[name]
    x = I.make_step_inputs(w, seed=1234)
    xd = to_device(x)
    y = _step_gpu(xd, xd["state"])
    yr, hr = _step_oracle(x)
    _check(w, y, xd["state"], yr, hr)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_step_chain_in_a_cuda_graph(dtype):
    # eight consecutive decode steps captured in one CUDA graph: each step is a
    # programmatic dependent of the one before (it may start while that one
    # drains and waits for it before reading the state it wrote)
    S = 8
    w = I.Workload(f"stepgraph_{dtype}", 3, 1000, S, 16, dtype)
    x = I.make_inputs(w, seed=71)
    h0 = I.make_state(w.batch, w.dim, w.dstate, seed=72)
    xd = to_device(x)
    toks = [{k: xd[k][:, :, t].contiguous() for k in ("u", "delta", "z", "B", "C")} for t in range(S)]
    state = torch.from_numpy(h0).cuda()
    ys = [torch.empty(w.batch, w.dim, device="cuda") for _ in range(S)]

    def chain():
        for t in range(S):
            tk = toks[t]
            ss.ss_scan_step(state, tk["u"], tk["delta"], xd["A"], tk["B"], tk["C"], D=xd["D"],
                            z=tk["z"], delta_bias=xd["delta_bias"], y_out=ys[t])

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm up outside the capture
        chain()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        chain()
    state.copy_(torch.from_numpy(h0))
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    assert ss.ss_last_device_error() == ss.SS_OK
    yr, hr = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"],
                             x["delta_bias"], h0=h0)
    _check(w, torch.stack(ys, dim=2), state, yr, hr)
