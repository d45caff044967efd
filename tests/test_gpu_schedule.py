"""The load-balanced schedule: CTAs own equal ranges of (channel group, chunk)
units, split groups hand their state to the next CTA through the workspace, and
those waits are bounded.  Forced worker counts exercise the handoff on small
shapes; a skipped publish exercises the timeout path (no hang, no fault: the
kernel gives up, reports SS_ERR_TIMEOUT and the next call is correct)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import selective_state_space_ss_b200 as ss  # noqa: E402
from selective_state_space_ss_b200 import inputs as I  # noqa: E402
from tests.helpers import TOL, rel_err, run_gpu, to_device  # noqa: E402


def _check(w, x, y, h):
    yr, hr = oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"],
                             x["delta_bias"], softplus=w.softplus)
    assert rel_err(y.cpu().numpy(), yr) <= TOL[w.dtype]
    assert rel_err(h.cpu().numpy(), hr) <= TOL[w.dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [16, 32, 64, 128])
@pytest.mark.parametrize("L,workers", [(1000, 3), (4097, 5), (256, 7), (33, 2), (8, 4)])
def test_forced_split_parity(dtype, N, L, workers):
    # 5 batch rows x 40 channels: several channel groups per row, a partial
    # last group, ranges that start and end inside groups
    w = I.Workload(f"split_{dtype}_{N}_{L}", 5, 40, L, N, dtype)
    x = I.make_inputs(w, seed=L + N)
    xd = to_device(x)
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, workers)
    need = ss.ss_scan_workspace_bytes(w.batch, w.dim, w.seqlen, w.dstate)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    y, h = run_gpu(xd, workspace=ws)
    assert ss.ss_last_device_error() == ss.SS_OK
    _check(w, x, y, h)


def test_split_workspace_is_reused_across_calls():
    w = I.Workload("reuse", 4, 64, 700, 16, "bf16")
    x = I.make_inputs(w, seed=11)
    xd = to_device(x)
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, 3)
    ws = torch.full((ss.ss_scan_workspace_bytes(w.batch, w.dim, w.seqlen, w.dstate),), 0xAB,
                    dtype=torch.uint8, device="cuda")
    for _ in range(3):  # stale flags from earlier calls must never be taken as fresh
        ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, 3)
        y, h = run_gpu(xd, workspace=ws)
        assert ss.ss_last_device_error() == ss.SS_OK
        _check(w, x, y, h)


def test_carry_wait_times_out_cleanly():
    w = I.Workload("timeout", 4, 64, 512, 16, "bf16")
    x = I.make_inputs(w, seed=12)
    xd = to_device(x)
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, 3)
    ws = torch.empty(ss.ss_scan_workspace_bytes(w.batch, w.dim, w.seqlen, w.dstate),
                     dtype=torch.uint8, device="cuda")
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, 3)
    ss.ss_debug_inject(ss.SS_DEBUG_SKIP_PUBLISH, 1)   # worker 2 waits for a carry that never comes
    ss.ss_debug_inject(ss.SS_DEBUG_SPIN_LIMIT, 2000)
    run_gpu(xd, workspace=ws)
    assert ss.ss_last_device_error() == ss.SS_ERR_TIMEOUT
    assert ss.ss_last_device_error() == ss.SS_OK  # read-and-clear
    # the context is intact and the next call is right
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, 3)
    y, h = run_gpu(xd, workspace=ws)
    assert ss.ss_last_device_error() == ss.SS_OK
    _check(w, x, y, h)


def test_debug_hooks_clear():
    # one channel group of 8 channels x 2 chunks: a single segment of one chunk
    # needs no scratch, so any bytes here would come from a pending setting
    w = I.Workload("clear", 1, 8, 32, 16, "f32")
    assert ss.ss_scan_workspace_bytes(w.batch, w.dim, w.seqlen, w.dstate) == 0
    for hook in (ss.SS_DEBUG_FORCE_WORKERS, ss.SS_DEBUG_FORCE_SEGMENTS):
        ss.ss_debug_inject(hook, 2)
        ss.ss_debug_inject(ss.SS_DEBUG_CLEAR)
        assert ss.ss_scan_workspace_bytes(w.batch, w.dim, w.seqlen, w.dstate) == 0
    w2 = I.Workload("clear2", 1, 8, 64, 16, "f32")  # two chunks: segments when asked
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_SEGMENTS, 2)
    assert ss.ss_scan_workspace_bytes(w2.batch, w2.dim, w2.seqlen, w2.dstate) > 0
    ss.ss_debug_inject(ss.SS_DEBUG_CLEAR)


@pytest.mark.parametrize("workers", [0, 3])
def test_replay_in_a_cuda_graph(workers):
    """The scan captured once into a CUDA graph and replayed on new inputs
    copied into the captured buffers: the balanced schedule's carry flags are
    consumed by each replay, so a replay never takes the previous one's carry."""
    w = I.Workload(f"graph_{workers}", 5, 40, 1000, 16, "bf16")
    xs = [I.make_inputs(w, seed=s) for s in (21, 22, 23)]
    static = to_device(xs[0])
    need = ss.ss_scan_workspace_bytes(w.batch, w.dim, w.seqlen, w.dstate) if not workers else None
    if workers:
        ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, workers)
        need = ss.ss_scan_workspace_bytes(w.batch, w.dim, w.seqlen, w.dstate)
    ws = torch.zeros(max(need, 1), dtype=torch.uint8, device="cuda")
    y = torch.empty(w.batch, w.dim, w.seqlen, device="cuda")
    h = torch.empty(w.batch, w.dim, w.dstate, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm up outside the capture
        if workers:
            ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, workers)
        run_gpu(static, y_out=y, last_state_out=h, workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    if workers:
        ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, workers)
    with torch.cuda.graph(graph):
        run_gpu(static, y_out=y, last_state_out=h, workspace=ws)
    for x in xs + [xs[0]]:
        src = to_device(x)
        for k, v in src.items():
            if v is not None:
                static[k].copy_(v)
        graph.replay()
        torch.cuda.synchronize()
        assert ss.ss_last_device_error() == ss.SS_OK
        _check(w, x, y, h)


def test_balanced_schedule_beside_other_work():
    # The balanced schedule's workers take their ids from a counter as they
    # start, so a worker only ever waits for one that is already running.  A
    # matmul on another stream holds SM slots while the scan launches more
    # workers than channel groups fit at once; the scan must finish without a
    # carry wait giving up.
    w = I.Workload("split_busy", 64, 512, 2048, 16, "bf16")
    x = I.make_inputs(w, seed=41)
    xd = to_device(x)
    groups = w.batch * (w.dim // 32)
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, groups - 1)
    need = ss.ss_scan_workspace_bytes(w.batch, w.dim, w.seqlen, w.dstate)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    a = torch.randn(8192, 8192, device="cuda")
    side = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(side):
        for _ in range(4):
            a = a @ a.T * 1e-4
    ss.ss_debug_inject(ss.SS_DEBUG_FORCE_WORKERS, groups - 1)
    y, h = run_gpu(xd, workspace=ws)
    torch.cuda.synchronize()
    assert ss.ss_last_device_error() == ss.SS_OK
    _check(w, x, y, h)
