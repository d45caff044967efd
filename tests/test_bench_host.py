"""Host-side arithmetic of bench.py that needs no GPU: the algorithmic byte
counts behind the step and backward rooflines, and argument checks."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from selective_state_space_ss_b200 import inputs as I  # noqa: E402


def test_step_bytes_by_hand():
    # B=2, D=3, N=16, bf16: state 2*3*16*4 read + write, u/delta/z 3*2*3*2,
    # B/C 2*2*16*2, A 3*16*4, D and bias 2*3*4, y 2*3*4
    w = I.Workload("t", 2, 3, 1, 16, "bf16")
    expect = 2 * 384 + 36 + 128 + 192 + 24 + 24
    assert I.step_bytes(w) == expect


def test_step_workload_is_over_four_l2_when_rotated():
    w = I.STEP_WORKLOADS["step_b128_d8192_n16_bf16"]
    assert 140e6 < I.step_bytes(w) < 150e6
    nsets = -(-4 * bench.L2_BYTES // I.step_bytes(w))
    assert nsets * I.step_bytes(w) >= 4 * bench.L2_BYTES


def test_bwd_bytes_by_hand():
    # B=1, D=2, L=4, N=16, f32: reads u/delta/z 3*8*4 + B/C 2*64*4 + dy 8*4
    # + A, D, bias 2*18*4; writes du/ddelta/dz 3*8*4 + dB/dC 2*64*4 + dA, dD, dbias 2*18*4
    w = I.Workload("t", 1, 2, 4, 16, "f32")
    rd = 96 + 512 + 32 + 144
    wr = 96 + 512 + 144
    assert bench.bwd_bytes(w) == rd + wr


def test_forward_bytes_by_hand():
    # B=1, D=2, L=4, N=16, bf16 with z, D, bias: u/delta/z 3*8*2 + B/C 2*64*2
    # + A 2*16*4 + D, bias 2*2*4; y 8*4 + last state 2*16*4
    w = I.Workload("t", 1, 2, 4, 16, "bf16")
    assert w.algorithmic_bytes() == 48 + 256 + 128 + 16 + 32 + 128


def test_cli_rejects_mixed_modes():
    run = lambda *a: subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *a],
                                    capture_output=True, text=True)
    assert run("--conv", "4", "--zoh").returncode != 0
    assert run("--warmup", "2").returncode != 0
    assert run("--workload", "step_b128_d8192_n16_bf16").returncode != 0
    assert run("--op", "step", "--gpus", "2").returncode != 0


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the fp64 oracle on the host cores) prints one
    JSON line with the contract's keys on the default workload."""
    import json

    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == bench.DEFAULT_WORKLOAD
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_traffic_records_key_the_code_not_the_comments():
    # a comment or blank-line edit keeps a kernel's traffic record valid; any
    # code edit voids it
    src = "// header\nint f(int x) {  // trailing\n  /* block\n  comment */ return x + 1;\n\n}\n"
    assert bench._code_only(src) == bench._code_only(src.replace("trailing", "other") + "\n// more\n")
    assert bench._code_only(src) != bench._code_only(src.replace("x + 1", "x + 2"))
    assert "header" not in bench._code_only(src) and "block" not in bench._code_only(src)


def test_traffic_records_match_the_current_sources():
    # every record the bench reports on the committed sources was taken on them
    import json

    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        recs = json.load(f)
    fwd = bench.kernel_hash()
    keys = {bench.kernel_hash(), bench.kernel_hash(bench.BWD_KERNEL_SOURCES),
            bench.kernel_hash(bench.STEP_KERNEL_SOURCES)}
    assert recs["b1_l1048576_d1536_n16_bf16"]["kernel_hash"] == fwd
    assert all(r["kernel_hash"] in keys for r in recs.values())
