"""Multi-rank logic of bench.py on CPU (gloo, world size 2): ranks time their
own batch and the job's time is the maximum over ranks; the reference arm runs
on rank 0 only.  No GPU and no data-path collective (the scan shards with no
exchange)."""
import json
import os
import re
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")
        dist.barrier()
        out[rank] = ms
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    port = bench._free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        assert dict(out) == {0: 15.0, 1: 15.0}


def test_job_throughput_is_weak_scaling():
    # two ranks each doing E elements per step in the slowest rank's time
    assert bench.job_throughput(1000, 2, 10, 5.0) == pytest.approx(2 * 1000 * 10 / 5e-3)
    assert bench.rank_seed(0, 0) != bench.rank_seed(1, 0)


def test_gpus_two_launches_two_ranks():
    """`bench.py --gpus 2` with no launcher starts two ranks itself; both join
    (gloo), rank 0 alone times the oracle and prints one line with n_gpus 2."""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "b2_l1024_d512_n16_f32", "--steps", "1", "--warmup", "3",
                        "--gpus", "2"], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0
    joined = sorted(re.findall(r"reference arm: rank \d of \d joined", r.stderr))
    assert joined == ["reference arm: rank 0 of 2 joined", "reference arm: rank 1 of 2 joined"]


def test_gpus_mismatch_with_launcher_is_refused():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "b2_l1024_d512_n16_f32", "--gpus", "2"], env=env,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "launcher started 1" in r.stderr
