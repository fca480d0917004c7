"""Multi-process host logic of the benchmark on CPU (gloo, world size 2).

The decode path shards by batch with no exchange (replicas), so the only
cross-rank steps are the max-over-ranks timing reduction and the whole-job
rate; the reference arm runs on rank 0 alone under torchrun.
"""
import datetime
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        vals = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 2.0 * (rank + 1)], "cpu")
        seed = bench.rank_seed("v3", rank)
        dist.barrier()
        q.put((rank, vals, seed))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_per_rank_batches_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = [q.get(timeout=180) for _ in range(2)]
    finally:
        for p in procs:
            p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    by_rank = {r: (v, s) for r, v, s in res}
    # every rank sees the slowest rank's figure for each timing
    assert by_rank[0][0] == by_rank[1][0] == [2.0, 5.0, 4.0]
    # replicas decode different batches
    assert by_rank[0][1] != by_rank[1][1]


def test_max_over_ranks_is_identity_without_a_process_group():
    assert bench.max_over_ranks([3.0, 1.5], "cpu") == [3.0, 1.5]


def test_job_rate_counts_every_rank():
    # 1 GB per rank per step, 4 ranks, 1 s per step -> 4 GB/s for the job
    assert bench.job_rate(1e9, 4, 1000.0) == pytest.approx(4.0)
    assert bench.job_rate(1e9, 1, 1000.0) == pytest.approx(1.0)


def test_reference_arm_under_torchrun_prints_one_line_from_rank_zero(tmp_path):
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "5",
           "--cpu-seconds", "0.3", "--workload", "tiny"]
    env = dict(os.environ, TMPDIR=str(tmp_path))  # torchrun's scratch files go to pytest's tmp dir
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
