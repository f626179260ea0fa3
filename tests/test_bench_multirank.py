"""The benchmark's multi-rank logic on CPU: two gloo ranks.

Each rank runs an independent replica (weak scaling, no data-path
collective); the only cross-rank steps are the barriers around the timed
region and the max over ranks of the step time.  These tests run those
steps with world size 2 on the gloo backend, and launch the reference arm
under torchrun to check that rank 0 alone prints its line.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(None)
    assert (w, r) == (world, rank)
    bench.barrier(w)
    # rank 1 is the slow one: every rank must see its time
    ms = 2.0 if rank == 0 else 5.0
    m = bench.max_over_ranks(ms, w)
    rate = bench.whole_job_rate(1e9, m, w)
    q.put((rank, m, rate, bench.rank_seed(1002, rank)))
    bench.barrier(w)
    dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert [g[1] for g in got] == [5.0, 5.0]
    # 2 ranks x 1e9 units in 5 ms
    assert got[0][2] == pytest.approx(4e11) and got[1][2] == pytest.approx(4e11)
    assert got[0][3] != got[1][3]  # each replica draws its own batch


def test_single_rank_helpers():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(5e9, 10.0, 1) == pytest.approx(5e11)
    assert bench.rank_seed(7, 0) == 7


def test_reference_arm_under_torchrun_prints_one_line():
    port = _free_port()
    env = dict(os.environ, OMP_NUM_THREADS="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    # the launcher's OMP_NUM_THREADS=1 does not shrink the oracle: it runs on,
    # and reports, every core of the host
    assert d["cpu_baseline"]["cores"] == len(os.sched_getaffinity(0))
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_on_the_decode_workload():
    """--impl reference --workload decode: the oracle's decode over the first
    sequences of the same seeded batch, one JSON line in KV GB/s."""
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--workload", "decode", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == "decode KV GB/s" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["cores"] == len(os.sched_getaffinity(0)) and "sequences" in d["config"]["sample"]


def test_decode_cpu_baseline_helper():
    import bench
    w = bench.WORKLOADS["decode"]
    c = bench.oracle_decode_baseline(w, bench.rank_seed(w["seed"], 0), min_seconds=0.2)
    assert c["kind"] == "oracle" and c["unit"] == "GB/s" and c["value"] > 0
    assert c["cores"] == len(os.sched_getaffinity(0))
