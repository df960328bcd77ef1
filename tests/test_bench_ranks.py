"""The benchmark's multi-process (replica) logic on CPU: world_size-2 gloo
process groups over 127.0.0.1, the max-over-ranks timing every rank joins,
the whole-job throughput, and the reference arm leaving non-zero ranks
without work.  The GPU path replicates the model per GPU with no data-path
collective, so these are the only cross-rank steps."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        t = bench.max_over_ranks(dist, world, times[rank], "cpu")
        out[rank] = t
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world, port = 2, _free_port()
    times = [12.5, 17.25]
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, port, times, out), nprocs=world, join=True)
    assert dict(out) == {0: 17.25, 1: 17.25}


def test_job_throughput_counts_every_replica_at_the_slowest_time():
    # 2 replicas x B=1 x u=2 tokens x 10 steps in 50 ms (the slower replica)
    assert bench.job_tokens_per_s(2, 1, 2, 10, 50.0) == pytest.approx(800.0)
    assert bench.job_tokens_per_s(1, 1, 2, 10, 50.0) == pytest.approx(400.0)


def test_reference_arm_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, env=env, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_world_size_must_match_gpus():
    assert bench.check_world(1, {}) == 1
    assert bench.check_world(2, {}) == 0            # outside a launcher: start the ranks
    assert bench.check_world(2, {"WORLD_SIZE": "2"}) == 2
    with pytest.raises(SystemExit):
        bench.check_world(8, {"WORLD_SIZE": "1"})
    argv = bench.launch_argv(2, ["--gpus", "2"], 29512)
    assert argv[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=2" in argv and "127.0.0.1" in argv and argv[-2:] == ["--gpus", "2"]


def test_gpus_2_without_launcher_starts_two_ranks():
    # the reference arm needs no GPU: run as `bench.py --gpus 2` outside any
    # launcher, it relaunches itself as two gloo-free ranks; rank 0 prints the
    # one line (n_gpus = 2), rank 1 exits without work, and the status is 0
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, env=env, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["extrapolated_x32"] is True and rec["steps"] == 1
