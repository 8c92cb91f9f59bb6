"""Host logic of the N > 1 path on CPU: two gloo ranks.

The layer needs no collective, so N GPUs run N independent replicas and the only cross-rank
step is the timing reduction (the slowest rank sets the job's time, throughput counts every
rank's tokens).  Those steps, and the reference arm's rank handling under torchrun (rank 0
alone runs and prints; the others exit 0 without work), are exercised here with world size 2.
"""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # rank r reports times (r + 1, 10 - r): the maximum over ranks is (world, 10)
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank], torch.device("cpu"))
        tput = bench.job_tokens_per_s(world, 4096, got[0])
        q.put((rank, got, tput))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


PORT = _free_port()


def test_max_over_ranks_and_job_throughput_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world = 2
    procs = [ctx.Process(target=_worker, args=(r, world, PORT, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, tput in res:
        assert got == [2.0, 10.0], (rank, got)
        # 2 ranks x 4096 tokens in the slowest rank's 2 ms
        assert tput == pytest.approx(2 * 4096 / 2e-3)



def test_single_process_reduction_is_identity():
    import bench
    assert not bench.dist_on()
    assert bench.max_over_ranks([3.5, 1.25], torch.device("cpu")) == [3.5, 1.25]
    assert bench.job_tokens_per_s(1, 4096, 0.5) == pytest.approx(4096 / 5e-4)


def test_reference_arm_under_torchrun_world2():
    """Reference arm, 2 ranks: rank 0 prints one JSON line; rank 1 exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "0"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["n_gpus"] == 2
    assert res["value"] > 0 and res["cpu_baseline"]["kind"] == "oracle"
    assert res["e2e"]["h2d_bytes_per_step"] == 0
