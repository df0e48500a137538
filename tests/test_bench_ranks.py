"""Host-side logic of bench.py's multi-rank path, on CPU with gloo (world size 2).

Each rank runs its own batch (weak scaling, no collective on the data path);
the timed region's length is the maximum over ranks and rank 0 reports the
whole-job tokens/s.  The reference arm (the CPU oracle) runs on rank 0 only.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [120.0, 180.0][rank]  # the slower rank sets the job's time
        mx = bench.max_over_ranks(local_ms, world)
        value = bench.whole_job_tokens_per_s(mx, steps=10, world=world)
        q.put((rank, mx, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for _, mx, value in res:
        assert mx == 180.0
        assert value == pytest.approx(2 * 4096 * 10 / 0.180)


def test_single_rank_helpers_are_identities():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_tokens_per_s(1000.0, 5, 1) == pytest.approx(4096 * 5)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
