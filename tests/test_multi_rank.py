"""The benchmark's multi-rank bookkeeping on CPU ranks (gloo, world size 2).

Replicas share nothing on the data path; the only cross-rank step is the
timing: every rank's elapsed time is reduced with MAX, and the whole-job rate
is all ranks' units over that slowest time.  The reference arm runs on rank 0
only; the other ranks exit without work.
"""
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as td
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench

    td.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 20.0][rank]
        m = bench.max_over_ranks(local_ms, torch.device("cpu"))
        rate = bench.whole_job_rate(4096 * 10, m, world)
        out[rank] = (m, rate)
        td.barrier()
    finally:
        td.destroy_process_group()


def test_max_over_ranks_and_rate_gloo():
    port = _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    assert out[0][0] == out[1][0] == 20.0
    assert abs(out[0][1] - 2 * 40960 / 0.020) < 1e-6


def test_single_rank_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.0, torch.device("cpu")) == 3.0
    assert bench.whole_job_rate(100, 1000.0, 1) == 100.0


def test_reference_arm_on_non_zero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
