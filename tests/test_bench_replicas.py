"""bench.py's replica path (N > 1 GPUs run independent copies of the workload) on
CPU: the per-rank timings are reduced to the slowest rank's over a 2-rank gloo
group, and the whole-job throughput counts every rank's FLOPs over that time."""

import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r measured (step, forward) = (1 + r, 10 - r) ms
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank], world, "cpu")
        out[rank] = torch.tensor(got, dtype=torch.float64)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world, port = 2, _free_port()
    out = torch.zeros((world, 2), dtype=torch.float64).share_memory_()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    # every rank sees the element-wise maximum: slowest step 2 ms, slowest forward 10 ms
    assert out.tolist() == [[2.0, 10.0], [2.0, 10.0]]


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks([3.5, 1.25], 1, "cpu") == [3.5, 1.25]


def test_aggregate_counts_every_rank():
    # 2 replicas of 1e12 FLOPs each, slowest rank 2 ms per step -> 1000 TFLOP/s
    assert abs(bench.aggregate_tflops(1e12, 2, 2.0) - 1000.0) < 1e-9
    assert abs(bench.aggregate_tflops(1e12, 1, 2.0) - 500.0) < 1e-9


def test_reference_arm_prints_only_on_rank_zero():
    """Under torchrun the reference arm runs on rank 0 only; other ranks exit 0
    without output (no process group is needed for that)."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
