"""The N > 1 host path on CPU (gloo, world size 2).

Several GPUs run independent replicas (weak scaling, no collective on the data
path): each rank draws its own seeded inputs, times its steps, and the job's
time is the maximum over ranks, taken by one all-reduce. Under torchrun the
reference arm (the CPU oracle) runs on rank 0 alone, which prints the one JSON
line; the other ranks exit 0 without work.
"""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _replica(rank: int, world: int, port: int, out):
    sys.path.insert(0, ROOT)
    import bench
    import synth
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        # the job's time: the slowest rank's
        out[rank * 3] = bench._max_over_ranks(dist, 1.5 * (rank + 1))
        # each replica's inputs come from its own seed (setup uses seed = 1 + rank)
        K, _, _ = synth.fathom_kv(1, 1, 128, 64, seed=1 + rank, with_v=False)
        v = torch.tensor([float(K[0, 0, 0, 0])], dtype=torch.float64)
        got = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(got, v)
        out[rank * 3 + 1] = float(got[0])
        out[rank * 3 + 2] = float(got[1])
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_replicas_time_is_max_over_ranks_and_inputs_differ():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Array("d", 3 * world)
    mp.start_processes(_replica, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0] == out[3] == 3.0
    assert out[1] == out[4] and out[2] == out[5]  # both ranks saw the same gather
    assert out[1] != out[2]  # and the replicas' inputs differ


def test_reference_arm_under_torchrun_prints_once_from_rank_zero():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "1",
           "--warmup", "0"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"


def test_sparq_like_channel_choice():
    """The SparQ-like comparison scan of the selection-quality diagnostic reads
    the r channels of largest |qbar_c|, ties to the lower channel."""
    sys.path.insert(0, ROOT)
    import bench
    qbar = torch.tensor([[0.5, -2.0, 1.0, 2.0, -1.0, 0.1]])
    assert bench.sparq_channels(qbar, 3).tolist() == [[1, 2, 3]]
    assert bench.sparq_channels(qbar, 4).tolist() == [[1, 2, 3, 4]]
    assert bench.sparq_channels(torch.zeros(1, 5), 2).tolist() == [[0, 1]]
