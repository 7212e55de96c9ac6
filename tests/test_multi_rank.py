"""The N > 1 path of the benchmark on the CPU: one process per rank over the
gloo backend, world size 2.  The layer itself has no collective (every
(batch, head) sequence is independent, so N GPUs run N replicas); what runs
across ranks is the timing protocol (barriers, the max over ranks of the
step time) and the reference arm's rank-0-only rule."""

import json
import os
import socket
import subprocess
import sys

import pytest
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


def _max_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, local = bench.dist_env()
        assert (r, w, local) == (rank, world, rank)
        bench.barrier(world)
        ms = 3.0 + 4.0 * rank                       # per-rank step times
        got = bench.max_over_ranks(ms, world, torch.device("cpu"))
        out.put((rank, got))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_step_time_is_the_max_over_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.SimpleQueue()
    mp.start_processes(_max_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    got = sorted(out.get() for _ in range(world))
    assert got == [(0, 7.0), (1, 7.0)]


def test_replicas_draw_independent_inputs():
    """Weak scaling: rank r runs the same workload on its own seed (no data
    is exchanged, so the aggregate throughput counts every rank's tokens)."""
    from gated_linear_sliding_chunkwise_b200.synth import WORKLOADS, make_inputs

    w = WORKLOADS["tiny_fp32"]
    a = make_inputs(w, seed=w.seed + 0)
    b = make_inputs(w, seed=w.seed + 1)
    assert a["q"].shape == b["q"].shape
    assert not torch.equal(a["q"], b["q"])
    # the per-head parameters are the same draw on every rank only if the
    # seeds match; replicas are independent models of the same shape
    assert a["fmap_wq"].shape == b["fmap_wq"].shape


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun_two_ranks():
    """`bench.py --impl reference` launched as the driver launches N > 1:
    every rank exits 0, rank 0 alone prints one JSON line."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    res = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=540)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
