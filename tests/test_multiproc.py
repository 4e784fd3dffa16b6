"""The N > 1 host path of bench.py, run as 2 gloo ranks on the CPU.

Every rank runs its own instance of the workload (the (batch, head) scans
are independent; no collective on the data path); the process group carries
only the barrier and the max-over-ranks time.  These tests cover that logic
without a GPU.
"""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    from test_sequence_layers_ttt_b200.inputs import WORKLOADS, make_inputs
    w_, r_, _ = bench.dist_setup()
    assert (w_, r_) == (world, rank) and dist.get_backend() == "gloo"
    t = bench.dist_max(1.5 + rank, world)     # each rank's "time"
    bench.dist_barrier(world)
    # each rank draws its own shard of independent scans: seed + rank
    q = make_inputs(WORKLOADS["linear_tiny_f32"], 0 + rank)["Q"]
    qs = [torch.zeros_like(q) for _ in range(world)]
    dist.all_gather(qs, q)
    out[rank] = (t, bool(torch.equal(qs[0], qs[1])))
    dist.destroy_process_group()


def test_gloo_two_ranks_max_and_independent_shards():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 2.5          # max over ranks, seen by both
    assert res[0][1] is False                     # ranks hold different instances


def test_reference_arm_under_torchrun_prints_once():
    """Launched like the driver's N = 2 run: rank 0 prints one JSON line, the
    other rank exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--workload", "linear_125m_2k", "--steps", "1",
           "--warmup", "0", "--ref-seconds", "0.2"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    p = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "tokens/s" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"


def test_gpus_flag_starts_the_ranks_itself():
    """`bench.py --gpus 2` run without torchrun starts two ranks on this node
    (the same line as under torchrun: rank 0 prints it once)."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", MASTER_PORT=str(_free_port()))
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--workload",
           "linear_125m_2k", "--steps", "1", "--warmup", "0", "--ref-seconds", "0.2"]
    p = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout
    assert json.loads(lines[0])["n_gpus"] == 2


@pytest.mark.parametrize("world,ms", [(1, 2.0), (2, 2.0), (8, 4.0)])
def test_weak_scaling_value_counts_every_rank(world, ms):
    sys.path.insert(0, ROOT)
    import bench
    from test_sequence_layers_ttt_b200.inputs import WORKLOADS
    w = WORKLOADS["linear_1p3b_32k"]
    assert bench.weak_scaling_value(w, world, ms) == pytest.approx(w.B * w.T * world / (ms * 1e-3))
