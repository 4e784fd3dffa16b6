"""bench.py's accounting on the CPU: the algorithmic bytes and FLOPs per
launch that the roofline fraction divides by, the metric names and configs
of every workload it accepts, and the recorded-traffic lookup.

The per-unit figures are the ones the design notes state: 644 bytes per
head-token for Q, K, V (bf16), eta and Z (fp32), plus the state read once and
written once; 6 d^2 + 64 d FLOPs per head-token for TTT-Linear and
14 d h + 32 (2 d + 2 h) for TTT-MLP.
"""
from __future__ import annotations

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from test_sequence_layers_ttt_b200.inputs import WORKLOADS  # noqa: E402


def test_linear_bytes_and_flops_per_launch():
    w = WORKLOADS["linear_1p3b_32k"]
    head_tokens = 2 * 32 * 32768
    assert bench.algorithmic_bytes(w) == head_tokens * 644 + 64 * 2 * (64 * 64 + 64) * 4 + 2 * 32 * 64 * 4
    assert bench.algorithmic_bytes(w) == 1_352_712_192
    assert bench.algorithmic_flops(w) == head_tokens * (6 * 64 * 64 + 64 * 64)
    w = WORKLOADS["linear_125m_2k"]
    assert bench.algorithmic_bytes(w) == 8 * 12 * 2048 * 644 + 96 * 2 * (64 * 64 + 64) * 4 + 2 * 12 * 64 * 4


def test_mlp_bytes_and_flops_per_launch():
    w = WORKLOADS["mlp_8k"]
    head_tokens = 4 * 12 * 8192
    assert bench.algorithmic_flops(w) == head_tokens * (14 * 64 * 256 + 32 * (2 * 64 + 2 * 256))
    assert bench.algorithmic_flops(w) == 98_247_376_896
    state = 2 * (2 * 64 * 256 + 256 + 64) * 4
    assert bench.algorithmic_bytes(w) == head_tokens * 644 + 48 * state + 2 * 12 * 64 * 4


def test_decode_bytes_per_step():
    # running and mini-batch start state each read and written, plus the token in and z out
    w = WORKLOADS["decode_1p3b"]
    assert bench.decode_state_bytes(w) == 64 * (4 * 4 * (64 * 64 + 64) + 3 * 64 * 2 + 4 + 64 * 4)
    assert bench.decode_state_bytes(w) == 4_301_056
    w = WORKLOADS["decode_mlp_8k"]
    assert bench.decode_state_bytes(w) == 48 * (4 * 4 * (2 * 64 * 256 + 256 + 64) + 3 * 64 * 2 + 4 + 64 * 4)


@pytest.mark.parametrize("name", [k for k, v in WORKLOADS.items() if v.T >= 2048] + list(bench.DECODE_WORKLOADS))
def test_every_bench_workload_has_a_metric_and_config(name):
    w = WORKLOADS[name]
    assert bench.metric_name(w)
    cfg = bench.workload_config(w)
    assert cfg["workload"] == name and "l2" in cfg


def test_default_metric_is_the_headline():
    assert bench.metric_name(WORKLOADS["linear_1p3b_32k"]) == bench.METRIC


def test_recorded_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    kernel = "ttt_linear_lag_kernel"
    good = bench.kernel_source_hash(kernel)
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "dram_traffic.txt").write_text(
        "# kernel workload source_hash bytes\n"
        f"{kernel} linear_1p3b_32k {good} 123\n"
        f"{kernel} linear_125m_2k 0000000000000000 456\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the hash is taken over the real sources, which stay where they are
    monkeypatch.setattr(bench, "kernel_source_hash", lambda k: good)
    assert bench.recorded_traffic(kernel, "linear_1p3b_32k") == 123
    assert bench.recorded_traffic(kernel, "linear_125m_2k") is None   # stale record
    assert bench.recorded_traffic(kernel, "mlp_8k") is None           # no record


def test_committed_traffic_records_are_well_formed():
    """Every line of the committed table names a kernel bench.py can hash and a
    workload it runs, with a 16-digit hex hash and a positive byte count, and no
    (kernel, workload) pair appears twice."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    seen = set()
    with open(path) as fh:
        for line in fh:
            f = line.split("#")[0].split()
            if not f:
                continue
            assert len(f) == 4, line
            kernel, workload, digest, nbytes = f
            assert kernel in bench.KERNEL_SOURCES, line
            assert workload in WORKLOADS or workload in bench.PROLOGUES or workload in bench.BACKWARD, line
            assert len(digest) == 16 and int(digest, 16) >= 0, line
            assert int(nbytes) > 0, line
            assert (kernel, workload) not in seen, line
            seen.add((kernel, workload))
