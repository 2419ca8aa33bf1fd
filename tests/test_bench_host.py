"""Host logic of bench.py, on CPU: how each workload is launched, the launch
and byte counts its JSON line reports, and the reference arm's line (the
oracle timed on a bounded sample)."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

import bench
from workloads import WORKLOADS, algorithmic_bytes, make_projections

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _projs(name):
    shapes, M = WORKLOADS[name]
    return list(make_projections(shapes[:7], M=M, seed=0, with_weights=False))


@pytest.mark.parametrize("name,mode", [
    ("stack30_m1", "fused"), ("layer_m1", "fused"), ("ffn_m1", "fused"),
    ("ffn_m2", "batch"), ("ffn_m4", "batch"), ("ffn_m8", "batch"), ("ffn_m24", "batch"),
    ("stack30_m4", "batch"), ("stack30_m16", "batch"),
    ("single_640x2560_m1", "fused"), ("prefill_m512", "prefill"),
])
def test_step_mode(name, mode):
    assert bench.step_mode(_projs(name)) == mode


def test_batch_launch_counts():
    # 512 projections per quantiser launch; 256 projections per streaming
    # (M <= 2) or warp-MMA (3..24) launch, 64 per tensor-core group launch
    assert bench.batch_launches(3, 4) == 1 + 1
    assert bench.batch_launches(3, 16) == 1 + 1
    assert bench.batch_launches(210, 4) == 1 + 1
    assert bench.batch_launches(210, 16) == 1 + 1
    assert bench.batch_launches(210, 24) == 1 + 1
    assert bench.batch_launches(210, 32) == 1 + 4
    assert bench.batch_launches(300, 2) == 1 + 2
    assert bench.batch_launches(600, 2) == 2 + 3


def test_prefill_launch_counts():
    # 512 projections per quantiser launch, 16 per grouped prefill launch
    assert bench.prefill_launches(3, 512) == 1 + 1
    assert bench.prefill_launches(16, 64) == 1 + 1
    assert bench.prefill_launches(17, 512) == 1 + 2


def test_binary_kernel_name(monkeypatch):
    monkeypatch.delenv("TQ_BINARY_KERNEL", raising=False)
    assert [bench.binary_kernel_name(m) for m in (1, 2, 4)] == [
        "binary_mma_kernel", "binary_gemv_kernel", "binary_gemv_kernel"]
    monkeypatch.setenv("TQ_BINARY_KERNEL", "dp4a")
    assert bench.binary_kernel_name(1) == "binary_gemv_kernel"


def test_kernel_names_follow_the_choice_by_m(monkeypatch):
    monkeypatch.delenv("TQ_BATCH_KERNEL", raising=False)
    assert [bench.batch_kernel_name(m, "batch") for m in (1, 2, 3, 16, 17, 24, 25, 32)] == [
        "stream_gemv_kernel", "stream_gemv_kernel", "mma_gemv_kernel", "mma_gemv_kernel",
        "mma_gemv_kernel", "mma_gemv_kernel", "smallm_group_kernel", "smallm_group_kernel"]
    assert bench.batch_kernel_name(24, "per_projection") == "mma_gemv_kernel"
    assert bench.batch_kernel_name(28, "per_projection") == "smallm_tc_kernel"
    monkeypatch.setenv("TQ_BATCH_KERNEL", "tc")
    assert bench.batch_kernel_name(8, "batch") == "smallm_group_kernel"


def test_step_bytes_by_mode():
    fused = _projs("ffn_m1")
    # one quantising launch: GEMV bytes + bf16 activations read
    assert bench.workload_step_bytes("ffn_m1", fused) == sum(
        algorithmic_bytes(p.N, p.K, 1) + 2 * p.K for p in fused)
    batch = _projs("ffn_m16")
    # quantiser (bf16 in, int8 + scale + sum out) then the GEMV
    assert bench.workload_step_bytes("ffn_m16", batch) == sum(
        2 * 16 * p.K + 16 * p.K + 16 * 8 + algorithmic_bytes(p.N, p.K, 16) for p in batch)


def test_whole_job_rate_and_max_over_ranks_identity():
    assert bench.whole_job_rate(4, 1e9, 2.0) == pytest.approx(2e12)
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]


def test_reference_arm_line():
    out = subprocess.run(
        [sys.executable, "bench.py", "--impl", "reference", "--workload", "ffn_m4",
         "--steps", "1", "--warmup", "3"],
        cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    d = json.loads(out.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["steps"] == 1 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_warmup_below_three_is_rejected():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--warmup", "2"],
                         cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode != 0 and "warmup" in out.stderr


def test_recorded_binary_traffic_needs_the_same_kernel_and_workload():
    # a record is used only for the kernel version, kernel and workload it was taken on
    assert bench.recorded_binary_traffic("binary_ffn27b_m1", "binary_gemv_kernel") is None
    assert bench.recorded_binary_traffic("prefill_m512", "binary_mma_kernel") is None
    assert len(bench.binary_kernel_sha()) == 16


def test_prefill_kernel_name(monkeypatch):
    monkeypatch.delenv("TQ_PREFILL_PAIR", raising=False)
    assert [bench.prefill_kernel_name(m) for m in (33, 128, 129, 512)] == [
        "prefill_tc_kernel", "prefill_tc_kernel", "prefill_pair_kernel", "prefill_pair_kernel"]
    monkeypatch.setenv("TQ_PREFILL_PAIR", "0")
    assert bench.prefill_kernel_name(512) == "prefill_tc_kernel"



def test_percentile_matches_numpy():
    rng = np.random.default_rng(3)
    for n in (1, 2, 7, 125):
        v = sorted(rng.random(n).tolist())
        for q in (0, 10, 50, 90, 100):
            assert abs(bench.percentile(v, q) - np.percentile(v, q)) < 1e-12


def test_step_spread_from_chunk_events():
    class Mark:
        def __init__(self, t):
            self.t = t

        def elapsed_time(self, later):
            return later.t - self.t

    # four chunks of 16 steps: 1.6, 1.6, 1.8, 1.6 ms
    marks = [Mark(t) for t in (0.0, 1.6, 3.2, 5.0, 6.6)]
    sp = bench.step_spread(marks, 16)
    assert sp["chunks"] == 4 and sp["steps_per_chunk"] == 16
    assert sp["median_ms"] == 0.1 and sp["p10_ms"] == 0.1
    assert abs(sp["p90_ms"] - 0.10875) < 1e-9
    assert bench.step_spread(marks[:2], 16) is None
