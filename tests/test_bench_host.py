"""Host-side logic of bench.py (CPU only): the roofline's traffic record is used only while
the recorded source digest matches the sources, the per-launch row accounting of the timed
step, the algorithmic work per launch, and the clock reader without a GPU."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from invariant_logprobs_reinforce_b200.build import source_digest  # noqa: E402


def _traffic_root(tmp_path, digest):
    (tmp_path / "profiles").mkdir()
    rec = {"kernels": {"dh": {"family": "gemm", "source_digest": digest, "rows": 16384,
                              "bytes_per_row": 1000.0}}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    return str(tmp_path)


def test_traffic_is_used_only_while_the_digest_matches(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", _traffic_root(tmp_path, source_digest("gemm")))
    assert bench.traffic_for("dh", 16384) == 1000.0 * 16384
    assert bench.traffic_for("dh", 448) == 1000.0 * 448  # scaled by the rows of a launch
    assert bench.traffic_for("dw", 16384) is None        # no record for the kernel


def test_traffic_is_null_after_a_source_change(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", _traffic_root(tmp_path, "0" * 16))
    assert bench.traffic_for("dh", 16384) is None


def test_launch_rows_of_a_chunked_step():
    n = 2 * 16384 + 448  # two full chunks and a ragged one
    per_chunk = ["lmhead_lse", "merge_lse", "token_kappa", "dz", "dh", "dw"]
    kinds = ["response_coef", "block_first"] + per_chunk * 3 + ["loss_final"]
    rows = bench.launch_rows(kinds, n)
    assert rows[:2] == [n, n] and rows[-1] == n
    body = rows[2:-1]
    assert body == [16384] * 6 + [16384] * 6 + [448] * 6
    assert sum(r for k, r in zip(kinds, rows) if k == "dh") == n


def test_algorithmic_work_per_launch():
    d, V, r = 2560, 151936, 16384
    for k in ("lmhead_lse", "dh", "dw"):
        assert bench.algorithmic_flops(k, r, d, V) == 2.0 * r * d * V
    assert bench.algorithmic_flops("dz", r, d, V) == 0.0
    # dZ conversion: read fp16 e and write bf16 dZ over V padded to a multiple of 8
    assert bench.algorithmic_bytes("dz", r, d, 7) == 4.0 * r * 8
    assert bench.algorithmic_bytes("dz", r, d, V) == 4.0 * r * V  # V = 151936 is a multiple of 8
    assert bench.job_throughput(1000, 4, 250.0) == 16000.0


def test_clock_reader_without_a_gpu_reports_nothing():
    with bench.NvmlClock(0) as clk:
        pass
    # on a host without a GPU NVML cannot start (or has no samples in an empty region)
    assert clk.sm_mhz is None or clk.sm_mhz > 0


def test_host_cpu_model_is_a_string():
    assert isinstance(bench.host_cpu_model(), str) and bench.host_cpu_model()
