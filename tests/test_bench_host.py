"""Host-side logic of bench.py (CPU only): the roofline's traffic record is used only while
the recorded source digest matches the sources, the per-launch row accounting of the timed
step, the algorithmic work per launch, the clock reader without a GPU, and the batch-invariance
check's slicing and counting (with a CPU stand-in for the forward)."""
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


class _RowwiseForward:
    """CPU stand-in for rz_token_logprobs with the same slicing contract; `batch_term` makes
    each row's value depend on how many rows share the call (a batch-variant forward)."""

    def __init__(self, batch_term=0.0):
        self.batch_term = batch_term
        self.calls = 0

    def rz_token_logprobs(self, H, W, ids, lp_out=None, workspace=None, stream=None, want_lse=True):
        import torch
        assert H.shape[0] == ids.shape[0] == lp_out.shape[0] and H.shape[1] == W.shape[1]
        z = H.double() @ W.double().T
        lp = z.gather(1, ids.long()[:, None])[:, 0] - torch.logsumexp(z, 1)
        lp_out.copy_((lp + self.batch_term * (H.shape[0] > 1)).float())
        self.calls += 1
        return lp_out, None


def _invariance_case(n, batch_term):
    import torch
    g = torch.Generator()
    g.manual_seed(0)
    H = torch.randn(n, 16, generator=g).to(torch.bfloat16)
    W = torch.randn(40, 16, generator=g).to(torch.bfloat16)
    ids = torch.randint(0, 40, (n,), generator=g, dtype=torch.int32)
    fwd = _RowwiseForward(batch_term)
    lp_step = torch.empty(n)
    fwd.rz_token_logprobs(H, W, ids, lp_out=lp_step)
    return fwd, bench.run_batch_invariance(fwd, torch, torch.device("cpu"), None, H, W, ids, lp_step, None, seed=5,
                                           n_alone=20, window=300)


@pytest.mark.parametrize("n", [1000, 130])
def test_batch_invariance_check_reports_zero_for_a_rowwise_forward(n):
    fwd, inv = _invariance_case(n, 0.0)
    assert inv["diff"] == 0 and set(inv["rows_differing"].values()) == {0}
    w = min(n, 300)
    assert inv["rows_checked"] == {"alone": 20, "chunks": 3 * w, "permuted": n}
    # 20 single rows, the window in chunks of 64 / 512 / 2048, one permuted batch (plus the step)
    assert fwd.calls == 1 + 20 + sum(-(-w // c) for c in (64, 512, 2048)) + 1


def test_batch_invariance_check_counts_rows_of_a_batch_variant_forward():
    n = 1000
    _, inv = _invariance_case(n, 0.5)
    # computed alone, a row loses the batch term and differs; every batched row keeps it
    assert inv["rows_differing"]["alone"] == 20
    assert inv["rows_differing"]["chunks_64"] == 0 and inv["rows_differing"]["permuted"] == 0
    assert inv["diff"] == 20


@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_data_parallel_shards_cover_the_batch_in_whole_groups(world):
    import numpy as np
    import workloads as wl
    seg = wl.draw_segments("qwen3_4b")
    lo, resp = 0, 0
    for rank in range(world):
        sh, rewards, n_total = bench.dp_shard(seg, world, rank)
        assert n_total == seg.n_resp  # every rank's N is the whole batch's response count
        assert sh["tok_lo"] == lo and sh["resp_lo"] == resp
        assert np.array_equal(rewards, seg.rewards[sh["resp_lo"]:sh["resp_hi"]])
        gid = seg.group_ids[sh["resp_lo"]:sh["resp_hi"]]
        # whole groups: no group is split between two ranks
        assert sh["resp_lo"] == 0 or seg.group_ids[sh["resp_lo"] - 1] != gid[0]
        assert sh["resp_hi"] == seg.n_resp or seg.group_ids[sh["resp_hi"]] != gid[-1]
        assert sh["seg_offsets"][0] == 0 and sh["seg_offsets"][-1] == sh["tok_hi"] - sh["tok_lo"]
        lo, resp = sh["tok_hi"], sh["resp_hi"]
    assert lo == seg.n_tok and resp == seg.n_resp


def _fake_result():
    kern = {"lmhead_lse": {"launches": 23, "ms_per_step": 261.123456, "share": 0.34, "tflops": 1075.0,
                           "frac_of_peak": 0.7691234}}
    ls = {"frac": 0.72, "variant_clip_mask": {"frac": 0.67}, "ratio_stats": {"frac": 0.62}, "sm_mhz": 1252.0}
    return dict(cfg={"lengths": ("loguniform", 128, 2048)}, peak=1400.0, achieved=1075.0, d=2560, V=151936,
                n_tok=360896, G=64, R=512, value=468908.2, ms_per_step=769.6, dominant="lmhead_lse",
                traffic=None, peak_src="fallback", clocks={"sm_mhz": 1155.0}, launches=2820,
                e2e={"value": 4.4e5}, kernels=kern, invariance={"diff": 0}, loss_stage=ls, fwd_tok_s=1.5e6,
                fwd_ms=240.0, fwd8_ms=160.0, fwd4_ms=100.0, workloads={"lag64_1437610_tok": {"fwd_bwd_tok_s": 4.6e5}})


def test_line_puts_the_contract_keys_first_and_the_compact_figures_last():
    import argparse
    args = argparse.Namespace(steps=5, warmup=3, workload="qwen3_4b")
    line = bench.make_line(args, 1, _fake_result(), {"value": 8.5})
    keys = list(line)
    assert keys[:13] == ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                         "scaling", "vs_baseline", "dtype", "data", "config"]
    assert keys[-6:] == ["tensor_frac_6dV", "fwd_only", "fwd_only_fp8", "fwd_only_mxfp4", "loss_stage_frac",
                         "workloads"]
    assert line["roofline"]["frac"] == pytest.approx(1075.0 / 1400.0)
    assert line["kernels"]["lmhead_lse"]["frac_of_peak"] == 0.7691  # rounded to 4 significant digits
    # the compact tail fits in the part of the output a log tail keeps
    tail = json.dumps({k: line[k] for k in keys[-6:]})
    assert len(tail) < 1500


def test_dp_line_reports_strong_scaling():
    import argparse
    args = argparse.Namespace(steps=3, warmup=3, workload="qwen3_4b")
    r = dict(value=3.6e6, ms_per_step=100.0, n_tok=360896, shard_tokens=45000, d=2560, V=151936, status_ok=True,
             dW_same_bits_on_all_ranks=True, clocks=None, launches=60, n_resp=512, n_groups=64)
    line = bench.make_dp_line(args, 8, r)
    assert line["scaling"] == "strong" and line["n_gpus"] == 8 and line["dW_same_bits_on_all_ranks"]


def test_first_tokens_cuts_the_batch_at_exactly_n():
    import numpy as np
    import workloads as wl
    seg = wl.draw_segments("moe_head")
    prob = wl.Problem(np.zeros((seg.n_tok, 1), np.uint16), None, np.zeros(seg.n_tok, np.int32), seg, 1, 1)
    for n in (4096, 1 << 20, int(seg.seg_offsets[40])):
        sub, R = bench.first_tokens(prob, n, 16)
        off = sub.seg.seg_offsets
        assert sub.n_tok == n and off[0] == 0 and off[-1] == n and np.all(np.diff(off) >= 1)
        assert np.array_equal(off[:-1], seg.seg_offsets[:R])          # the same response starts
        assert np.array_equal(sub.seg.group_ids, np.arange(R) // 16)   # groups of 16
        assert sub.seg.n_groups == (R + 15) // 16
