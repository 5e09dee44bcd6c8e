"""Benchmark of the REINFORCE Zero logprob / loss / gradient path on B200.

One step = one rz_loss_fwd_bwd call over one batch of the Qwen3-4B-shaped workload
(d=2560, V=151936, 64 groups x 8 responses, lengths log-uniform 128..2048 tokens):
fused LM head + online log-sum-exp forward, the REINFORCE Zero loss stage, and the
backward (dZ chunks, dH, dW).  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl rz|reference] [--workload NAME]

--impl reference times the fp64 CPU oracle (the only reference this path has) on host
cores over a bounded sample of the same workload.  With N > 1 (torchrun) every rank runs
an independent replica (the path does not shard); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fwd+bwd logprob/loss tokens/s on 1 B200, % BF16 tensor peak, batch-invariance diff=0"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="rz", choices=["rz", "reference"])
    ap.add_argument("--workload", default="qwen3_4b")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-loss-stage", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other synthetic workloads (invariance head, lag64, moe_head at 2^20 tokens)")
    ap.add_argument("--sweep", action="store_true",
                    help="tokens-per-call sweep 2^12..2^20 of the workload (forward and forward+backward)")
    ap.add_argument("--dp", action="store_true",
                    help="data-parallel step: the one batch split into whole groups across the ranks, dW and the "
                         "loss summed with the deterministic all-reduce (strong scaling)")
    ap.add_argument("--n-tok-cap", type=int, default=None,
                    help="keep only the leading whole groups that fit (small profiling cases)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- clocks

class NvmlClock:
    """Median SM clock over a short timed region: NVML reads every 5 ms from a thread (reads
    only; nothing is set).  None where NVML is unavailable."""

    def __init__(self, device_index: int):
        self.idx = device_index
        self.samples = []
        self._stop = False
        self._thread = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            handle = pynvml.nvmlDeviceGetHandleByIndex(self.idx)
        except Exception:
            return self

        def run():
            while not self._stop:
                try:
                    self.samples.append(pynvml.nvmlDeviceGetClockInfo(handle, pynvml.NVML_CLOCK_SM))
                except Exception:
                    return
                time.sleep(0.005)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop = True
        if self._thread is not None:
            self._thread.join()
        return False

    @property
    def sm_mhz(self):
        return float(np.median(self.samples)) if self.samples else None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.idx)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- ranks

def max_over_ranks(value: float, device=None) -> float:
    """The largest value over all ranks of the default process group (the job's time)."""
    import torch
    import torch.distributed as tdist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank processes its own replica batch each step."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


# --------------------------------------------------------------------------- rz arm

def algorithmic_flops(kind: str, rows: int, d: int, V: int) -> float:
    """Dense contraction FLOPs of one launch: 2 * rows * d * V for each tensor-core kernel."""
    if kind in ("lmhead_lse", "dh", "dw"):
        return 2.0 * rows * d * V
    return 0.0


def algorithmic_bytes(kind: str, rows: int, d: int, V: int) -> float:
    """HBM bytes of one launch of the memory-bound kernels (per element read + write)."""
    if kind == "dz":  # read e (fp16) and write dZ (bf16) in place over [rows, V padded to 8]
        return 4.0 * rows * (-(-V // 8) * 8)
    return 0.0


def launch_rows(kinds, n_tok, chunk=16384):
    """Rows (tokens) each recorded launch covers, in launch order: the per-chunk launches
    (forward, merge, kappa, dZ, dH, dW) cover one chunk, the rest the whole batch."""
    rows = []
    c0 = -chunk
    for k in kinds:
        if k == "lmhead_lse":
            c0 += chunk
        if k in ("response_coef", "block_first", "loss_final"):
            rows.append(n_tok)
        else:
            rows.append(min(chunk, n_tok - c0))
    return rows


def traffic_for(kernel: str, rows_per_launch: float):
    """DRAM bytes per launch from the committed ncu record (profiles/traffic.json), scaled by
    the rows a launch covers, while the kernel's sources still match the recorded digest."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            rec = json.load(f)
        from invariant_logprobs_reinforce_b200.build import source_digest
        ent = rec.get("kernels", {}).get(kernel)
        if ent is None or ent.get("source_digest") != source_digest(ent.get("family", "gemm")):
            return None
        return ent["bytes_per_row"] * rows_per_launch
    except Exception:
        return None


def run_rz(args, rank, world, local_rank):
    import torch
    import workloads as wl
    import invariant_logprobs_reinforce_b200 as rz
    from invariant_logprobs_reinforce_b200 import build as rzbuild

    rzbuild.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    cfg = wl.CONFIGS[args.workload]
    prob = wl.full_config(args.workload, device=str(dev), n_tok_cap=args.n_tok_cap)
    seg = prob.seg
    n, d, V = prob.n_tok, prob.d, prob.V
    R, G = seg.n_resp, seg.n_groups
    H, W, ids = prob.H, prob.W, prob.ids
    rewards = torch.from_numpy(seg.rewards).to(dev)
    off = torch.from_numpy(seg.seg_offsets).to(dev)
    gid = torch.from_numpy(seg.group_ids).to(dev)

    # recorded rollout logprobs = learner logprobs + the workload's weight-lag noise
    lp0, _ = rz.rz_token_logprobs(H, W, ids)
    torch.cuda.synchronize()
    lp_roll = torch.from_numpy(wl.rollout_logprobs_with_lag(lp0.cpu().numpy(), prob.noise, prob.seed)).to(dev)

    ws = torch.empty(rz.rz_workspace_bytes_loss(n, R, G, d, V), dtype=torch.uint8, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    dH = torch.empty((n, d), dtype=torch.bfloat16, device=dev)
    dW = torch.empty((V, d), dtype=torch.float32, device=dev)
    lp = torch.empty(n, dtype=torch.float32, device=dev)
    kappa = torch.empty(n, dtype=torch.float32, device=dev)
    n_launch = rz.rz_num_launches_loss(n)
    events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * n_launch * (args.steps + 1))]
    for e in events:
        e.record(stream)  # materialise the handles
    torch.cuda.synchronize()

    def step(ev=None):
        if ev is None:
            rz.rz_loss_fwd_bwd(H, W, ids, lp_roll, rewards, off, gid, G, loss=loss, dH=dH, dW=dW, lp_out=lp,
                               kappa_out=kappa, workspace=ws, stream=stream)
            return None
        return rz.rz_loss_fwd_bwd_timed(ev, H, W, ids, lp_roll, rewards, off, gid, G, loss, dH, dW, lp, kappa, ws,
                                        stream=stream)

    for _ in range(args.warmup):
        step()
    code, bits = rz.rz_read_device_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} bits {bits}")

    dist = world > 1
    if dist:
        import torch.distributed as tdist
    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local_rank)
    clocks.start()
    time.sleep(0.5)
    if dist:
        tdist.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    all_kinds = []
    for s in range(args.steps):
        evs = events[2 * n_launch * s:2 * n_launch * (s + 1)]
        kinds = step(evs)
        all_kinds.append((evs, kinds))
    t_end.record(stream)
    torch.cuda.synchronize()
    if dist:
        tdist.barrier()
    clk = clocks.stop()
    ms = t_start.elapsed_time(t_end)
    code, bits = rz.rz_read_device_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} bits {bits}")

    # per-kernel durations from the recorded event pairs
    per = {}
    for evs, kinds in all_kinds:
        names = [rz.KERNEL_KINDS[k] for k in kinds]
        rows = launch_rows(names, n)
        for i, (name, r) in enumerate(zip(names, rows)):
            t = evs[2 * i].elapsed_time(evs[2 * i + 1])
            ent = per.setdefault(name, {"launches": 0, "ms": 0.0, "flops": 0.0, "bytes": 0.0, "rows": 0})
            ent["launches"] += 1
            ent["rows"] += r
            ent["ms"] += t
            ent["flops"] += algorithmic_flops(name, r, d, V)
            ent["bytes"] += algorithmic_bytes(name, r, d, V)
    launches_total = sum(v["launches"] for v in per.values())

    if dist:
        ms = max_over_ranks(ms, dev)

    # forward alone (rz_token_logprobs), same inputs
    lpf = torch.empty(n, dtype=torch.float32, device=dev)
    wsf = torch.empty(rz.rz_workspace_bytes_logprobs(n, d, V), dtype=torch.uint8, device=dev)
    for _ in range(2):
        rz.rz_token_logprobs(H, W, ids, lp_out=lpf, workspace=wsf, stream=stream, want_lse=False)
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    fsteps = max(2, args.steps)
    for _ in range(fsteps):
        rz.rz_token_logprobs(H, W, ids, lp_out=lpf, workspace=wsf, stream=stream, want_lse=False)
    f1.record(stream)
    torch.cuda.synchronize()
    fwd_ms = f0.elapsed_time(f1) / fsteps
    if dist:
        fwd_ms = max_over_ranks(fwd_ms, dev)

    # forward from e4m3 operands (quantised once, outside the timed region)
    H8, hs8 = rz.rz_quantize_rows_e4m3(H)
    W8, ws8 = rz.rz_quantize_rows_e4m3(W)
    lp8 = torch.empty(n, dtype=torch.float32, device=dev)
    for _ in range(2):
        rz.rz_token_logprobs_fp8(H8, hs8, W8, ws8, ids, lp_out=lp8, workspace=wsf, stream=stream, want_lse=False)
    f0.record(stream)
    for _ in range(fsteps):
        rz.rz_token_logprobs_fp8(H8, hs8, W8, ws8, ids, lp_out=lp8, workspace=wsf, stream=stream, want_lse=False)
    f1.record(stream)
    torch.cuda.synchronize()
    fwd8_ms = f0.elapsed_time(f1) / fsteps
    if dist:
        fwd8_ms = max_over_ranks(fwd8_ms, dev)
    del H8, W8

    # forward from MXFP4 operands (quantised once, outside the timed region)
    H4, hs4 = rz.rz_quantize_rows_mxfp4(H)
    W4, ws4 = rz.rz_quantize_rows_mxfp4(W)
    lp4 = torch.empty(n, dtype=torch.float32, device=dev)
    for _ in range(2):
        rz.rz_token_logprobs_mxfp4(H4, hs4, W4, ws4, ids, lp_out=lp4, workspace=wsf, stream=stream, want_lse=False)
    f0.record(stream)
    for _ in range(fsteps):
        rz.rz_token_logprobs_mxfp4(H4, hs4, W4, ws4, ids, lp_out=lp4, workspace=wsf, stream=stream, want_lse=False)
    f1.record(stream)
    torch.cuda.synchronize()
    fwd4_ms = f0.elapsed_time(f1) / fsteps
    if dist:
        fwd4_ms = max_over_ranks(fwd4_ms, dev)
    del H4, W4, hs4, ws4

    invariance = run_batch_invariance(rz, torch, dev, stream, H, W, ids, lp, wsf, prob.seed)
    if dist:
        invariance["diff"] = int(max_over_ranks(float(invariance["diff"]), dev))

    loss_stage = None
    if not args.no_loss_stage:
        loss_stage = run_loss_stage(rz, torch, dev, stream)

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(rz, torch, dev, stream, H, W, ids, lp_roll, rewards, off, gid, G, n, d, V, args, world)

    peaks, peak_src = load_peaks()
    peak_tflops = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    other = None
    if not args.no_workloads:
        del ws, dH, dW
        torch.cuda.empty_cache()
        other = run_workloads(rz, torch, dev, stream, peak_tflops)
    tens = {k: v for k, v in per.items() if v["flops"] > 0}
    dom = max(tens, key=lambda k: tens[k]["ms"])
    ach = tens[dom]["flops"] / (tens[dom]["ms"] * 1e-3) / 1e12
    kernels = {}
    for k, v in per.items():
        ent = {"launches": v["launches"] // args.steps, "ms_per_step": v["ms"] / args.steps,
               "share": v["ms"] / sum(x["ms"] for x in per.values())}
        if v["flops"]:
            ent["tflops"] = v["flops"] / (v["ms"] * 1e-3) / 1e12
            ent["frac_of_peak"] = ent["tflops"] / peak_tflops
        if v["bytes"]:
            ent["gbs"] = v["bytes"] / (v["ms"] * 1e-3) / 1e9
            ent["frac_of_hbm"] = ent["gbs"] / peaks["hbm_gbs"]
        kernels[k] = ent
    step_ms = ms / args.steps
    tok_s = job_throughput(n, world, step_ms)
    return dict(
        value=tok_s, ms_per_step=step_ms, n_tok=n, d=d, V=V, R=R, G=G, clocks=clk, kernels=kernels,
        dominant=dom, achieved=ach, peak=peak_tflops, peak_src=peak_src,
        traffic=traffic_for(dom, tens[dom]["rows"] / tens[dom]["launches"]),
        fwd_ms=fwd_ms, fwd_tok_s=world * n / (fwd_ms * 1e-3), launches=launches_total, e2e=e2e, cfg=cfg,
        loss_stage=loss_stage, fwd8_ms=fwd8_ms, fwd4_ms=fwd4_ms, invariance=invariance, workloads=other,
    )


def run_batch_invariance(rz, torch, dev, stream, H, W, ids, lp_step, ws, seed, n_alone=256, window=16384):
    """The metric's "diff = 0", measured on the bench's own batch after the timed region: the
    timed step's lp (from rz_loss_fwd_bwd) against the same rows from rz_token_logprobs
    (a) alone, batch size 1, for n_alone sampled rows; (b) in prefill chunks of 64, 512 and
    2048 rows over a window of the batch; (c) inside a permuted copy of the whole batch.
    Counts the rows whose 32 bits differ anywhere."""
    n = H.shape[0]
    ref = lp_step.view(torch.int32)
    g = torch.Generator()
    g.manual_seed(seed)
    rows = torch.randperm(n, generator=g)[:min(n_alone, n)].sort().values
    lp1 = torch.empty(rows.numel(), dtype=torch.float32, device=dev)
    for j, r in enumerate(rows.tolist()):
        rz.rz_token_logprobs(H[r:r + 1], W, ids[r:r + 1], lp_out=lp1[j:j + 1], workspace=ws, stream=stream,
                             want_lse=False)
    differing = {"alone": int((lp1.view(torch.int32) != ref[rows.to(dev)]).sum())}
    w0 = int(torch.randint(0, max(0, n - window) + 1, (1,), generator=g))
    w1 = min(n, w0 + window)
    lpc = torch.empty(w1 - w0, dtype=torch.float32, device=dev)
    for c in (64, 512, 2048):
        for c0 in range(w0, w1, c):
            c1 = min(w1, c0 + c)
            rz.rz_token_logprobs(H[c0:c1], W, ids[c0:c1], lp_out=lpc[c0 - w0:c1 - w0], workspace=ws, stream=stream,
                                 want_lse=False)
        differing[f"chunks_{c}"] = int((lpc.view(torch.int32) != ref[w0:w1]).sum())
    perm = torch.randperm(n, generator=g).to(dev)
    lpp = torch.empty(n, dtype=torch.float32, device=dev)
    rz.rz_token_logprobs(H[perm].contiguous(), W, ids[perm].contiguous(), lp_out=lpp, workspace=ws, stream=stream,
                         want_lse=False)
    differing["permuted"] = int((lpp.view(torch.int32) != ref[perm]).sum())
    return {"diff": sum(differing.values()), "rows_differing": differing,
            "rows_checked": {"alone": rows.numel(), "chunks": 3 * (w1 - w0), "permuted": n},
            "compared": "bits of the timed step's lp against rz_token_logprobs: rows alone, prefill chunks "
                        f"of 64/512/2048 over rows {w0}..{w1 - 1}, the whole batch permuted"}


def run_loss_stage(rz, torch, dev, stream, n_tok=1 << 26, reps=200):
    """The loss stage alone (rz_segment_loss) at 2^26 tokens with the moe_head response
    shape (lengths U{256..4096}, groups of 16, Bernoulli(0.5) rewards): HBM-bound, 12
    algorithmic bytes per token (read lp and lp_rollout, write kappa) plus 16 per
    response (reward, offset, group id)."""
    import workloads as wl
    cfg = wl.CONFIGS["moe_head"]
    rng = np.random.Generator(np.random.PCG64(cfg["seed"] + 2))
    L = rng.integers(256, 4097, size=n_tok // 256 + 1)
    csum = np.cumsum(L)
    R = int(np.searchsorted(csum, n_tok)) + 1
    L = L[:R].copy()
    L[-1] -= int(csum[R - 1] - n_tok)
    if L[-1] < 1:
        L = L[:-1]
        L[-1] += n_tok - int(L.sum())
    R = len(L)
    off = np.zeros(R + 1, np.int64)
    off[1:] = np.cumsum(L)
    gid = (np.arange(R) // 16).astype(np.int32)
    G = int(gid[-1]) + 1
    rewards = (rng.uniform(size=R) < 0.5).astype(np.float32)
    g = torch.Generator(device=dev)
    g.manual_seed(cfg["seed"] + 3)
    lp = -2.0 * torch.rand(n_tok, generator=g, device=dev) - 0.05
    lr = lp + 0.05 * torch.randn(n_tok, generator=g, device=dev)
    t_r = torch.from_numpy(rewards).to(dev)
    t_off = torch.from_numpy(off).to(dev)
    t_gid = torch.from_numpy(gid).to(dev)
    ws = torch.empty(rz.rz_workspace_bytes_segment_loss(n_tok, R, G), dtype=torch.uint8, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    kappa = torch.empty(n_tok, dtype=torch.float32, device=dev)
    for _ in range(3):
        rz.rz_segment_loss(lp, lr, t_r, t_off, t_gid, G, loss=loss, kappa_out=kappa, workspace=ws, stream=stream)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with NvmlClock(dev.index if dev.index is not None else 0) as clk:
        e0.record(stream)
        for _ in range(reps):
            rz.rz_segment_loss(lp, lr, t_r, t_off, t_gid, G, loss=loss, kappa_out=kappa, workspace=ws,
                               stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    nbytes = 12 * n_tok + 16 * R
    peaks, src = load_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9

    def timed(fn, n_rep):
        for _ in range(3):
            fn()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        with NvmlClock(dev.index if dev.index is not None else 0) as c:
            a.record(stream)
            for _ in range(n_rep):
                fn()
            b.record(stream)
            torch.cuda.synchronize()
        return a.elapsed_time(b) / n_rep, c.sm_mhz

    # the truncated-IS + token-mask variant (adds a 1-byte mask read per token)
    mask = (torch.rand(n_tok, generator=g, device=dev) < 0.9).to(torch.uint8)
    opts = rz.loss_options(clip_max=1.05, token_mask=mask)
    ms_var, _ = timed(lambda: rz.rz_segment_loss_ex(lp, lr, t_r, t_off, t_gid, G, opts, workspace=ws, stream=stream),
                      reps)
    var_bytes = 13 * n_tok + 16 * R
    # ratio diagnostics: three passes over lp and lp_rollout (radix select), 8 B/token each
    ws_st = torch.empty(int(rz.lib().rz_workspace_bytes_ratio_stats(n_tok, R)), dtype=torch.uint8, device=dev)
    ms_st, mhz_st = timed(lambda: rz.rz_ratio_stats(lp, lr, t_off, want_resp_mean=False, workspace=ws_st,
                                                    stream=stream), reps // 2)
    st_bytes = 3 * 8 * n_tok
    hbm = peaks["hbm_gbs"]
    return {"n_tok": n_tok, "n_resp": R, "n_groups": G, "ms_per_call": ms, "algorithmic_bytes": nbytes,
            "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
            "bound": "hbm", "peak_source": f"hbm_gbs of {src}",
            "note": "whole rz_segment_loss call (coefficients, block starts, kappa, loss); inputs 768 MB > L2",
            "sm_mhz": clk.sm_mhz,
            "variant_clip_mask": {"ms_per_call": ms_var, "achieved": var_bytes / (ms_var * 1e-3) / 1e9,
                                  "frac": var_bytes / (ms_var * 1e-3) / 1e9 / hbm},
            "ratio_stats": {"ms_per_call": ms_st, "achieved": st_bytes / (ms_st * 1e-3) / 1e9,
                            "frac": st_bytes / (ms_st * 1e-3) / 1e9 / hbm,
                            "sm_mhz": mhz_st, "note": "3 radix-select passes, 8 B/token each"}}


def run_e2e(rz, torch, dev, stream, H, W, ids, lp_roll, rewards, off, gid, G, n, d, V, args, world=1):
    """The same step through the public calls from host inputs to host results: every input
    copied host -> device and every result (dH, dW, lp, loss) device -> host inside the timed
    region, all host buffers pinned.  W and the small inputs are copied first (the first
    forward needs all of W); rz_loss_fwd_bwd_host_io copies H chunk by chunk on one stream and
    each chunk's dH rows back on another while the next chunk computes, then dW after the
    last chunk; lp and the loss follow."""
    host = {k: t.cpu().pin_memory() for k, t in
            dict(H=H, W=W, ids=ids, lp_roll=lp_roll, rewards=rewards, off=off, gid=gid).items()}
    dbuf = {k: torch.empty_like(t, device=dev) for k, t in host.items()}
    loss_h = torch.empty(1, dtype=torch.float32).pin_memory()
    lp_h = torch.empty(n, dtype=torch.float32).pin_memory()
    dH_h = torch.empty((n, d), dtype=torch.bfloat16).pin_memory()
    dW_h = torch.empty((V, d), dtype=torch.float32).pin_memory()
    R = rewards.shape[0]
    ws = torch.empty(rz.rz_workspace_bytes_loss(n, R, G, d, V), dtype=torch.uint8, device=dev)
    out = dict(loss=torch.empty(1, dtype=torch.float32, device=dev),
               dH=torch.empty((n, d), dtype=torch.bfloat16, device=dev),
               dW=torch.empty((V, d), dtype=torch.float32, device=dev),
               lp=torch.empty(n, dtype=torch.float32, device=dev))

    def step():
        for k in host:
            if k != "H":
                dbuf[k].copy_(host[k], non_blocking=True)
        rz.rz_loss_fwd_bwd_host_io(host["H"], dbuf["H"], dbuf["W"], dbuf["ids"], dbuf["lp_roll"], dbuf["rewards"],
                                   dbuf["off"], dbuf["gid"], G, dH_host=dH_h, dW_host=dW_h, out=out, workspace=ws,
                                   stream=stream)
        loss_h.copy_(out["loss"], non_blocking=True)
        lp_h.copy_(out["lp"], non_blocking=True)

    for _ in range(1):
        step()
    torch.cuda.synchronize()
    ok = bool(torch.equal(dW_h.view(torch.int32), out["dW"].cpu().view(torch.int32)))
    steps = max(2, min(args.steps, 3))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    if world > 1:  # every rank copies its own inputs: the job's time is the slowest rank's
        ms = max_over_ranks(ms, dev)
    h2d = world * sum(t.numel() * t.element_size() for t in host.values())
    d2h = world * sum(t.numel() * t.element_size() for t in (loss_h, lp_h, dH_h, dW_h))
    return {"value": world * n / (ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": ms, "host_results_equal_device": ok,
            "bytes_note": "summed over all ranks; in: H, W, ids, lp_rollout, rewards, offsets, group ids; "
                          "out: dH, dW, lp, loss"}


def first_tokens(prob, n, group_size):
    """The problem cut to its first n tokens: the responses that start before token n, the
    last one shortened to end at n, in groups of `group_size` consecutive responses (the last
    possibly partial).  Returns (problem, n_resp)."""
    import workloads as wl
    seg = prob.seg
    R = int(np.searchsorted(seg.seg_offsets, n, side="left"))
    off = seg.seg_offsets[:R + 1].copy()
    off[-1] = n
    gid = (np.arange(R) // group_size).astype(np.int32)
    G = int(gid[-1]) + 1
    sub = wl.Segments(off, gid, seg.rewards[:R].copy(), G)
    return wl.Problem(prob.H[:n], prob.W, prob.ids[:n], sub, prob.d, prob.V, prob.noise, prob.seed), R


def _time_calls(torch, stream, fn, reps, warm=1):
    """Mean milliseconds per call of fn() over `reps` calls (CUDA events on `stream`)."""
    for _ in range(warm):
        fn()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def run_workloads(rz, torch, dev, stream, peak_tflops):
    """The other synthetic workloads, each through the same public calls as the headline:
    - invariance (d=1536, V=151936): the forward over its 4096 rows in one call, and the
      decode-shaped calls of 1 and 64 rows it is also checked with (microseconds per call);
    - lag64 (d=2560, V=151936, 256 responses of 1K-16K tokens, all ~1.44M tokens): forward
      alone and forward + loss + backward;
    - moe_head (d=7168, V=129280) at 2^20 tokens (the largest call of its sweep): the same.
    Tensor fractions are against the sustained bf16 peak: 2dV FLOP per token forward, 6dV
    forward + loss + backward."""
    import workloads as wl
    res = {}
    cfg = wl.CONFIGS["invariance"]
    d, V = cfg["d"], cfg["V"]
    H, W = wl.draw_matrices(cfg["n_rows"], d, V, cfg["seed"], device=str(dev))
    ids = torch.from_numpy(wl.draw_uniform_ids(cfg["n_rows"], V, cfg["seed"])).to(dev)
    n = H.shape[0]
    lp = torch.empty(n, dtype=torch.float32, device=dev)
    ws = torch.empty(rz.rz_workspace_bytes_logprobs(n, d, V), dtype=torch.uint8, device=dev)
    ms = _time_calls(torch, stream, lambda: rz.rz_token_logprobs(H, W, ids, lp_out=lp, workspace=ws, stream=stream,
                                                                  want_lse=False), 20, 3)
    ent = {"fwd_tok_s": n / (ms * 1e-3), "fwd_frac": n * 2 * d * V / (ms * 1e-3) / (peak_tflops * 1e12)}
    for rows in (1, 64):
        ms_r = _time_calls(torch, stream, lambda: rz.rz_token_logprobs(
            H[:rows], W, ids[:rows], lp_out=lp[:rows], workspace=ws, stream=stream, want_lse=False), 50, 3)
        ent[f"us_per_call_{rows}_rows"] = ms_r * 1e3
    res["invariance_d1536"] = ent
    del H, W, ids, lp, ws

    for name, cap in (("lag64", None), ("moe_head", 1 << 20)):
        prob = wl.full_config(name, device=str(dev), n_tok_cap=None if cap is None else cap + (1 << 17))
        if cap is not None:  # exactly `cap` tokens: the responses up to it, the last one cut short
            prob, _ = first_tokens(prob, cap, wl.CONFIGS[name]["group_size"])
        seg = prob.seg
        n, d, V = prob.n_tok, prob.d, prob.V
        lp0, _ = rz.rz_token_logprobs(prob.H, prob.W, prob.ids, want_lse=False)
        torch.cuda.synchronize()
        lr = torch.from_numpy(wl.rollout_logprobs_with_lag(lp0.cpu().numpy(), prob.noise, prob.seed)).to(dev)
        t_r = torch.from_numpy(seg.rewards).to(dev)
        t_off = torch.from_numpy(seg.seg_offsets).to(dev)
        t_gid = torch.from_numpy(seg.group_ids).to(dev)
        out = dict(loss=torch.empty(1, device=dev), dH=torch.empty((n, d), dtype=torch.bfloat16, device=dev),
                   dW=torch.empty((V, d), dtype=torch.float32, device=dev))
        ws = torch.empty(rz.rz_workspace_bytes_loss(n, seg.n_resp, seg.n_groups, d, V), dtype=torch.uint8,
                         device=dev)
        wsf = torch.empty(rz.rz_workspace_bytes_logprobs(n, d, V), dtype=torch.uint8, device=dev)
        ms_f = _time_calls(torch, stream, lambda: rz.rz_token_logprobs(prob.H, prob.W, prob.ids, lp_out=lp0,
                                                                        workspace=wsf, stream=stream,
                                                                        want_lse=False), 2)
        ms_b = _time_calls(torch, stream, lambda: rz.rz_loss_fwd_bwd(
            prob.H, prob.W, prob.ids, lr, t_r, t_off, t_gid, seg.n_groups, loss=out["loss"], dH=out["dH"],
            dW=out["dW"], want_lp=False, want_kappa=False, workspace=ws, stream=stream), 2)
        code, _ = rz.rz_read_device_status(ws)
        res[f"{name}_{n}_tok"] = {
            "d": d, "V": V, "n_resp": seg.n_resp, "status_ok": code == 0,
            "fwd_tok_s": n / (ms_f * 1e-3), "fwd_frac": n * 2 * d * V / (ms_f * 1e-3) / (peak_tflops * 1e12),
            "fwd_bwd_tok_s": n / (ms_b * 1e-3),
            "fwd_bwd_frac_6dV": n * 6 * d * V / (ms_b * 1e-3) / (peak_tflops * 1e12)}
        del prob, lr, out, ws, wsf, lp0
        torch.cuda.empty_cache()
    return res


def dp_shard(seg, world: int, rank: int):
    """This rank's part of the batch for the data-parallel mode: whole groups balanced by
    tokens (dp.shard_groups), with the global response count every rank's N must use."""
    from invariant_logprobs_reinforce_b200 import dp
    sh = dp.shard_groups(seg.seg_offsets, seg.group_ids, world)[rank]
    rewards = seg.rewards[sh["resp_lo"]:sh["resp_hi"]].copy()
    return sh, rewards, seg.n_resp


def run_dp(args, rank, world, local_rank):
    """The data-parallel step over one batch of the workload: rank r takes its shard of whole
    groups and runs dp.dp_loss_fwd_bwd (the shard through rz_loss_fwd_bwd_ex with N = the
    global response count, then the deterministic all-reduce of dW and the loss: all-to-all,
    rank-order fp64 sum in librz, all-gather).  Timed on the device, max over ranks; value =
    the batch's tokens / that time.  Also checks that every rank ends with the same dW bits."""
    import torch
    import torch.distributed as tdist
    import workloads as wl
    import invariant_logprobs_reinforce_b200 as rz
    from invariant_logprobs_reinforce_b200 import build as rzbuild
    from invariant_logprobs_reinforce_b200 import dp
    rzbuild.build()
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    prob = wl.full_config(args.workload, device=str(dev), n_tok_cap=args.n_tok_cap)
    seg = prob.seg
    d, V = prob.d, prob.V
    lp0, _ = rz.rz_token_logprobs(prob.H, prob.W, prob.ids, want_lse=False)
    torch.cuda.synchronize()
    lr_all = torch.from_numpy(wl.rollout_logprobs_with_lag(lp0.cpu().numpy(), prob.noise, prob.seed)).to(dev)
    sh, rewards, n_total = dp_shard(seg, world, rank)
    t0, t1 = sh["tok_lo"], sh["tok_hi"]
    H, ids, lr = prob.H[t0:t1].contiguous(), prob.ids[t0:t1].contiguous(), lr_all[t0:t1].contiguous()
    t_r = torch.from_numpy(rewards).to(dev)
    t_off = torch.from_numpy(sh["seg_offsets"]).to(dev)
    t_gid = torch.from_numpy(sh["group_ids"]).to(dev)
    n = t1 - t0
    ws = torch.empty(rz.rz_workspace_bytes_loss(n, rewards.shape[0], sh["n_groups"], d, V), dtype=torch.uint8,
                     device=dev)

    def step():
        return dp.dp_loss_fwd_bwd(H, prob.W, ids, lr, t_r, t_off, t_gid, sh["n_groups"], workspace=ws,
                                  n_resp_total=n_total)

    for _ in range(args.warmup):
        out = step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.5)
    tdist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        out = step()
    e1.record(stream)
    torch.cuda.synchronize()
    tdist.barrier()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), dev) / args.steps
    code, bits = rz.rz_read_device_status(ws)
    # the same dW bits on every rank: compare a checksum of the bit patterns
    csum = torch.tensor([int(out["dW"].view(torch.int32).to(torch.int64).sum().item()),
                         int(out["loss"].view(torch.int32).item())], dtype=torch.int64, device=dev)
    allsums = [torch.empty_like(csum) for _ in range(world)]
    tdist.all_gather(allsums, csum)
    same = all(torch.equal(allsums[0], x) for x in allsums)
    launches = rz.rz_num_launches_loss(n) + 2  # + the rank-order sums of dW and the loss
    return dict(value=seg.n_tok / (ms * 1e-3), ms_per_step=ms, n_tok=seg.n_tok, shard_tokens=n, d=d, V=V,
                status_ok=code == 0 and bits == 0, dW_same_bits_on_all_ranks=same, clocks=clk,
                launches=int(max_over_ranks(float(launches * args.steps), dev)), n_resp=seg.n_resp,
                n_groups=seg.n_groups)


# --------------------------------------------------------------------------- sweep

def run_sweep(args, local_rank):
    """Tokens per call 2^12 .. 2^20 over one generated batch of the workload: forward alone
    and forward + loss + backward, tokens/s and fraction of the sustained bf16 peak."""
    import torch
    import workloads as wl
    import invariant_logprobs_reinforce_b200 as rz
    from invariant_logprobs_reinforce_b200 import build as rzbuild
    rzbuild.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    # a little more than 2^20 tokens in whole groups, so that the 2^20 point exists
    prob = wl.full_config(args.workload, device=str(dev), n_tok_cap=args.n_tok_cap or ((1 << 20) + (1 << 17)))
    seg = prob.seg
    d, V = prob.d, prob.V
    peaks, src = load_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    lp_all, _ = rz.rz_token_logprobs(prob.H, prob.W, prob.ids)
    torch.cuda.synchronize()
    lr_all = torch.from_numpy(wl.rollout_logprobs_with_lag(lp_all.cpu().numpy(), prob.noise, prob.seed)).to(dev)
    points = []
    for e in range(12, 21):
        n = 1 << e
        if n > prob.n_tok:
            break
        # whole responses up to n tokens (the last one truncated), one group per 16 responses
        R = int(np.searchsorted(seg.seg_offsets, n, side="left"))
        off = seg.seg_offsets[:R + 1].copy()
        off[-1] = n
        if off[-2] == n:
            off = off[:-1]
            R -= 1
        gid = (np.arange(R) // 16).astype(np.int32)
        G = int(gid[-1]) + 1
        H, ids = prob.H[:n], prob.ids[:n]
        t_off = torch.from_numpy(off).to(dev)
        t_gid = torch.from_numpy(gid).to(dev)
        t_r = torch.from_numpy(seg.rewards[:R].copy()).to(dev)
        ws = torch.empty(rz.rz_workspace_bytes_loss(n, R, G, d, V), dtype=torch.uint8, device=dev)
        wsf = torch.empty(rz.rz_workspace_bytes_logprobs(n, d, V), dtype=torch.uint8, device=dev)
        lp = torch.empty(n, dtype=torch.float32, device=dev)
        out = dict(loss=torch.empty(1, device=dev), dH=torch.empty((n, d), dtype=torch.bfloat16, device=dev),
                   dW=torch.empty((V, d), dtype=torch.float32, device=dev))

        def fwd():
            rz.rz_token_logprobs(H, prob.W, ids, lp_out=lp, workspace=wsf, stream=stream, want_lse=False)

        def step():
            rz.rz_loss_fwd_bwd(H, prob.W, ids, lr_all[:n], t_r, t_off, t_gid, G, loss=out["loss"], dH=out["dH"],
                               dW=out["dW"], want_lp=False, want_kappa=False, workspace=ws, stream=stream)

        res = {"n_tok": n, "n_resp": R}
        for name, fn, flops in (("fwd", fwd, 2.0), ("fwd_bwd", step, 6.0)):
            reps = max(2, min(20, int(2e15 / (flops * n * d * V)) + 1))
            for _ in range(2):
                fn()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                fn()
            b.record(stream)
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / reps
            res[name] = {"ms": ms, "tokens_per_s": n / (ms * 1e-3),
                         "tensor_frac": n * flops * d * V / (ms * 1e-3) / (peak * 1e12)}
        points.append(res)
        del ws, wsf, out
    return {"workload": args.workload, "d": d, "V": V, "peak_tflops": peak, "peak_source": src, "points": points}


# --------------------------------------------------------------------------- CPU oracle

def cpu_oracle_sample(workload: str, budget_s: float = 15.0):
    """The fp64 oracle as it stands, fwd+loss+bwd on a bounded sub-batch of the workload's
    shape (one group of two responses of k/2 tokens each, the workload's d and V)."""
    import oracle
    import workloads as wl
    oracle.build()
    cfg = wl.CONFIGS[workload]
    d, V = cfg["d"], cfg["V"]
    rng = np.random.Generator(np.random.PCG64(cfg["seed"] + 1))
    W = wl.bf16_bits(rng.standard_normal((V, d), dtype=np.float32) * np.float32(1.0 / math.sqrt(d)))

    def run(k):
        H = wl.bf16_bits(rng.standard_normal((k, d), dtype=np.float32))
        ids = rng.integers(0, V, size=k).astype(np.int32)
        off = np.array([0, k // 2, k], np.int64)
        lr = np.full(k, -12.0)
        t0 = time.perf_counter()
        oracle.loss_fwd_bwd(H, W, ids, lr, np.array([1.0, 0.0]), off, np.zeros(2, np.int32), 1)
        return time.perf_counter() - t0

    k = 4
    t = run(k)
    k2 = int(max(2, min(512, 2 * round(0.5 * k * budget_s / max(t, 1e-3)))))
    t2 = run(k2)
    return {"value": k2 / t2, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "cpu_model": host_cpu_model(), "host_cpus": os.cpu_count(),
            "sample": f"{k2} tokens of {workload} (2 responses x {k2 // 2} tokens, d={d}, V={V}): "
                      f"fp64 lp, loss, dH and dW; {t2:.1f} s"}


def host_cpu_model() -> str:
    """The host CPU's model name (/proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import workloads as wl
    cfg = wl.CONFIGS[args.workload]
    budget = max(3.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    vals = []
    last = None
    for i in range(args.warmup + args.steps):
        last = cpu_oracle_sample(args.workload, budget_s=budget)
        if i >= args.warmup:
            vals.append(last["value"])
    v = float(np.mean(vals)) if vals else float(last["value"])
    seg = wl.draw_segments(args.workload)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": seg.n_tok / v * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.workload}: d={cfg['d']}, V={cfg['V']}, n_tok={seg.n_tok}, "
                               f"n_resp={seg.n_resp} (timed on a bounded token sample; tokens/s extrapolates "
                               f"linearly, the cost is row-linear)"},
        "cpu_baseline": dict(last, value=v),
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def _round(x, sig=4):
    """Floats rounded to `sig` significant digits (nested), to keep the line short."""
    if isinstance(x, float):
        return float(f"{x:.{sig}g}") if math.isfinite(x) else x
    if isinstance(x, dict):
        return {k: _round(v, sig) for k, v in x.items()}
    if isinstance(x, (list, tuple)):
        return [_round(v, sig) for v in x]
    return x


def make_line(args, world, res, cpu):
    """The JSON line: the contract's keys first, the detailed records next, and the compact
    headline figures last (a consumer that keeps only the end of the output still has them)."""
    cfg = res["cfg"]
    peak = res["peak"]
    frac = res["achieved"] / peak
    d, V, n = res["d"], res["V"], res["n_tok"]
    line = {
        "metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": f"{args.workload}: d={d}, V={V}, {res['G']} groups x {res['R'] // res['G']} responses, "
                        f"lengths {cfg['lengths'][0]} {cfg['lengths'][1]}-{cfg['lengths'][2]}, n_tok={n} per GPU",
            "n_tok": n, "d": d, "V": V, "n_resp": res["R"], "n_groups": res["G"],
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "inputs larger than L2 (H %.2f GB, W %.2f GB)" % (n * d * 2 / 1e9, V * d * 2 / 1e9),
        },
        "roofline": {"bound": "tensor", "kernel": res["dominant"], "achieved": res["achieved"], "peak": peak,
                     "unit": "TFLOP/s", "frac": frac, "traffic": res["traffic"],
                     "peak_source": f"bf16_tflops_sustained of {res['peak_src']}"},
        "clocks": res["clocks"],
        "gpu_launches": res["launches"],
        "e2e": res["e2e"],
        "cpu_baseline": cpu,
        # detailed records
        "kernels": _round(res["kernels"]),
        "batch_invariance": res["invariance"],
        "loss_stage": _round(res["loss_stage"]),
        # compact headline figures, last
        "tensor_frac_6dV": _round(res["value"] / world * 6 * d * V / (peak * 1e12)),
        "fwd_only": _round({"tokens_per_s": res["fwd_tok_s"], "ms_per_step": res["fwd_ms"],
                            "tensor_frac_2dV": res["fwd_tok_s"] / world * 2 * d * V / (peak * 1e12)}),
        "fwd_only_fp8": _round({"tokens_per_s": n * world / (res["fwd8_ms"] * 1e-3), "ms_per_step": res["fwd8_ms"],
                                "tensor_frac_2dV": n * 2 * d * V / (res["fwd8_ms"] * 1e-3) / (2 * peak * 1e12),
                                "peak": "2 x sustained bf16 (nominal e4m3 ratio)"}),
        "fwd_only_mxfp4": _round({"tokens_per_s": n * world / (res["fwd4_ms"] * 1e-3), "ms_per_step": res["fwd4_ms"],
                                  "tensor_frac_2dV": n * 2 * d * V / (res["fwd4_ms"] * 1e-3) / (4 * peak * 1e12),
                                  "peak": "4 x sustained bf16 (nominal dense fp4 ratio)"}),
    }
    ls = res["loss_stage"]
    if ls is not None:
        line["loss_stage_frac"] = _round({"segment_loss": ls["frac"], "clip_mask": ls["variant_clip_mask"]["frac"],
                                          "ratio_stats": ls["ratio_stats"]["frac"], "sm_mhz": ls["sm_mhz"]})
    line["workloads"] = _round(res["workloads"])
    return line


def make_dp_line(args, world, r):
    """The JSON line of the data-parallel mode (strong scaling over one fixed batch)."""
    return {
        "metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{args.workload}: d={r['d']}, V={r['V']}, {r['n_resp']} responses in "
                               f"{r['n_groups']} groups, n_tok={r['n_tok']} for the whole job",
                   "parallelism": f"data-parallel x{world}: whole groups per rank, dW and loss summed by a "
                                  f"deterministic all-reduce (all-to-all, rank-order fp64 sum, all-gather)",
                   "shard_tokens_rank0": r["shard_tokens"]},
        "clocks": r["clocks"], "gpu_launches": r["launches"], "status_ok": r["status_ok"],
        "dW_same_bits_on_all_ranks": r["dW_same_bits_on_all_ranks"],
        "roofline": None, "e2e": None, "cpu_baseline": None,
        "note": "the data-parallel mode reports throughput and cross-rank consistency; the default mode "
                "carries the roofline, e2e and cpu_baseline",
    }


def free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


# --------------------------------------------------------------------------- main

def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0

    if args.sweep:
        if rank == 0:
            print(json.dumps({"sweep": run_sweep(args, local_rank)}), flush=True)
        return 0

    if world > 1 or args.dp:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        if world == 1:  # a one-rank group for the data-parallel mode on one GPU
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", str(free_port()))
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                 device_id=torch.device("cuda", local_rank))
    if args.dp:
        r = run_dp(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(make_dp_line(args, world, r)), flush=True)
        import torch.distributed as tdist
        tdist.barrier()
        tdist.destroy_process_group()
        return 0
    res = run_rz(args, rank, world, local_rank)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(args.workload)
    if rank == 0:
        print(json.dumps(make_line(args, world, res, cpu)), flush=True)
    if world > 1:
        import torch.distributed as tdist
        tdist.barrier()
        tdist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
