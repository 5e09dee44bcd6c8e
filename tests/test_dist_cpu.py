"""The multi-rank plumbing on CPU (gloo): bench.py's job time is the maximum over ranks,
throughput counts every rank's replica, and the reference arm under torchrun prints one
line from rank 0 while the other ranks exit 0 without work; the deterministic all-reduce's
orchestration; and the data-parallel step's decomposition (whole-group shards, N = the
global response count, rank-order sums) against the full batch at world sizes 2 and 3."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = bench.max_over_ranks(10.0 + 5.0 * rank)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_throughput():
    sys.path.insert(0, ROOT)
    import bench
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
        assert dict(out) == {0: 15.0, 1: 15.0}
    assert bench.job_throughput(1000, 2, 500.0) == pytest.approx(4000.0)


def _dar_worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch
    from invariant_logprobs_reinforce_b200 import dp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(100 + rank)
        x = (torch.randn(1001, generator=g) * 10 ** torch.randn(1001, generator=g)).float()  # 1001: uneven slices

        def rank_order_sum(stacked):  # the librz kernel's arithmetic (fp64, rank order), for CPU ranks
            acc = torch.zeros(stacked.shape[1], dtype=torch.float64)
            for r in range(stacked.shape[0]):
                acc += stacked[r].double()
            return acc.float()

        y = dp.deterministic_all_reduce(x, sum_shards=rank_order_sum)
        out[rank] = (x.numpy().tobytes(), y.numpy().tobytes())
    finally:
        dist.destroy_process_group()


def test_deterministic_all_reduce_orchestration():
    """all-to-all of slices, rank-order sum, all-gather: the same bits on every rank,
    equal to the rank-order fp64 sum of the inputs."""
    import numpy as np
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_dar_worker, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    x0 = np.frombuffer(res[0][0], np.float32)
    x1 = np.frombuffer(res[1][0], np.float32)
    y0 = np.frombuffer(res[0][1], np.float32)
    y1 = np.frombuffer(res[1][1], np.float32)
    assert y0.tobytes() == y1.tobytes()
    ref = (x0.astype(np.float64) + x1.astype(np.float64)).astype(np.float32)
    assert np.array_equal(y0.view(np.uint32), ref.view(np.uint32))


def test_reference_arm_under_torchrun_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "tiny"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["value"] > 0 and rec["unit"] == "tokens/s"
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["e2e"]["h2d_bytes_per_step"] == 0


def _dp_problem():
    import oracle
    import workloads as wl
    p = wl.custom(6, 3, ("uniform", 5, 12), 64, 300, seed=404)
    lp, _ = oracle.token_logprobs(p.H, p.W, p.ids)
    lr = wl.rollout_logprobs_with_lag(lp, ("normal", 0.05), p.seed).astype("float64")
    return p, lr


def _dp_worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import oracle
    from invariant_logprobs_reinforce_b200 import dp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        p, lr = _dp_problem()
        s = dp.shard_groups(p.seg.seg_offsets, p.seg.group_ids, world)[rank]
        t0, t1, r0, r1 = s["tok_lo"], s["tok_hi"], s["resp_lo"], s["resp_hi"]

        def shard_step(H, W, ids, lp_rollout, rewards, seg_offsets, group_ids, n_groups, opts, workspace=None):
            # the oracle in place of the GPU call (CPU ranks have no GPU); same N as the kernels get
            lp, lse = oracle.token_logprobs(H, W, ids)
            loss, _, kappa = oracle.loss_from_lp_ex(lp, lp_rollout, rewards.numpy(), seg_offsets, group_ids, n_groups,
                                                    n_resp_total=opts.n_resp_total)
            return dict(loss=torch.tensor([loss], dtype=torch.float32),
                        dW=torch.from_numpy(oracle.dw_rows(H, W, ids, lse, kappa)).float(),
                        dH=oracle.dh_rows(H, W, ids, None, lse, kappa))

        def rank_order_sum(stacked):
            acc = torch.zeros(stacked.shape[1], dtype=torch.float64)
            for r in range(stacked.shape[0]):
                acc += stacked[r].double()
            return acc.float()

        dp.rz_loss_fwd_bwd_ex = shard_step
        res = dp.dp_loss_fwd_bwd(p.H[t0:t1], p.W, p.ids[t0:t1], lr[t0:t1], torch.from_numpy(p.seg.rewards[r0:r1]),
                                 s["seg_offsets"], s["group_ids"], s["n_groups"], sum_shards=rank_order_sum)
        out[rank] = (res["loss"].numpy().tobytes(), res["dW"].numpy().tobytes(), res["dH"], t0, t1)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_data_parallel_step_equals_the_full_batch(world):
    """Whole groups per rank, N = the global response count, dW and the loss summed in rank
    order: every rank holds the same bits, equal to the full batch's loss and dW up to the
    fp32 rounding of each shard, and each rank's dH rows are the full batch's rows."""
    import numpy as np
    import oracle
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_dp_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert len({res[r][0] for r in res}) == 1 and len({res[r][1] for r in res}) == 1
    p, lr = _dp_problem()
    ref = oracle.loss_fwd_bwd(p.H, p.W, p.ids, lr, p.seg.rewards, p.seg.seg_offsets, p.seg.group_ids, p.seg.n_groups)
    loss = float(np.frombuffer(res[0][0], np.float32)[0])
    scale = np.abs(ref["kappa"]).sum()
    assert abs(loss - ref["loss"]) <= 1e-6 * max(abs(ref["loss"]), scale)
    dW = np.frombuffer(res[0][1], np.float32).reshape(ref["dW"].shape).astype(np.float64)
    assert np.linalg.norm(dW - ref["dW"]) <= 1e-6 * np.linalg.norm(ref["dW"])
    covered = 0
    for r in range(world):
        dH, t0, t1 = res[r][2], res[r][3], res[r][4]
        assert np.abs(dH - ref["dH"][t0:t1]).max() <= 1e-12 * np.abs(ref["dH"]).max()
        covered += t1 - t0
    assert covered == p.n_tok
    # control: with each shard's own response count as N the shards would not add up
    from invariant_logprobs_reinforce_b200 import dp
    local = 0.0
    for s in dp.shard_groups(p.seg.seg_offsets, p.seg.group_ids, world):
        t0, t1, r0, r1 = s["tok_lo"], s["tok_hi"], s["resp_lo"], s["resp_hi"]
        local += oracle.loss_from_lp(ref["lp"][t0:t1], lr[t0:t1], p.seg.rewards[r0:r1], s["seg_offsets"],
                                     s["group_ids"], s["n_groups"])[0]
    assert abs(local - ref["loss"]) > 1e-3 * max(abs(ref["loss"]), scale)


def test_shard_groups_balances_whole_groups():
    import numpy as np
    from invariant_logprobs_reinforce_b200 import dp
    off = np.array([0, 5, 9, 20, 22, 30, 41, 50, 51, 60])
    gid = np.array([0, 0, 3, 3, 1, 1, 7, 7, 2])
    for world in range(1, 6):
        sh = dp.shard_groups(off, gid, world)
        assert [s["tok_lo"] for s in sh][0] == 0 and sh[-1]["tok_hi"] == 60
        for a, b in zip(sh, sh[1:]):
            assert a["tok_hi"] == b["tok_lo"] and a["resp_hi"] == b["resp_lo"]
        for s in sh:
            assert s["resp_hi"] > s["resp_lo"]
            g = gid[s["resp_lo"]:s["resp_hi"]]
            # whole groups only: no group id of this shard appears outside it
            outside = np.r_[gid[:s["resp_lo"]], gid[s["resp_hi"]:]]
            assert not set(g.tolist()) & set(outside.tolist())
            # local ids are 0.. in order of first appearance
            _, first = np.unique(s["group_ids"], return_index=True)
            assert s["group_ids"][np.sort(first)].tolist() == list(range(s["n_groups"]))
            assert s["seg_offsets"][0] == 0 and s["seg_offsets"][-1] == s["tok_hi"] - s["tok_lo"]
    # two shards: the cut closest to half the tokens (30) is at token 22 (not 41)
    assert dp.shard_groups(off, gid, 2)[0]["tok_hi"] == 22
    with pytest.raises(ValueError):
        dp.shard_groups(off, gid, 6)  # five groups
    with pytest.raises(ValueError):
        dp.shard_groups(off, np.array([0, 0, 1, 1, 0, 2, 2, 3, 3]), 2)  # group 0 split in two runs
