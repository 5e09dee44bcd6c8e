"""The multi-rank plumbing of bench.py on CPU (gloo, world size 2): the job's time is the
maximum over ranks, throughput counts every rank's replica, and the reference arm under
torchrun prints one line from rank 0 while the other ranks exit 0 without work."""
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
