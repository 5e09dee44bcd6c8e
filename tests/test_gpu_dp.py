"""Cross-GPU consistency pieces on one GPU: the rank-order shard sum kernel bit for bit,
and a one-rank NCCL data-parallel step equal to the single-GPU call."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import workloads as wl
from tests import helpers as h

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rz():
    from invariant_logprobs_reinforce_b200 import build
    build.build()
    import invariant_logprobs_reinforce_b200 as rz
    return rz


@pytest.mark.parametrize("nshards,count", [(1, 10), (3, 100003), (8, 2 ** 20 + 7)])
def test_sum_shards_is_the_rank_order_fp64_sum(rz, nshards, count):
    g = torch.Generator(device="cuda")
    g.manual_seed(nshards)
    x = torch.randn((nshards, count), generator=g, device="cuda") * torch.exp2(
        torch.randint(-20, 20, (nshards, count), generator=g, device="cuda").float())
    out = rz.rz_sum_shards_f32(x).cpu().numpy()
    xs = x.cpu().numpy().astype(np.float64)
    ref = np.zeros(count, np.float64)
    for r in range(nshards):
        ref += xs[r]
    assert np.array_equal(out.view(np.uint32), ref.astype(np.float32).view(np.uint32))


def test_one_rank_data_parallel_step_equals_the_single_gpu_call(rz):
    from invariant_logprobs_reinforce_b200 import dp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        p = wl.custom(2, 3, ("uniform", 30, 70), 128, 3000, seed=77)
        dev = h.to_device(p)
        lr = torch.full((p.n_tok,), -8.0, device="cuda")
        a = rz.rz_loss_fwd_bwd(dev["H"], dev["W"], dev["ids"], lr, dev["rewards"], dev["seg_offsets"],
                               dev["group_ids"], p.seg.n_groups)
        b = dp.dp_loss_fwd_bwd(dev["H"], dev["W"], dev["ids"], lr, dev["rewards"], dev["seg_offsets"],
                               dev["group_ids"], p.seg.n_groups)
        torch.cuda.synchronize()
        # one rank: the rank-order sum of one shard rounds fp32 -> fp64 -> fp32 exactly
        assert torch.equal(a["dW"].view(torch.int32), b["dW"].view(torch.int32))
        assert torch.equal(a["loss"].view(torch.int32), b["loss"].view(torch.int32))
        assert torch.equal(a["dH"].view(torch.int16), b["dH"].view(torch.int16))
    finally:
        dist.destroy_process_group()


def test_bench_data_parallel_mode_at_world_size_one():
    """bench.py --dp on one GPU: the whole-group shard is the whole (capped) batch, the
    deterministic all-reduce runs through a one-rank NCCL group, and the line reports a
    clean status and the same dW bits on every rank."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_PORT")}
    r = subprocess.run([sys.executable, "bench.py", "--dp", "--steps", "2", "--warmup", "1", "--n-tok-cap", "20000"],
                       cwd=root, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["scaling"] == "strong" and line["n_gpus"] == 1
    assert line["status_ok"] and line["dW_same_bits_on_all_ranks"]
    assert line["value"] > 0 and line["gpu_launches"] > 0
