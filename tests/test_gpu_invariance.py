"""Batch invariance ("diff = 0") on the 1.5B-shaped head (d=1536, V=151936, bf16).

One fixed set of 4096 token rows; the reference is one call over all of them.  Every
other way of evaluating the same rows must give the same lp and lse BITS: (a) each row
alone (batch size 1, one-token decode calls), (b) inside random batches of 1..1024 rows
with random batch-mates at random positions, (c) permuted, (d) as prefill chunks of
64 / 512 / 2048 rows and mixed chunk + decode sequences; plus the loss entry point and
a second stream.  Following "vLLM Train-Inference Consistency Release Notes"
(agentlenshq.com), section "Achieving Bitwise Consistency" (determinism, batch
independence, phase consistency).
"""
import numpy as np
import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu

N_ROWS, N_POOL = 4096, 2048


@pytest.fixture(scope="module")
def rz():
    from invariant_logprobs_reinforce_b200 import build
    build.build()
    import invariant_logprobs_reinforce_b200 as rz
    return rz


@pytest.fixture(scope="module")
def inv(rz):
    cfg = wl.CONFIGS["invariance"]
    d, V = cfg["d"], cfg["V"]
    H_all, W = wl.draw_matrices(N_ROWS + N_POOL, d, V, cfg["seed"], device="cuda")
    ids_all = torch.from_numpy(wl.draw_uniform_ids(N_ROWS + N_POOL, V, cfg["seed"])).cuda()
    H, pool = H_all[:N_ROWS].contiguous(), H_all[N_ROWS:].contiguous()
    ids, pool_ids = ids_all[:N_ROWS].contiguous(), ids_all[N_ROWS:].contiguous()
    ref_lp, ref_lse = rz.rz_token_logprobs(H, W, ids)
    torch.cuda.synchronize()
    ws = torch.empty(rz.rz_workspace_bytes_logprobs(N_ROWS + N_POOL, d, V), dtype=torch.uint8, device="cuda")
    return dict(H=H, W=W, ids=ids, pool=pool, pool_ids=pool_ids, lp=ref_lp, lse=ref_lse, ws=ws, d=d, V=V)


def _bits_equal(a, b):
    return torch.equal(a.view(torch.int32), b.view(torch.int32))


def _eval(rz, inv, H, ids):
    lp = torch.empty(H.shape[0], device="cuda")
    lse = torch.empty(H.shape[0], device="cuda")
    rz.rz_token_logprobs(H, inv["W"], ids, lp_out=lp, lse_out=lse, workspace=inv["ws"])
    return lp, lse


def test_a_each_row_alone(rz, inv):
    lp = torch.empty(N_ROWS, device="cuda")
    lse = torch.empty(N_ROWS, device="cuda")
    for i in range(N_ROWS):
        rz.rz_token_logprobs(inv["H"][i:i + 1], inv["W"], inv["ids"][i:i + 1], lp_out=lp[i:i + 1],
                             lse_out=lse[i:i + 1], workspace=inv["ws"])
    torch.cuda.synchronize()
    assert _bits_equal(lp, inv["lp"]) and _bits_equal(lse, inv["lse"])


def test_b_random_batches_with_random_batch_mates(rz, inv):
    rng = np.random.default_rng(33)
    for _ in range(3):
        order = rng.permutation(N_ROWS)
        pos = 0
        lp = torch.full((N_ROWS,), float("nan"), device="cuda")
        lse = torch.full((N_ROWS,), float("nan"), device="cuda")
        while pos < N_ROWS:
            size = int(rng.integers(1, 1025))
            own = order[pos:pos + size]
            pos += len(own)
            mates = rng.integers(0, N_POOL, size=int(rng.integers(0, 1025 - len(own))))
            # assemble the batch: own rows and batch-mates at random positions
            src = np.concatenate([own, N_ROWS + mates])
            perm = rng.permutation(len(src))
            src = src[perm]
            Hb = torch.cat([inv["H"], inv["pool"]])[torch.from_numpy(src).cuda()].contiguous()
            ib = torch.cat([inv["ids"], inv["pool_ids"]])[torch.from_numpy(src).cuda()].contiguous()
            blp, blse = _eval(rz, inv, Hb, ib)
            mine = np.nonzero(src < N_ROWS)[0]
            idx = torch.from_numpy(src[mine]).cuda()
            lp[idx] = blp[torch.from_numpy(mine).cuda()]
            lse[idx] = blse[torch.from_numpy(mine).cuda()]
        torch.cuda.synchronize()
        assert _bits_equal(lp, inv["lp"]) and _bits_equal(lse, inv["lse"])


def test_c_permuted(rz, inv):
    perm = torch.from_numpy(np.random.default_rng(7).permutation(N_ROWS)).cuda()
    lp, lse = _eval(rz, inv, inv["H"][perm].contiguous(), inv["ids"][perm].contiguous())
    out_lp = torch.empty_like(lp)
    out_lse = torch.empty_like(lse)
    out_lp[perm] = lp
    out_lse[perm] = lse
    assert _bits_equal(out_lp, inv["lp"]) and _bits_equal(out_lse, inv["lse"])


@pytest.mark.parametrize("chunk", [64, 512, 2048])
def test_d_prefill_chunks(rz, inv, chunk):
    lp = torch.empty(N_ROWS, device="cuda")
    lse = torch.empty(N_ROWS, device="cuda")
    for c0 in range(0, N_ROWS, chunk):
        c1 = min(N_ROWS, c0 + chunk)
        rz.rz_token_logprobs(inv["H"][c0:c1], inv["W"], inv["ids"][c0:c1], lp_out=lp[c0:c1], lse_out=lse[c0:c1],
                             workspace=inv["ws"])
    torch.cuda.synchronize()
    assert _bits_equal(lp, inv["lp"]) and _bits_equal(lse, inv["lse"])


def test_d_mixed_prefill_and_decode(rz, inv):
    rng = np.random.default_rng(5)
    lp = torch.empty(N_ROWS, device="cuda")
    lse = torch.empty(N_ROWS, device="cuda")
    pos = 0
    while pos < N_ROWS:
        # a prefill chunk of random length, then a run of one-token decode calls
        c1 = min(N_ROWS, pos + int(rng.integers(1, 700)))
        rz.rz_token_logprobs(inv["H"][pos:c1], inv["W"], inv["ids"][pos:c1], lp_out=lp[pos:c1], lse_out=lse[pos:c1],
                             workspace=inv["ws"])
        pos = c1
        for _ in range(int(rng.integers(0, 40))):
            if pos >= N_ROWS:
                break
            rz.rz_token_logprobs(inv["H"][pos:pos + 1], inv["W"], inv["ids"][pos:pos + 1], lp_out=lp[pos:pos + 1],
                                 lse_out=lse[pos:pos + 1], workspace=inv["ws"])
            pos += 1
    torch.cuda.synchronize()
    assert _bits_equal(lp, inv["lp"]) and _bits_equal(lse, inv["lse"])


def test_loss_entry_point_and_second_stream(rz, inv):
    off = torch.arange(0, N_ROWS + 1, 512, dtype=torch.int64, device="cuda")
    R = off.numel() - 1
    gid = (torch.arange(R, device="cuda") // 4).to(torch.int32)
    rewards = (torch.arange(R, device="cuda") % 3 == 0).float()
    lr = inv["lp"] - 0.01
    out = rz.rz_loss_fwd_bwd(inv["H"], inv["W"], inv["ids"], lr, rewards, off, gid, int(gid.max().item()) + 1)
    torch.cuda.synchronize()
    assert _bits_equal(out["lp"], inv["lp"])
    side = torch.cuda.Stream()
    ws2 = torch.empty_like(inv["ws"])
    with torch.cuda.stream(side):
        lp2, lse2 = rz.rz_token_logprobs(inv["H"], inv["W"], inv["ids"], workspace=ws2, stream=side)
    lp3, lse3 = _eval(rz, inv, inv["H"], inv["ids"])
    torch.cuda.synchronize()
    assert _bits_equal(lp2, inv["lp"]) and _bits_equal(lse2, inv["lse"])
    assert _bits_equal(lp3, inv["lp"]) and _bits_equal(lse3, inv["lse"])
