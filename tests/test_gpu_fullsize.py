"""Parity at full size, in the launch configuration bench.py times: the Qwen3-4B-shaped
workload (d=2560, V=151936, 512 responses, ~360k tokens, 23 backward chunks), the lag-64
agentic workload (the same head, 256 responses of 1K-16K tokens, ~1.4M tokens, heavy-tailed
Student-t lag) and the MoE-shaped head (d=7168, V=129280) at 2^20 tokens, the largest call
of its throughput sweep.

The oracle cannot recompute all of it in fp64, so it checks sampled outputs one by one
(lp, lse, kappa and dH of sampled token rows) and the rest through properties that hold
at any size: the loss equals the sum of kappa; every column of dW sums to ~0 (each dZ
row sums to zero); the loss call's logprobs equal the forward call's bit for bit.

The recorded rollout logprobs of the sampled rows are the oracle's lp plus the
workload's seeded lag noise, so every oracle input is independent of the CUDA path.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from tests import helpers as h

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rz():
    from invariant_logprobs_reinforce_b200 import build
    build.build()
    import invariant_logprobs_reinforce_b200 as rz
    return rz


@pytest.mark.parametrize("name,cap", [("qwen3_4b", None), ("lag64", None), ("moe_head", 1 << 20)])
def test_full_size_sampled_rows(rz, oracle, name, cap):
    prob = wl.full_config(name, device="cuda", n_tok_cap=cap)
    seg = prob.seg
    n, d, V = prob.n_tok, prob.d, prob.V
    lp0, lse0 = rz.rz_token_logprobs(prob.H, prob.W, prob.ids)
    rng = np.random.default_rng(2024)
    rows = np.sort(np.concatenate([[0, n - 1], rng.choice(n, 10, replace=False)])).astype(np.int64)
    W_bits = prob.W.view(torch.int16).cpu().numpy().view(np.uint16)
    H_rows = prob.H[torch.from_numpy(rows).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
    ids_rows = prob.ids[torch.from_numpy(rows).cuda()].cpu().numpy()
    lp_o, lse_o = oracle.token_logprobs(H_rows, W_bits, ids_rows)

    eps = wl.rollout_logprobs_with_lag(np.zeros(n), prob.noise, prob.seed).astype(np.float64)
    lr = lp0.cpu().numpy().astype(np.float64) + eps
    lr[rows] = lp_o + eps[rows]
    lr = lr.astype(np.float32)
    out = rz.rz_loss_fwd_bwd(prob.H, prob.W, prob.ids, torch.from_numpy(lr).cuda(),
                             torch.from_numpy(seg.rewards).cuda(), torch.from_numpy(seg.seg_offsets).cuda(),
                             torch.from_numpy(seg.group_ids).cuda(), seg.n_groups)
    assert rz.rz_read_device_status(out["workspace"]) == (0, 0)

    # sampled rows against the oracle
    lp_g = out["lp"].cpu().numpy().astype(np.float64)
    assert np.abs(lp_g[rows] - lp_o).max() <= h.LP_ATOL
    assert np.abs(lse0.cpu().numpy()[rows] - lse_o).max() <= h.LP_ATOL
    # oracle kappa of the sampled rows: only their own lp and lp_rollout enter it
    lp_vec = lr.astype(np.float64).copy()
    lp_vec[rows] = lp_o
    _, _, kappa_o = oracle.loss_from_lp(lp_vec, lr.astype(np.float64), seg.rewards, seg.seg_offsets,
                                        seg.group_ids, seg.n_groups)
    kappa_g = out["kappa"].cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(kappa_g[rows], kappa_o[rows], rtol=5e-3, atol=0)
    dh_o = oracle.dh_rows(H_rows, W_bits, ids_rows, None, lse_o, kappa_o[rows])
    dh_g = out["dH"][torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
    assert h.rel_fro(dh_g, dh_o) <= h.GRAD_RFRO, h.rel_fro(dh_g, dh_o)

    # properties of the whole batch
    assert torch.equal(out["lp"].view(torch.int32), lp0.view(torch.int32))
    ksum = float(out["kappa"].double().sum().item())
    kabs = float(out["kappa"].double().abs().sum().item())
    assert abs(out["loss"].item() - ksum) <= 1e-6 * kabs + 1e-7 * abs(ksum)
    dW = out["dW"]
    colsum = dW.double().sum(dim=0).abs()
    colabs = dW.double().abs().sum(dim=0)
    assert torch.all(colsum <= 1e-2 * colabs)
    assert torch.isfinite(dW).all() and torch.isfinite(out["dH"].float()).all()
    del out, dW, lp0, lse0, prob
    torch.cuda.empty_cache()
