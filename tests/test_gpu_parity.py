"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle, element by
element, on seeded inputs that span several tiles, vocabulary segments, backward chunks
and ragged tails, plus degenerate cases.  Tolerances: |dlp| <= 2e-3, loss relative 1e-4
(with the cancellation guard), dH and dW relative Frobenius <= 5e-3."""
import numpy as np
import pytest
import torch

import workloads as wl
from tests import helpers as h

pytestmark = pytest.mark.gpu

CASES = {
    # name: (n_groups, group_size, lengths, d, V, seed)
    "tiny": None,
    "ragged_multiseg": (3, 3, ("uniform", 20, 90), 128, 5000, 201),
    "one_tile_vocab": (1, 3, ("uniform", 1, 5), 64, 7, 202),
    "single_vocab": (1, 2, ("uniform", 3, 4), 64, 1, 203),
    "single_token": (1, 1, ("uniform", 1, 1), 256, 300, 204),
    "two_chunks": (2, 4, ("uniform", 2100, 2300), 64, 300, 205),
    "wide_d": (2, 2, ("uniform", 40, 70), 1600, 2100, 206),
    "max_d": (1, 2, ("uniform", 30, 60), 32768, 600, 210),  # the largest d the library accepts
}


# exact response lengths at the backward's 16384-token chunk boundary: one full chunk, and
# a full chunk plus a one-token chunk (one row in a 128-row tile; dW with K = 1)
FIXED = {
    "chunk_exact": ([8000, 8384], 64, 300, 211),
    "chunk_plus_one": ([8000, 8385], 64, 300, 212),
}
CASES.update({k: None for k in FIXED})


def _fixed_problem(lengths, d, V, seed):
    off = np.zeros(len(lengths) + 1, np.int64)
    off[1:] = np.cumsum(lengths)
    n = int(off[-1])
    seg = wl.Segments(off, np.zeros(len(lengths), np.int32), np.array([1.0, 0.0], np.float32), 1)
    H, W = wl.draw_matrices(n, d, V, seed)
    return wl.Problem(H, W, wl.draw_uniform_ids(n, V, seed), seg, d, V, ("normal", 0.05), seed)


def _problem(name):
    if name == "tiny":
        return wl.tiny()
    if name in FIXED:
        return _fixed_problem(*FIXED[name])
    g, gs, lengths, d, V, seed = CASES[name]
    return wl.custom(g, gs, lengths, d, V, seed)


@pytest.fixture(scope="module")
def rz():
    import invariant_logprobs_reinforce_b200 as rz
    from invariant_logprobs_reinforce_b200 import build
    build.build()
    return rz


def _run(rz, oracle, name):
    p = _problem(name)
    dev = h.to_device(p)
    lp_o, lse_o = oracle.token_logprobs(p.H, p.W, p.ids)
    lr = wl.rollout_logprobs_with_lag(lp_o, p.noise, p.seed)
    ref = oracle.loss_fwd_bwd(p.H, p.W, p.ids, lr, p.seg.rewards, p.seg.seg_offsets, p.seg.group_ids,
                              p.seg.n_groups)
    lp_g, lse_g = rz.rz_token_logprobs(dev["H"], dev["W"], dev["ids"])
    out = rz.rz_loss_fwd_bwd(dev["H"], dev["W"], dev["ids"], torch.from_numpy(lr).cuda(), dev["rewards"],
                             dev["seg_offsets"], dev["group_ids"], p.seg.n_groups)
    code, bits = rz.rz_read_device_status(out["workspace"])
    assert code == 0 and bits == 0, (code, bits)
    return p, lr, ref, lp_g, lse_g, out


@pytest.mark.parametrize("name", list(CASES))
def test_parity_against_oracle(rz, oracle, name):
    p, lr, ref, lp_g, lse_g, out = _run(rz, oracle, name)
    lp = lp_g.cpu().numpy().astype(np.float64)
    lse = lse_g.cpu().numpy().astype(np.float64)
    assert np.abs(lp - ref["lp"]).max() <= h.LP_ATOL
    assert np.abs(lse - ref["lse"]).max() <= h.LP_ATOL
    # the loss call's logprobs are the forward call's, bit for bit
    assert torch.equal(out["lp"].view(torch.int32), lp_g.view(torch.int32))
    A = oracle.advantages(p.seg.rewards, p.seg.group_ids, p.seg.n_groups)
    wm = h.response_means(ref["w"], p.seg.seg_offsets)
    assert h.loss_close(float(out["loss"].item()), ref["loss"], A, wm), (out["loss"].item(), ref["loss"])
    kappa = out["kappa"].cpu().numpy().astype(np.float64)
    kscale = np.abs(ref["kappa"]).max()
    if kscale > 0:
        assert np.abs(kappa - ref["kappa"]).max() <= 5e-3 * kscale
    else:
        assert np.all(kappa == 0.0)
    dH = h.torch_bf16_to_f64(out["dH"])
    dW = out["dW"].cpu().numpy().astype(np.float64)
    if np.linalg.norm(ref["dH"]) == 0.0:
        assert np.all(dH == 0.0) and np.all(dW == 0.0)
    else:
        assert h.rel_fro(dH, ref["dH"]) <= h.GRAD_RFRO, h.rel_fro(dH, ref["dH"])
        assert h.rel_fro(dW, ref["dW"]) <= h.GRAD_RFRO, h.rel_fro(dW, ref["dW"])


def test_repeat_calls_are_bitwise_identical(rz):
    p = _problem("ragged_multiseg")
    dev = h.to_device(p)
    lr = torch.full((p.n_tok,), -8.0, dtype=torch.float32, device="cuda")
    a = rz.rz_loss_fwd_bwd(dev["H"], dev["W"], dev["ids"], lr, dev["rewards"], dev["seg_offsets"],
                           dev["group_ids"], p.seg.n_groups)
    b = rz.rz_loss_fwd_bwd(dev["H"], dev["W"], dev["ids"], lr, dev["rewards"], dev["seg_offsets"],
                           dev["group_ids"], p.seg.n_groups)
    for k in ("loss", "lp", "kappa", "dW"):
        assert torch.equal(a[k].view(torch.int32), b[k].view(torch.int32)), k
    assert torch.equal(a["dH"].view(torch.int16), b["dH"].view(torch.int16))


def test_equal_rewards_give_exact_zero_gradient(rz):
    """All rewards equal within each group: A = 0 exactly, so kappa, dH and dW are exactly 0."""
    p = _problem("ragged_multiseg")
    dev = h.to_device(p)
    rewards = torch.tensor([1.0, 1.0, 1.0, 0.0, 0.0, 0.0, 1.0, 1.0, 1.0], device="cuda")
    lr = torch.full((p.n_tok,), -8.0, dtype=torch.float32, device="cuda")
    out = rz.rz_loss_fwd_bwd(dev["H"], dev["W"], dev["ids"], lr, rewards, dev["seg_offsets"], dev["group_ids"],
                             p.seg.n_groups)
    assert out["loss"].item() == 0.0
    assert torch.all(out["kappa"] == 0) and torch.all(out["dH"] == 0) and torch.all(out["dW"] == 0)


def test_zero_head_gives_minus_log_V(rz):
    """W = 0: every logit is 0 and lp = -ln V (fp32 sum of V ones is exact)."""
    for V in (1, 300, 4096, 5000):
        H = torch.randn(200, 128, device="cuda").to(torch.bfloat16)
        W = torch.zeros(V, 128, device="cuda", dtype=torch.bfloat16)
        ids = torch.randint(0, V, (200,), device="cuda", dtype=torch.int32)
        lp, lse = rz.rz_token_logprobs(H, W, ids)
        assert torch.allclose(lp.double(), torch.full_like(lp.double(), -np.log(V)), atol=4e-6, rtol=0)
        assert torch.allclose(lse.double(), torch.full_like(lse.double(), np.log(V)), atol=4e-6, rtol=0)


def _segments_for(layout):
    if layout == "contiguous_groups":  # moe_head shape: 128 groups x 16, lengths U{256..4096}
        return wl.draw_segments("moe_head")
    rng = np.random.default_rng(17)
    if layout == "interleaved_groups":  # group ids not sorted: response i in group i % 37
        L = rng.integers(1, 300, size=37 * 11)
        gid = (np.arange(L.size) % 37).astype(np.int32)
        G = 37
    else:  # "short_responses": 1..3 tokens each, > 256 responses per 4096-token block
        L = rng.integers(1, 4, size=20000)
        gid = (np.arange(L.size) // 5).astype(np.int32)
        G = int(gid[-1]) + 1
    off = np.zeros(L.size + 1, np.int64)
    off[1:] = np.cumsum(L)
    r = (rng.uniform(size=L.size) < 0.4).astype(np.float32)
    return wl.Segments(off, gid, r, G)


@pytest.mark.parametrize("layout", ["contiguous_groups", "interleaved_groups", "short_responses"])
def test_segment_loss_stage_against_oracle(rz, oracle, layout):
    """The loss stage alone, fed the same synthetic logprobs on both sides: relative 1e-4."""
    seg = _segments_for(layout)
    rng = np.random.default_rng(9)
    n = seg.n_tok
    lp = (-rng.exponential(2.0, n)).astype(np.float32)
    lr = wl.rollout_logprobs_with_lag(lp, ("normal", 0.05), 105)
    loss_o, w_o, kappa_o = oracle.loss_from_lp(lp.astype(np.float64), lr.astype(np.float64), seg.rewards,
                                               seg.seg_offsets, seg.group_ids, seg.n_groups)
    out = rz.rz_segment_loss(torch.from_numpy(lp).cuda(), torch.from_numpy(lr).cuda(),
                             torch.from_numpy(seg.rewards).cuda(), torch.from_numpy(seg.seg_offsets).cuda(),
                             torch.from_numpy(seg.group_ids).cuda(), seg.n_groups, want_w=True)
    assert rz.rz_read_device_status(out["workspace"]) == (0, 0)
    A = oracle.advantages(seg.rewards, seg.group_ids, seg.n_groups)
    scale = float(np.mean(np.abs(A) * h.response_means(w_o, seg.seg_offsets)))
    assert abs(out["loss"].item() - loss_o) <= 1e-4 * max(abs(loss_o), scale)
    # the ratio is 2^((lp - lp_rollout) log2 e) on the MUFU ex2 unit: about 2 + 1.2|x| ulp
    np.testing.assert_allclose(out["w"].cpu().numpy(), w_o, rtol=2e-6)
    np.testing.assert_allclose(out["kappa"].cpu().numpy(), kappa_o, rtol=1e-5, atol=1e-30)


def test_segment_loss_sorted_and_unsorted_groups_agree_bitwise(rz):
    """Contiguous and scattered group layouts take different kernel paths but add the same
    rewards in the same order: permuting responses permutes kappa exactly."""
    seg = _segments_for("contiguous_groups")
    rng = np.random.default_rng(4)
    lp = (-rng.exponential(2.0, seg.n_tok)).astype(np.float32)
    lr = (lp + 0.03).astype(np.float32)
    a = rz.rz_segment_loss(torch.from_numpy(lp).cuda(), torch.from_numpy(lr).cuda(),
                           torch.from_numpy(seg.rewards).cuda(), torch.from_numpy(seg.seg_offsets).cuda(),
                           torch.from_numpy(seg.group_ids).cuda(), seg.n_groups)
    # reverse the response order (group ids become decreasing: the general path)
    R = seg.n_resp
    perm = np.arange(R)[::-1]
    off = seg.seg_offsets
    tok = np.concatenate([np.arange(off[i], off[i + 1]) for i in perm])
    off2 = np.zeros(R + 1, np.int64)
    off2[1:] = np.cumsum(np.diff(off)[perm])
    b = rz.rz_segment_loss(torch.from_numpy(lp[tok]).cuda(), torch.from_numpy(lr[tok]).cuda(),
                           torch.from_numpy(seg.rewards[perm].copy()).cuda(), torch.from_numpy(off2).cuda(),
                           torch.from_numpy(seg.group_ids[perm].copy()).cuda(), seg.n_groups)
    ka = a["kappa"].cpu().numpy()
    kb = b["kappa"].cpu().numpy()
    assert np.array_equal(ka[tok].view(np.int32), kb.view(np.int32))
