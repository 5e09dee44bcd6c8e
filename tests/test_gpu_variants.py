"""GPU parity of the loss-stage variants (truncated IS, sequence gate, token mask, global
N) and of the ratio diagnostics / gradient norms against the fp64 oracle."""
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


def _stage_inputs(seed=21):
    seg = wl.draw_segments("moe_head", n_groups=16, group_size=8)
    rng = np.random.default_rng(seed)
    n = seg.n_tok
    lp = (-rng.exponential(2.0, n)).astype(np.float32)
    lr = wl.rollout_logprobs_with_lag(lp, ("normal", 0.05), seed)
    mask = (rng.uniform(size=n) < 0.8).astype(np.uint8)
    return seg, lp, lr, mask


def _t(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


VARIANTS = {
    "clip": dict(clip_max=1.02),
    "gate": dict(gate=(0.995, 1.005)),
    "mask": dict(mask=True),
    "n_total": dict(n_resp_total=1000),
    "all": dict(clip_max=1.03, gate=(0.99, 1.01), mask=True, n_resp_total=777),
}


def _oracle_kwargs(spec, mask):
    import oracle as o
    kw, flags = {}, 0
    if "clip_max" in spec:
        flags |= o.CLIP
        kw["clip_max"] = spec["clip_max"]
    if "gate" in spec:
        flags |= o.GATE
        kw["gate_lo"], kw["gate_hi"] = spec["gate"]
    if spec.get("mask"):
        flags |= o.MASK
        kw["mask"] = mask
    if "n_resp_total" in spec:
        kw["n_resp_total"] = spec["n_resp_total"]
    kw["flags"] = flags
    return kw


def _rz_options(rz, spec, mask_t):
    return rz.loss_options(clip_max=spec.get("clip_max"), gate=spec.get("gate"),
                           token_mask=mask_t if spec.get("mask") else None, n_resp_total=spec.get("n_resp_total", 0))


@pytest.mark.parametrize("name", list(VARIANTS))
def test_loss_stage_variants_against_oracle(rz, oracle, name):
    spec = VARIANTS[name]
    seg, lp, lr, mask = _stage_inputs()
    loss_o, w_o, kappa_o = oracle.loss_from_lp_ex(lp.astype(np.float64), lr.astype(np.float64), seg.rewards,
                                                  seg.seg_offsets, seg.group_ids, seg.n_groups,
                                                  **_oracle_kwargs(spec, mask))
    mask_t = _t(mask)
    out = rz.rz_segment_loss_ex(_t(lp), _t(lr), _t(seg.rewards), _t(seg.seg_offsets), _t(seg.group_ids),
                                seg.n_groups, _rz_options(rz, spec, mask_t), want_w=True)
    assert rz.rz_read_device_status(out["workspace"]) == (0, 0)
    kg = out["kappa"].cpu().numpy().astype(np.float64)
    assert np.abs(kg - kappa_o).max() <= 1e-5 * np.abs(kappa_o).max()
    assert np.array_equal(kg == 0.0, kappa_o == 0.0)  # the same tokens are gated / masked out
    scale = np.abs(kappa_o).sum()
    assert abs(out["loss"].item() - loss_o) <= 1e-4 * max(abs(loss_o), scale)
    np.testing.assert_allclose(out["w"].cpu().numpy(), w_o, rtol=2e-6)


def test_default_options_are_bitwise_the_plain_calls(rz):
    seg, lp, lr, _ = _stage_inputs()
    a = rz.rz_segment_loss(_t(lp), _t(lr), _t(seg.rewards), _t(seg.seg_offsets), _t(seg.group_ids), seg.n_groups)
    b = rz.rz_segment_loss_ex(_t(lp), _t(lr), _t(seg.rewards), _t(seg.seg_offsets), _t(seg.group_ids),
                              seg.n_groups, rz.loss_options())
    assert torch.equal(a["kappa"].view(torch.int32), b["kappa"].view(torch.int32))
    assert torch.equal(a["loss"].view(torch.int32), b["loss"].view(torch.int32))
    p = wl.custom(2, 3, ("uniform", 30, 60), 128, 3000, seed=55)
    dev = h.to_device(p)
    lrt = torch.full((p.n_tok,), -8.0, device="cuda")
    c = rz.rz_loss_fwd_bwd(dev["H"], dev["W"], dev["ids"], lrt, dev["rewards"], dev["seg_offsets"],
                           dev["group_ids"], p.seg.n_groups)
    d = rz.rz_loss_fwd_bwd_ex(dev["H"], dev["W"], dev["ids"], lrt, dev["rewards"], dev["seg_offsets"],
                              dev["group_ids"], p.seg.n_groups, None)
    for k in ("loss", "lp", "kappa", "dW"):
        assert torch.equal(c[k].view(torch.int32), d[k].view(torch.int32)), k
    assert torch.equal(c["dH"].view(torch.int16), d["dH"].view(torch.int16))


def test_full_path_with_all_variants_against_oracle(rz, oracle):
    p = wl.custom(3, 3, ("uniform", 20, 90), 128, 5000, seed=207)
    dev = h.to_device(p)
    lp_o, lse_o = oracle.token_logprobs(p.H, p.W, p.ids)
    lr = wl.rollout_logprobs_with_lag(lp_o, ("normal", 0.05), p.seed)
    rng = np.random.default_rng(5)
    mask = (rng.uniform(size=p.n_tok) < 0.85).astype(np.uint8)
    spec = dict(clip_max=1.04, gate=(0.98, 1.02), mask=True, n_resp_total=20)
    loss_o, _, kappa_o = oracle.loss_from_lp_ex(lp_o, lr.astype(np.float64), p.seg.rewards, p.seg.seg_offsets,
                                                p.seg.group_ids, p.seg.n_groups, **_oracle_kwargs(spec, mask))
    dH_o = oracle.dh_rows(p.H, p.W, p.ids, None, lse_o, kappa_o)
    dW_o = oracle.dw_rows(p.H, p.W, p.ids, lse_o, kappa_o)
    mask_t = _t(mask)
    out = rz.rz_loss_fwd_bwd_ex(dev["H"], dev["W"], dev["ids"], _t(lr), dev["rewards"], dev["seg_offsets"],
                                dev["group_ids"], p.seg.n_groups, _rz_options(rz, spec, mask_t))
    assert rz.rz_read_device_status(out["workspace"]) == (0, 0)
    kg = out["kappa"].cpu().numpy().astype(np.float64)
    assert np.array_equal(kg == 0.0, kappa_o == 0.0)
    assert np.abs(kg - kappa_o).max() <= 5e-3 * np.abs(kappa_o).max()
    assert abs(out["loss"].item() - loss_o) <= 1e-4 * max(abs(loss_o), np.abs(kappa_o).sum())
    assert h.rel_fro(h.torch_bf16_to_f64(out["dH"]), dH_o) <= h.GRAD_RFRO
    assert h.rel_fro(out["dW"].cpu().numpy().astype(np.float64), dW_o) <= h.GRAD_RFRO
    # the gate's extra forward pass gives the same logprobs as the plain call
    lp_plain, _ = rz.rz_token_logprobs(dev["H"], dev["W"], dev["ids"])
    assert torch.equal(out["lp"].view(torch.int32), lp_plain.view(torch.int32))


@pytest.mark.parametrize("masked", [False, True])
def test_ratio_stats_against_oracle(rz, oracle, masked):
    seg, lp, lr, mask = _stage_inputs(seed=31)
    m = mask if masked else None
    st_o, rm_o = oracle.ratio_stats(lp.astype(np.float64), lr.astype(np.float64), seg.seg_offsets, mask=m)
    stats, rm = rz.rz_ratio_stats(_t(lp), _t(lr), _t(seg.seg_offsets), token_mask=_t(mask) if masked else None)
    st = dict(zip(rz.STAT_NAMES, stats.cpu().numpy().tolist()))
    assert st["count"] == st_o["count"]
    for k in ("k1", "k2", "k3"):  # fp64 on both sides from the same fp32 inputs
        assert abs(st[k] - st_o[k]) <= 1e-9 * abs(st_o[k]) + 1e-15, k
    for k in ("w_min", "w_max", "dev_max", "dev_median"):
        assert abs(st[k] - st_o[k]) <= 2e-6 * max(1.0, abs(st_o[k])) + 1e-7, (k, st[k], st_o[k])
    assert abs(st["dev_peak_over_median"] - st_o["dev_peak_over_median"]) <= 1e-3 * st_o["dev_peak_over_median"]
    np.testing.assert_allclose(rm.cpu().numpy(), rm_o, rtol=2e-6)


def test_ratio_stats_same_bits_at_any_alignment(rz, oracle):
    """16-byte aligned inputs take vector loads, others scalar ones; the token -> thread
    assignment is the same, so the statistics must not change by a bit.  A ragged n
    (not a multiple of 4) exercises the scalar tail of both."""
    seg, lp, lr, mask = _stage_inputs(seed=41)
    n = int(seg.seg_offsets[-1]) - 3
    off = seg.seg_offsets.copy()
    off[-1] = n
    off_t = _t(off)
    a_lp, a_lr, a_m = _t(lp[:n]), _t(lr[:n]), _t(mask[:n])
    # the same values one element into a fresh buffer: 4-byte but not 16-byte aligned
    b_lp = torch.zeros(n + 1, device="cuda")
    b_lr = torch.zeros(n + 1, device="cuda")
    b_lp[1:] = a_lp
    b_lr[1:] = a_lr
    assert a_lp.data_ptr() % 16 == 0 and b_lp[1:].data_ptr() % 16 == 4
    for m in (None, a_m):
        sa, ra = rz.rz_ratio_stats(a_lp, a_lr, off_t, token_mask=m)
        sb, rb = rz.rz_ratio_stats(b_lp[1:], b_lr[1:], off_t, token_mask=m)
        assert torch.equal(sa.view(torch.int64), sb.view(torch.int64))
        assert torch.equal(ra.view(torch.int32), rb.view(torch.int32))
    st_o, _ = oracle.ratio_stats(lp[:n].astype(np.float64), lr[:n].astype(np.float64), off, mask=None)
    st = dict(zip(rz.STAT_NAMES, rz.rz_ratio_stats(b_lp[1:], b_lr[1:], off_t)[0].cpu().numpy().tolist()))
    assert st["count"] == st_o["count"] == n
    for k in ("k1", "k2", "k3"):
        assert abs(st[k] - st_o[k]) <= 1e-9 * abs(st_o[k]) + 1e-15, k


def test_ratio_stats_k3_far_from_zero(rz, oracle):
    """|lp - lp_rollout| beyond 1/2 leaves the series for expm1; both ranges against fp64."""
    rng = np.random.default_rng(9)
    n = 50_000
    lp = (-rng.exponential(2.0, n)).astype(np.float32)
    lr = (lp + rng.choice([-1.5, -0.6, -0.49, 0.3, 0.51, 2.0], n) * rng.uniform(0.5, 1.0, n)).astype(np.float32)
    off = np.array([0, n // 3, n], np.int64)
    st_o, _ = oracle.ratio_stats(lp.astype(np.float64), lr.astype(np.float64), off)
    st = dict(zip(rz.STAT_NAMES, rz.rz_ratio_stats(_t(lp), _t(lr), _t(off))[0].cpu().numpy().tolist()))
    for k in ("k1", "k2", "k3"):
        assert abs(st[k] - st_o[k]) <= 1e-9 * abs(st_o[k]) + 1e-15, k


def test_grad_norms_match_fp64_norms(rz):
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    dH = torch.randn((3000, 256), generator=g, device="cuda").to(torch.bfloat16)
    dW = torch.randn((5001, 256), generator=g, device="cuda") * 1e-3
    norms = rz.rz_grad_norms(dH, dW).cpu().numpy()
    assert abs(norms[0] - torch.linalg.norm(dH.double()).item()) <= 1e-12 * norms[0]
    assert abs(norms[1] - torch.linalg.norm(dW.double()).item()) <= 1e-12 * norms[1]
    again = rz.rz_grad_norms(dH, dW).cpu().numpy()
    assert np.array_equal(norms, again)
