"""Pins for the oracle's loss-stage variants and ratio diagnostics (CPU only).

The variants are the baselines the pages contrast REINFORCE Zero with ("vLLM says
aligned kernels make asynchronous RL stable at lag 64", sections "REINFORCE Zero removes
the mismatch first" and "Zero mismatch expands to newer models"): truncated importance
weights, a sequence-level gate and a token mask; the diagnostics are the pages'
observables (importance-weight deviation peak vs median, rollout-to-learner KL).
"""
import math

import numpy as np
import pytest
from scipy.stats import entropy

import oracle as o


def _case(seed=3, lengths=(3, 5, 2, 4, 6, 1), gs=3):
    rng = np.random.default_rng(seed)
    L = np.asarray(lengths)
    off = np.zeros(len(L) + 1, np.int64)
    off[1:] = np.cumsum(L)
    n = int(off[-1])
    gid = (np.arange(len(L)) // gs).astype(np.int32)
    r = rng.uniform(size=len(L))
    lp = -rng.exponential(2.0, n)
    lr = lp + rng.normal(0, 0.3, n)
    return dict(lp=lp, lr=lr, r=r, off=off, gid=gid, G=int(gid.max()) + 1)


def _ex(c, **kw):
    return o.loss_from_lp_ex(c["lp"], c["lr"], c["r"], c["off"], c["gid"], c["G"], **kw)


def test_default_options_reproduce_the_method():
    c = _case()
    a = o.loss_from_lp(c["lp"], c["lr"], c["r"], c["off"], c["gid"], c["G"])
    b = _ex(c)
    assert a[0] == b[0]
    np.testing.assert_array_equal(a[2], b[2])
    np.testing.assert_array_equal(a[1], b[1])


def test_clip_above_every_ratio_changes_nothing():
    c = _case()
    base = _ex(c)
    w_max = float(np.exp(c["lp"] - c["lr"]).max())
    clip = _ex(c, flags=o.CLIP, clip_max=w_max * 1.0001)
    assert clip[0] == base[0]
    np.testing.assert_array_equal(clip[2], base[2])


def test_clip_below_every_ratio_gives_constant_weights():
    """With every ratio above c, each token's weight is c: same as a batch whose learner
    logprobs sit exactly ln c above the rollout's."""
    c = _case()
    cmax = 0.5 * float(np.exp(c["lp"] - c["lr"]).min())
    clip = _ex(c, flags=o.CLIP, clip_max=cmax)
    flat = o.loss_from_lp(c["lr"] + math.log(cmax), c["lr"], c["r"], c["off"], c["gid"], c["G"])
    assert abs(clip[0] - flat[0]) < 1e-14
    np.testing.assert_allclose(clip[2], flat[2], rtol=1e-13, atol=1e-18)
    np.testing.assert_allclose(clip[1], np.exp(c["lp"] - c["lr"]), rtol=1e-15)  # w_out stays unclipped


def test_mask_all_ones_and_mask_as_token_removal():
    c = _case()
    base = _ex(c)
    ones = _ex(c, flags=o.MASK, mask=np.ones(len(c["lp"]), np.uint8))
    assert ones[0] == base[0]
    # masking tokens = removing them (the advantage does not depend on tokens)
    rng = np.random.default_rng(8)
    mask = (rng.uniform(size=len(c["lp"])) < 0.6).astype(np.uint8)
    off = c["off"]
    for i in range(len(off) - 1):  # keep at least one token per response
        mask[off[i]] = 1
    m = _ex(c, flags=o.MASK, mask=mask)
    keep = mask.astype(bool)
    L2 = np.array([mask[off[i]:off[i + 1]].sum() for i in range(len(off) - 1)])
    off2 = np.zeros_like(off)
    off2[1:] = np.cumsum(L2)
    red = o.loss_from_lp(c["lp"][keep], c["lr"][keep], c["r"], off2, c["gid"], c["G"])
    assert abs(m[0] - red[0]) < 1e-15
    np.testing.assert_allclose(m[2][keep], red[2], rtol=1e-14)
    assert np.all(m[2][~keep] == 0.0)


def test_fully_masked_response_contributes_nothing_but_keeps_its_reward_in_the_mean():
    c = _case()
    off = c["off"]
    mask = np.ones(len(c["lp"]), np.uint8)
    mask[off[1]:off[2]] = 0
    m = _ex(c, flags=o.MASK, mask=mask)
    base = _ex(c)
    assert np.all(m[2][off[1]:off[2]] == 0.0)
    others = np.ones(len(c["lp"]), bool)
    others[off[1]:off[2]] = False
    np.testing.assert_array_equal(m[2][others], base[2][others])


def test_sequence_gate_threshold_and_rejection():
    c = _case(lengths=(4, 4, 4), gs=3)
    off = c["off"]
    x = np.concatenate([np.full(4, 0.1), np.full(4, -0.2), np.full(4, 0.02)])  # geometric means e^0.1, e^-0.2, e^0.02
    c["lp"] = c["lr"] + x
    base = _ex(c)
    open_gate = _ex(c, flags=o.GATE, gate_lo=0.0, gate_hi=float("inf"))
    assert open_gate[0] == base[0]
    g = _ex(c, flags=o.GATE, gate_lo=0.5, gate_hi=1.05)
    assert np.all(g[2][off[0]:off[1]] == 0.0)  # e^0.1 > 1.05: rejected
    np.testing.assert_array_equal(g[2][off[1]:], base[2][off[1]:])  # the others are unchanged
    g2 = _ex(c, flags=o.GATE, gate_lo=0.9, gate_hi=1.2)
    assert np.all(g2[2][off[1]:off[2]] == 0.0)  # e^-0.2 < 0.9: rejected
    np.testing.assert_array_equal(g2[2][off[0]:off[1]], base[2][off[0]:off[1]])


def test_global_response_count_scales_the_loss():
    c = _case()
    base = _ex(c)
    R = len(c["r"])
    s = _ex(c, n_resp_total=4 * R)
    assert abs(s[0] - base[0] / 4) < 1e-16
    np.testing.assert_allclose(s[2], base[2] / 4, rtol=1e-15)


def test_kl_estimators_on_exact_samples():
    """Tokens drawn from the rollout distribution p in exact proportions, with learner q:
    k1 and k3 both equal KL(p || q) (scipy), k2 is the second-order term."""
    p = np.array([0.5, 0.3, 0.2])
    q = np.array([0.3, 0.3, 0.4])
    counts = (p * 1000).astype(int)
    outcome = np.repeat(np.arange(3), counts)
    lr = np.log(p[outcome])
    lp = np.log(q[outcome])
    off = np.array([0, 400, 1000], np.int64)
    st, rm = o.ratio_stats(lp, lr, off)
    kl = entropy(p, q)
    assert abs(st["k1"] - kl) < 1e-14
    assert abs(st["k3"] - kl) < 1e-14
    assert abs(st["k2"] - 0.5 * np.sum(p * np.log(p / q) ** 2)) < 1e-14
    assert st["count"] == 1000


def test_deviation_peak_and_median_by_hand():
    # w = 1, 2, 1/2, 3  ->  |w - 1| = 0, 1, 1/2, 2: peak 2, lower median 1/2
    x = np.log([1.0, 2.0, 0.5, 3.0])
    st, rm = o.ratio_stats(x, np.zeros(4), np.array([0, 1, 4], np.int64))
    assert st["dev_max"] == pytest.approx(2.0, abs=1e-15)
    assert st["dev_median"] == pytest.approx(0.5, abs=1e-15)
    assert st["dev_peak_over_median"] == pytest.approx(4.0, abs=1e-14)
    assert st["w_min"] == pytest.approx(0.5) and st["w_max"] == pytest.approx(3.0)
    np.testing.assert_allclose(rm, [1.0, (2.0 + 0.5 + 3.0) / 3], rtol=1e-15)
    st2, _ = o.ratio_stats(x, np.zeros(4), np.array([0, 1, 4], np.int64), mask=np.array([1, 0, 1, 1], np.uint8))
    assert st2["count"] == 3 and st2["dev_median"] == pytest.approx(0.5) and st2["dev_max"] == pytest.approx(2.0)


def test_on_policy_ratio_statistics_vanish():
    c = _case()
    st, rm = o.ratio_stats(c["lp"], c["lp"], c["off"])
    assert st["k1"] == 0 and st["k2"] == 0 and st["k3"] == 0 and st["dev_max"] == 0
    np.testing.assert_array_equal(rm, 1.0)


@pytest.mark.parametrize("n,masked", [(101, False), (100, False), (1001, True), (2, False), (1, False)])
def test_ratio_statistics_against_brute_force(n, masked):
    """Peak, exact lower median (rank floor((m-1)/2) of the m counted tokens), extremes, count
    and per-response mean ratio against a direct sort / mean of |w - 1| and w."""
    rng = np.random.default_rng(n)
    lp = -rng.exponential(2.0, n)
    lr = lp + rng.normal(0.0, 0.2, n)
    cuts = np.sort(rng.choice(np.arange(1, n), size=min(4, n - 1), replace=False)) if n > 1 else np.array([], int)
    off = np.concatenate([[0], cuts, [n]]).astype(np.int64)
    mask = (rng.uniform(size=n) < 0.7).astype(np.uint8) if masked else None
    st, rm = o.ratio_stats(lp, lr, off, mask=mask)
    keep = np.ones(n, bool) if mask is None else mask.astype(bool)
    w = np.exp(lp - lr)
    dev = np.sort(np.abs(w[keep] - 1.0))
    m = dev.size
    assert st["count"] == m
    assert st["dev_median"] == pytest.approx(dev[(m - 1) // 2], rel=1e-14)
    assert st["dev_max"] == pytest.approx(dev[-1], rel=1e-14)
    assert st["w_min"] == pytest.approx(w[keep].min(), rel=1e-14)
    assert st["w_max"] == pytest.approx(w[keep].max(), rel=1e-14)
    for i in range(len(off) - 1):
        sel = keep[off[i]:off[i + 1]]
        expect = w[off[i]:off[i + 1]][sel].mean() if sel.any() else 0.0
        assert rm[i] == pytest.approx(expect, rel=1e-14, abs=0.0)
