"""Pins for the fp64 oracle: closed forms, invariants and brute force (CPU only).

None of these re-types the oracle's formulas; each checks a fact the pages or the
mathematics fix, chosen so that a plausible slip in the oracle (a dropped 1/L_i or 1/N,
a wrong sign, the ratio inverted, a transposed operand, a global instead of a group
mean, std-normalised advantages, a wrong gradient term) fails at least one of them.

Page cited throughout: "vLLM says aligned kernels make asynchronous RL stable at lag 64"
(ainewsbites.com), section "REINFORCE Zero removes the mismatch first".
"""
import math

import numpy as np
import pytest
from scipy.special import logsumexp

import workloads as wl


def _bf(x):
    return wl.bf16_bits(np.asarray(x, np.float32))


def _segments(lengths, group_size):
    L = np.asarray(lengths, np.int64)
    off = np.zeros(len(L) + 1, np.int64)
    off[1:] = np.cumsum(L)
    gid = (np.arange(len(L)) // group_size).astype(np.int32)
    return off, gid


# ---------------------------------------------------------------- forward (token logprob)

def test_p1_zero_head_gives_minus_log_V(oracle):
    """W = 0 makes every logit 0, so lp = -ln V and lse = ln V exactly."""
    rng = np.random.default_rng(0)
    for V in (1, 7, 4096):
        H = _bf(rng.standard_normal((5, 64)))
        W = np.zeros((V, 64), np.uint16)
        ids = rng.integers(0, V, 5).astype(np.int32)
        lp, lse = oracle.token_logprobs(H, W, ids)
        np.testing.assert_allclose(lp, -math.log(V), rtol=0, atol=1e-15)
        np.testing.assert_allclose(lse, math.log(V), rtol=0, atol=1e-15)
    assert abs(-math.log(4096) - (-8.317766166719343)) < 1e-15


def test_p2_two_valued_logits_closed_form(oracle):
    """H_t = e_0, W[y] = a e_0, other rows 0: lp = a - ln(e^a + V - 1)."""
    V, d, a = 37, 8, 2.5  # 2.5 is exact in bf16
    H = np.zeros((3, d), np.float32)
    H[:, 0] = 1.0
    for t, y in enumerate((0, 11, 36)):
        W = np.zeros((V, d), np.float32)
        W[y, 0] = a
        lp, _ = oracle.token_logprobs(_bf(H[t:t + 1]), _bf(W), np.array([y], np.int32))
        assert abs(lp[0] - (a - math.log(math.exp(a) + V - 1))) < 1e-14
        # a token other than the raised one sees logit 0
        other = (y + 1) % V
        lp2, _ = oracle.token_logprobs(_bf(H[t:t + 1]), _bf(W), np.array([other], np.int32))
        assert abs(lp2[0] - (0.0 - math.log(math.exp(a) + V - 1))) < 1e-14


def test_onehot_hidden_selects_head_column(oracle):
    """H_t = e_k gives z_v = W[v,k]: lp = W[y,k] - logsumexp_v W[v,k] (scipy)."""
    rng = np.random.default_rng(1)
    V, d = 50, 16
    W = _bf(rng.standard_normal((V, d)))
    Wf = wl.bits_to_f32(W).astype(np.float64)
    ks = np.array([0, 3, 15, 7], np.int64)
    H = np.zeros((len(ks), d), np.float32)
    H[np.arange(len(ks)), ks] = 1.0
    ids = np.array([5, 0, 49, 23], np.int32)
    lp, lse = oracle.token_logprobs(_bf(H), W, ids)
    for t, k in enumerate(ks):
        ref = logsumexp(Wf[:, k])
        assert abs(lse[t] - ref) < 1e-13
        assert abs(lp[t] - (Wf[ids[t], k] - ref)) < 1e-13


def test_p3_probabilities_sum_to_one(oracle):
    """sum_v exp(lp(t, v)) = 1 for every row (normalisation of the log-softmax)."""
    rng = np.random.default_rng(2)
    V, d, n = 16, 8, 3
    H = _bf(rng.standard_normal((n, d)))
    W = _bf(rng.standard_normal((V, d)))
    Hr = np.repeat(H, V, axis=0)
    ids = np.tile(np.arange(V, dtype=np.int32), n)
    lp, _ = oracle.token_logprobs(Hr, W, ids)
    s = np.exp(lp).reshape(n, V).sum(axis=1)
    np.testing.assert_allclose(s, 1.0, rtol=0, atol=1e-14)


def test_rows_subset_matches_full(oracle):
    p = wl.custom(1, 2, ("uniform", 3, 5), 16, 40, seed=5)
    lp, lse = oracle.token_logprobs(p.H, p.W, p.ids)
    rows = np.array([p.n_tok - 1, 0, 2], np.int64)
    lp2, lse2 = oracle.token_logprobs(p.H, p.W, p.ids, rows=rows)
    np.testing.assert_array_equal(lp2, lp[rows])
    np.testing.assert_array_equal(lse2, lse[rows])


# ---------------------------------------------------------------- advantages and loss

def test_p4_group_advantages(oracle):
    """Advantage = reward minus its group's mean: zero-sum per group, 0 for singletons."""
    r = np.array([1, 0, 0, 0, 0.5, 0.25, 1], np.float64)
    gid = np.array([0, 0, 0, 0, 1, 1, 2], np.int32)
    A = oracle.advantages(r, gid, 3)
    np.testing.assert_allclose(A[:4], [0.75, -0.25, -0.25, -0.25], atol=1e-16)
    np.testing.assert_allclose(A[4:6], [0.125, -0.125], atol=1e-16)
    assert A[6] == 0.0
    rng = np.random.default_rng(3)
    gid = rng.integers(0, 9, 200).astype(np.int32)
    gid[:9] = np.arange(9)
    A = oracle.advantages(rng.uniform(size=200), gid, 9)
    for g in range(9):
        assert abs(A[gid == g].sum()) < 1e-13


def _tiny_problem(seed=11, n_groups=2, group_size=2, lengths=(3, 1, 2, 4), d=8, V=16):
    rng = np.random.default_rng(seed)
    off, gid = _segments(lengths, group_size)
    n = int(off[-1])
    H = rng.standard_normal((n, d))
    W = rng.standard_normal((V, d)) * 0.7
    ids = rng.integers(0, V, n).astype(np.int32)
    rewards = rng.uniform(size=len(lengths))
    lp_roll = rng.standard_normal(n) * 0.3 - 2.5
    return dict(H=H, W=W, ids=ids, lp_rollout=lp_roll, rewards=rewards, seg_offsets=off,
                group_ids=gid, n_groups=n_groups)


def _loss(oracle, p):
    return oracle.loss_fwd_bwd(p["H"], p["W"], p["ids"], p["lp_rollout"], p["rewards"], p["seg_offsets"],
                               p["group_ids"], p["n_groups"], want_dh=False, want_dw=False)["loss"]


def test_p5_on_policy_ratio_is_one_and_loss_vanishes(oracle):
    """lp_rollout = lp gives w = 1 exactly and, for complete groups, loss = 0."""
    p = _tiny_problem()
    lp, _ = oracle.token_logprobs(p["H"], p["W"], p["ids"])
    loss, w, _ = oracle.loss_from_lp(lp, lp, p["rewards"], p["seg_offsets"], p["group_ids"], p["n_groups"])
    assert np.all(w == 1.0)
    assert abs(loss) < 1e-16


def test_loss_per_response_token_mean(oracle):
    """Repeating every response's tokens twice leaves the loss unchanged (1/L_i)."""
    p = _tiny_problem()
    base = _loss(oracle, p)
    off = p["seg_offsets"]
    idx = np.concatenate([np.tile(np.arange(off[i], off[i + 1]), 2) for i in range(len(off) - 1)])
    q = dict(p, H=p["H"][idx], ids=p["ids"][idx], lp_rollout=p["lp_rollout"][idx],
             seg_offsets=off * 2)
    assert abs(_loss(oracle, q) - base) < 1e-14 * max(1.0, abs(base))
    assert abs(base) > 1e-3  # the problem is not degenerate


def test_loss_mean_over_responses(oracle):
    """Duplicating the whole batch as new groups leaves the loss unchanged (1/N)."""
    p = _tiny_problem()
    base = _loss(oracle, p)
    n = p["H"].shape[0]
    off = p["seg_offsets"]
    q = dict(p, H=np.concatenate([p["H"], p["H"]]), ids=np.concatenate([p["ids"], p["ids"]]),
             lp_rollout=np.concatenate([p["lp_rollout"], p["lp_rollout"]]),
             rewards=np.concatenate([p["rewards"], p["rewards"]]),
             seg_offsets=np.concatenate([off, off[1:] + n]),
             group_ids=np.concatenate([p["group_ids"], p["group_ids"] + p["n_groups"]]).astype(np.int32),
             n_groups=2 * p["n_groups"])
    assert abs(_loss(oracle, q) - base) < 1e-14 * max(1.0, abs(base))


def test_loss_scales_with_rewards_no_std_normalisation(oracle):
    """Scaling rewards by c scales the loss by c (advantage is not divided by a std)."""
    p = _tiny_problem()
    base = _loss(oracle, p)
    q = dict(p, rewards=p["rewards"] * 3.0)
    assert abs(_loss(oracle, q) - 3.0 * base) < 1e-13


def test_p10_group_constant_shift_invariance(oracle):
    """Adding a constant per group to the rewards changes nothing (group, not global, mean)."""
    p = _tiny_problem(n_groups=2, group_size=2)
    a = oracle.loss_fwd_bwd(p["H"], p["W"], p["ids"], p["lp_rollout"], p["rewards"], p["seg_offsets"],
                            p["group_ids"], p["n_groups"])
    shift = np.array([5.0, -2.0])[p["group_ids"]]
    b = oracle.loss_fwd_bwd(p["H"], p["W"], p["ids"], p["lp_rollout"], p["rewards"] + shift, p["seg_offsets"],
                            p["group_ids"], p["n_groups"])
    assert abs(a["loss"] - b["loss"]) < 1e-13
    np.testing.assert_allclose(b["dH"], a["dH"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(b["dW"], a["dW"], rtol=0, atol=1e-13)
    # a global (non-group) shift of one group only must matter if the mean were global:
    # here the group mean absorbs it, so kappa is unchanged as well
    np.testing.assert_allclose(b["kappa"], a["kappa"], rtol=0, atol=1e-14)


def test_loss_sign_and_ratio_direction(oracle):
    """Raising the learner/rollout ratio of a better-than-average response lowers the loss.

    The loss is minimised; w = pi_learner / pi_rollout, so lowering the recorded rollout
    logprob of the rewarded response (A > 0) raises its w and must decrease the loss;
    doing the same to the unrewarded response (A < 0) must increase it.
    """
    off, gid = _segments((2, 3), 2)
    rng = np.random.default_rng(4)
    H = rng.standard_normal((5, 4))
    W = rng.standard_normal((6, 4))
    ids = rng.integers(0, 6, 5).astype(np.int32)
    lp_roll = np.full(5, -1.8)
    r = np.array([1.0, 0.0])
    base = oracle.loss_fwd_bwd(H, W, ids, lp_roll, r, off, gid, 1, False, False)["loss"]
    good = lp_roll.copy()
    good[0:2] -= 0.2
    bad = lp_roll.copy()
    bad[2:5] -= 0.2
    assert oracle.loss_fwd_bwd(H, W, ids, good, r, off, gid, 1, False, False)["loss"] < base - 1e-6
    assert oracle.loss_fwd_bwd(H, W, ids, bad, r, off, gid, 1, False, False)["loss"] > base + 1e-6


def test_p9_equal_rewards_give_exact_zero_gradient(oracle):
    """All rewards equal within each group: A = 0, kappa = 0, dH = dW = 0 and loss = 0 exactly."""
    p = _tiny_problem()
    p["rewards"] = np.array([1.0, 1.0, 0.0, 0.0])
    out = oracle.loss_fwd_bwd(p["H"], p["W"], p["ids"], p["lp_rollout"], p["rewards"], p["seg_offsets"],
                              p["group_ids"], p["n_groups"])
    assert out["loss"] == 0.0
    assert np.all(out["kappa"] == 0.0)
    assert np.all(out["dH"] == 0.0) and np.all(out["dW"] == 0.0)


# ---------------------------------------------------------------- gradients

def _fd_check(oracle, p, loss_fn, out):
    h = 1e-5
    for name, grad in (("H", out["dH"]), ("W", out["dW"])):
        X = p[name]
        for idx in np.ndindex(X.shape):
            Xp = X.copy()
            Xp[idx] += h
            Xm = X.copy()
            Xm[idx] -= h
            fd = (loss_fn(dict(p, **{name: Xp})) - loss_fn(dict(p, **{name: Xm}))) / (2 * h)
            g = grad[idx]
            assert abs(fd - g) <= 1e-6 * max(abs(g), 1e-3 * np.abs(grad).max()), (name, idx, fd, g)


def test_p8_finite_difference_gradients(oracle):
    """Central differences of the loss (ratio recomputed) match dH and dW element by element."""
    p = _tiny_problem(lengths=(3, 1, 2, 6), d=8, V=16)
    out = oracle.loss_fwd_bwd(p["H"], p["W"], p["ids"], p["lp_rollout"], p["rewards"], p["seg_offsets"],
                              p["group_ids"], p["n_groups"])
    assert np.abs(out["dH"]).max() > 1e-4 and np.abs(out["dW"]).max() > 1e-4
    _fd_check(oracle, p, lambda q: _loss(oracle, q), out)


def test_p5_on_policy_gradient_is_plain_reinforce(oracle):
    """At lp_rollout = lp the gradient is plain REINFORCE: -(1/N) sum_i (A_i/L_i) sum_t grad lp_t.

    The right-hand side is differentiated numerically from the oracle's token logprobs
    alone (no loss routine involved).
    """
    p = _tiny_problem(lengths=(2, 3, 1, 2), d=6, V=9)
    lp, _ = oracle.token_logprobs(p["H"], p["W"], p["ids"])
    out = oracle.loss_fwd_bwd(p["H"], p["W"], p["ids"], lp, p["rewards"], p["seg_offsets"],
                              p["group_ids"], p["n_groups"])
    A = oracle.advantages(p["rewards"], p["group_ids"], p["n_groups"])
    off = p["seg_offsets"]
    L = np.diff(off)
    N = len(L)
    coef = np.repeat(-A / (N * L), L)

    def reinforce(q):
        lpq, _ = oracle.token_logprobs(q["H"], q["W"], q["ids"])
        return float(np.dot(coef, lpq))

    _fd_check(oracle, p, reinforce, out)


def test_p6_dW_columns_sum_to_zero(oracle):
    """sum_v dZ[t,v] = 0 for every token, hence sum_v dW[v,:] = 0."""
    p = wl.tiny()
    lp, _ = oracle.token_logprobs(p.H, p.W, p.ids)
    lr = wl.rollout_logprobs_with_lag(lp, p.noise, p.seed)
    out = oracle.loss_fwd_bwd(p.H, p.W, p.ids, lr, p.seg.rewards, p.seg.seg_offsets, p.seg.group_ids,
                              p.seg.n_groups)
    col = out["dW"].sum(axis=0)
    assert np.abs(col).max() < 1e-12 * max(1.0, np.abs(out["dW"]).sum(axis=0).max())


def test_p7_dH_is_kappa_times_target_row_minus_softmax_mean_row(oracle):
    """dH_t = kappa_t (W[y_t] - sum_v p_tv W[v]): the factored form, with p from scipy's
    softmax of logits formed here in fp64 (not the oracle's lse); only kappa comes from the
    oracle (pinned by the finite differences)."""
    from scipy.special import softmax
    p = wl.tiny()
    lp, _ = oracle.token_logprobs(p.H, p.W, p.ids)
    lr = wl.rollout_logprobs_with_lag(lp, p.noise, p.seed)
    out = oracle.loss_fwd_bwd(p.H, p.W, p.ids, lr, p.seg.rewards, p.seg.seg_offsets, p.seg.group_ids,
                              p.seg.n_groups)
    Hf = wl.bits_to_f32(p.H).astype(np.float64)
    Wf = wl.bits_to_f32(p.W).astype(np.float64)
    P = softmax(Hf @ Wf.T, axis=1)
    ref = out["kappa"][:, None] * (Wf[p.ids] - P @ Wf)
    assert np.abs(out["dH"] - ref).max() <= 1e-12 * np.abs(ref).max()


def test_dh_dw_row_subsets_match_full(oracle):
    p = _tiny_problem()
    out = oracle.loss_fwd_bwd(p["H"], p["W"], p["ids"], p["lp_rollout"], p["rewards"], p["seg_offsets"],
                              p["group_ids"], p["n_groups"])
    rows = np.array([4, 0, 9], np.int64)
    dh = oracle.dh_rows(p["H"], p["W"], p["ids"], rows, out["lse"][rows], out["kappa"][rows])
    np.testing.assert_allclose(dh, out["dH"][rows], rtol=1e-13, atol=1e-15)
    vr = np.array([15, 2], np.int64)
    dw = oracle.dw_rows(p["H"], p["W"], p["ids"], out["lse"], out["kappa"], vr)
    np.testing.assert_allclose(dw, out["dW"][vr], rtol=1e-13, atol=1e-15)


def test_p12_permuting_responses_permutes_outputs(oracle):
    p = _tiny_problem(lengths=(3, 1, 2, 4))
    a = oracle.loss_fwd_bwd(p["H"], p["W"], p["ids"], p["lp_rollout"], p["rewards"], p["seg_offsets"],
                            p["group_ids"], p["n_groups"])
    perm = np.array([2, 0, 3, 1])
    off = p["seg_offsets"]
    tok = np.concatenate([np.arange(off[i], off[i + 1]) for i in perm])
    L = np.diff(off)[perm]
    off2 = np.zeros(5, np.int64)
    off2[1:] = np.cumsum(L)
    b = oracle.loss_fwd_bwd(p["H"][tok], p["W"], p["ids"][tok], p["lp_rollout"][tok], p["rewards"][perm],
                            off2, p["group_ids"][perm], p["n_groups"])
    assert abs(a["loss"] - b["loss"]) < 1e-15
    np.testing.assert_array_equal(b["lp"], a["lp"][tok])
    np.testing.assert_allclose(b["kappa"], a["kappa"][tok], rtol=1e-15, atol=0)
    np.testing.assert_allclose(b["dH"], a["dH"][tok], rtol=1e-13, atol=1e-16)
    np.testing.assert_allclose(b["dW"], a["dW"], rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------- argument checks

@pytest.mark.parametrize("bad", ["id", "group", "offsets", "empty"])
def test_invalid_inputs_are_rejected(oracle, bad):
    p = _tiny_problem()
    if bad == "id":
        p["ids"] = p["ids"].copy()
        p["ids"][3] = 16
    elif bad == "group":
        p["group_ids"] = np.array([0, 0, 1, 2], np.int32)
    elif bad == "offsets":
        p["seg_offsets"] = p["seg_offsets"].copy()
        p["seg_offsets"][-1] += 1
    else:
        p["seg_offsets"] = np.array([0, 3, 3, 6, 10], np.int64)
    with pytest.raises(oracle.OracleError):
        _loss(oracle, p)


# ---------------------------------------------------------------- e4m3 operands

def test_e4m3_quantisation_reference(oracle):
    """Codes decode to x / scale rounded to e4m3 (3 mantissa bits): exact for values that
    are e4m3 numbers times the scale, within half an e4m3 ulp otherwise; the row maximum
    maps to +-448; zero rows get scale 1 and zero codes."""
    rng = np.random.default_rng(0)
    X = rng.standard_normal((5, 64)).astype(np.float32)
    X[3] = 0.0
    X[4] = np.array([2.0 ** k for k in range(-6, 2)] * 8, np.float32)  # x / scale = 224 x: 3.5 .. 448, all e4m3
    bits = wl.bf16_bits(X)
    q, sc = oracle.quantize_rows_e4m3(bits)
    xf = wl.bits_to_f32(bits).astype(np.float64)
    dec = oracle.decode_e4m3(q) * sc[:, None].astype(np.float64)
    assert sc[3] == 1.0 and np.all(q[3] == 0)
    for r in (0, 1, 2):
        assert np.max(np.abs(oracle.decode_e4m3(q[r]))) == 448.0
        rel = np.abs(dec[r] - xf[r]) / np.maximum(np.abs(xf[r]), 2.0 ** -6 * sc[r])
        assert rel.max() <= 2.0 ** -4 + 1e-12
    np.testing.assert_array_equal(oracle.decode_e4m3(q[4]), xf[4] * 224.0)
