"""Property-based pins of the fp64 oracle (CPU only): identities that hold for every input,
checked over random shapes, group layouts, lengths, rewards and lags (hypothesis).  Page:
"vLLM says aligned kernels make asynchronous RL stable at lag 64" (ainewsbites.com),
section "REINFORCE Zero removes the mismatch first" (group-mean advantage, per-response
token mean, unclipped ratio)."""
import numpy as np
from hypothesis import given, settings, strategies as st

import workloads as wl

SETTINGS = settings(max_examples=40, deadline=None, derandomize=True)


@st.composite
def problems(draw):
    G = draw(st.integers(1, 4))
    sizes = [draw(st.integers(1, 4)) for _ in range(G)]
    R = sum(sizes)
    lengths = [draw(st.integers(1, 9)) for _ in range(R)]
    d = draw(st.sampled_from([8, 16]))
    V = draw(st.integers(2, 40))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    interleave = draw(st.booleans())
    rng = np.random.default_rng(seed)
    gid = np.repeat(np.arange(G), sizes).astype(np.int32)
    if interleave:
        gid = gid[rng.permutation(R)]
    off = np.zeros(R + 1, np.int64)
    off[1:] = np.cumsum(lengths)
    n = int(off[-1])
    H = wl.bf16_bits(rng.standard_normal((n, d)).astype(np.float32))
    W = wl.bf16_bits((rng.standard_normal((V, d)) / np.sqrt(d)).astype(np.float32))
    ids = rng.integers(0, V, n).astype(np.int32)
    rewards = rng.choice([0.0, 1.0, 0.5, -2.0], R)
    lag = rng.standard_normal(n) * draw(st.sampled_from([0.0, 0.05, 0.5]))
    return dict(H=H, W=W, ids=ids, rewards=rewards, off=off, gid=gid, G=G, lag=lag, n=n, R=R, sizes=sizes)


def _run(oracle, p, rewards=None, lr=None):
    lp, _ = oracle.token_logprobs(p["H"], p["W"], p["ids"])
    if lr is None:
        lr = lp + p["lag"]
    r = p["rewards"] if rewards is None else rewards
    return oracle.loss_fwd_bwd(p["H"], p["W"], p["ids"], lr, r, p["off"], p["gid"], p["G"]), lr


@SETTINGS
@given(problems())
def test_loss_is_the_sum_of_kappa(oracle, p):
    """loss = sum_t kappa_t: the loss and the per-token coefficients are written out
    separately in the oracle and must agree (a 1/L_i or 1/N missing in one of them fails)."""
    out, _ = _run(oracle, p)
    scale = np.abs(out["kappa"]).sum()
    assert abs(out["loss"] - out["kappa"].sum()) <= 1e-12 * max(scale, 1e-300)


@SETTINGS
@given(problems())
def test_group_advantages_sum_to_zero_and_shift_invariance(oracle, p):
    A = oracle.advantages(p["rewards"], p["gid"], p["G"])
    for g in range(p["G"]):
        assert abs(A[p["gid"] == g].sum()) <= 1e-12 * max(1.0, np.abs(p["rewards"]).max())
    shift = np.array([3.25, -1.0, 0.5, 7.0])[p["gid"] % 4]  # a constant per group
    a, lr = _run(oracle, p)
    b, _ = _run(oracle, p, rewards=p["rewards"] + shift, lr=lr)
    scale = np.abs(a["kappa"]).sum() + 1e-300
    assert abs(a["loss"] - b["loss"]) <= 1e-12 * max(scale, 1.0)
    assert np.abs(a["dW"] - b["dW"]).max() <= 1e-12 * max(1.0, np.abs(a["dW"]).max())


@SETTINGS
@given(problems())
def test_on_policy_loss_vanishes_and_dW_columns_sum_to_zero(oracle, p):
    lp, _ = oracle.token_logprobs(p["H"], p["W"], p["ids"])
    out, _ = _run(oracle, p, lr=lp)
    assert np.all(out["w"] == 1.0)
    assert abs(out["loss"]) <= 1e-12 * max(1.0, np.abs(p["rewards"]).max())
    col = out["dW"].sum(axis=0)
    assert np.abs(col).max() <= 1e-12 * max(1e-300, np.abs(out["dW"]).sum(axis=0).max())


@SETTINGS
@given(problems(), st.floats(0.25, 4.0))
def test_loss_is_linear_in_the_rewards(oracle, p, c):
    """Scaling every reward by c scales A, the loss and the gradient by c (no std
    normalisation of the advantage)."""
    a, lr = _run(oracle, p)
    b, _ = _run(oracle, p, rewards=c * p["rewards"], lr=lr)
    scale = np.abs(a["kappa"]).sum() + 1e-300
    assert abs(b["loss"] - c * a["loss"]) <= 1e-12 * c * max(scale, 1.0)
    assert np.abs(b["dH"] - c * a["dH"]).max() <= 1e-12 * c * max(1.0, np.abs(a["dH"]).max())


@SETTINGS
@given(problems())
def test_responses_in_any_order(oracle, p):
    """Reordering the responses (tokens move with their response) permutes lp, kappa and dH
    rows and leaves the loss and dW unchanged up to summation order."""
    rng = np.random.default_rng(p["n"] * 7 + p["R"])
    perm = rng.permutation(p["R"])
    L = np.diff(p["off"])
    tok = np.concatenate([np.arange(p["off"][i], p["off"][i + 1]) for i in perm])
    off2 = np.zeros(p["R"] + 1, np.int64)
    off2[1:] = np.cumsum(L[perm])
    a, lr = _run(oracle, p)
    q = dict(p, H=p["H"][tok], ids=p["ids"][tok], rewards=p["rewards"][perm], off=off2, gid=p["gid"][perm])
    b, _ = _run(oracle, q, lr=lr[tok])
    # rewards are dyadic (0, 1, 0.5, -2), so group sums are exact in any order and kappa too
    assert np.array_equal(b["lp"], a["lp"][tok]) and np.array_equal(b["kappa"], a["kappa"][tok])
    assert np.array_equal(b["dH"], a["dH"][tok])
    scale = np.abs(a["kappa"]).sum() + 1e-300
    assert abs(a["loss"] - b["loss"]) <= 1e-12 * max(scale, 1.0)
    assert np.abs(a["dW"] - b["dW"]).max() <= 1e-12 * max(1.0, np.abs(a["dW"]).max())
