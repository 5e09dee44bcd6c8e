"""Pins of the dense (matrix-form) oracle, oracle/dense.py (CPU only).

The dense form is what the mid-slice parity tests compare the CUDA path with at the real
head shapes, where the row-by-row C oracle is too slow.  It is pinned here against the C
oracle (written separately, row by row, itself pinned by closed forms, finite differences
and planted mistakes) on shapes with several row groups and ragged tails, and against
closed forms of its own: a zero head, two-valued logits, vanishing dW column sums and the
zero gradient of equal rewards.
"""
import math

import numpy as np
import pytest

import workloads as wl
from oracle import dense


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("case", ["tiny", "ragged"])
def test_dense_form_agrees_with_the_row_by_row_oracle(oracle, case):
    if case == "tiny":
        p = wl.tiny()
        row_block = 512
    else:  # 7 row groups of 100 with a ragged last one, V not a multiple of any tile
        p = wl.custom(2, 3, ("uniform", 90, 150), 192, 3001, 301, rewards=("uniform",))
        row_block = 100
    lp_c, lse_c = oracle.token_logprobs(p.H, p.W, p.ids)
    lp_d, lse_d = dense.token_logprobs(p.H, p.W, p.ids, row_block=row_block)
    np.testing.assert_allclose(lp_d, lp_c, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse_d, lse_c, rtol=1e-12, atol=1e-12)
    lr = wl.rollout_logprobs_with_lag(lp_c, p.noise, p.seed)
    _, _, kappa = oracle.loss_from_lp(lp_c, lr, p.seg.rewards, p.seg.seg_offsets, p.seg.group_ids, p.seg.n_groups)
    rows = np.array([0, 1, p.V // 2, p.V - 2, p.V - 1, int(p.ids[0]), int(p.ids[-1])], np.int64)
    dH_d, dW_d = dense.gradients(p.H, p.W, p.ids, lse_c, kappa, dw_vocab_rows=rows, row_block=row_block)
    dH_c = oracle.dh_rows(p.H, p.W, p.ids, None, lse_c, kappa)
    dW_c = oracle.dw_rows(p.H, p.W, p.ids, lse_c, kappa, vocab_rows=rows)
    assert _rel(dH_d, dH_c) <= 1e-12
    assert _rel(dW_d, dW_c) <= 1e-12
    # every vocabulary row at once equals the listed rows (up to the library product's
    # rounding order, which depends on the operand shapes)
    _, dW_all = dense.gradients(p.H, p.W, p.ids, lse_c, kappa, row_block=row_block)
    assert dW_all.shape == (p.V, p.d)
    assert _rel(dW_all[rows], dW_d) <= 1e-13


def test_zero_head_gives_minus_log_V():
    rng = np.random.default_rng(1)
    for V in (1, 7, 4096, 5000):
        H = wl.bf16_bits(rng.standard_normal((40, 64), dtype=np.float32))
        W = np.zeros((V, 64), np.uint16)
        ids = rng.integers(0, V, 40)
        lp, lse = dense.token_logprobs(H, W, ids, row_block=16)
        assert np.all(np.abs(lp + math.log(V)) <= 1e-14 * max(1.0, math.log(V)))
        assert np.all(np.abs(lse - math.log(V)) <= 1e-14 * max(1.0, math.log(V)))


def test_two_valued_logits_closed_form():
    # H_t = e_0, W[y] = a e_0, every other row 0: z = a at y, 0 elsewhere
    V, d = 300, 64
    for a, y in ((1.5, 0), (-3.25, 17), (8.0, V - 1)):
        H = np.zeros((1, d), np.float32)
        H[0, 0] = 1.0
        Wf = np.zeros((V, d), np.float32)
        Wf[y, 0] = a
        lp, _ = dense.token_logprobs(wl.bf16_bits(H), wl.bf16_bits(Wf), [y])
        assert abs(lp[0] - (a - math.log(math.exp(a) + V - 1))) <= 1e-14


def test_dW_columns_sum_to_zero_and_equal_rewards_give_zero_gradient():
    p = wl.custom(2, 2, ("uniform", 20, 40), 128, 700, 302)
    lp, lse = dense.token_logprobs(p.H, p.W, p.ids, row_block=32)
    kappa = np.linspace(-1e-3, 2e-3, p.n_tok)
    dH, dW = dense.gradients(p.H, p.W, p.ids, lse, kappa, row_block=32)
    # each dZ row sums to zero over the vocabulary, so every column of dW sums to ~0
    assert np.all(np.abs(dW.sum(axis=0)) <= 1e-12 * np.abs(dW).sum(axis=0))
    dH0, dW0 = dense.gradients(p.H, p.W, p.ids, lse, np.zeros(p.n_tok), row_block=32)
    assert not np.any(dH0) and not np.any(dW0)
    assert np.any(dH) and np.any(dW)


def test_rejects_out_of_range_ids_and_rows():
    H = np.zeros((2, 64), np.uint16)
    W = np.zeros((10, 64), np.uint16)
    with pytest.raises(ValueError):
        dense.token_logprobs(H, W, [0, 10])
    with pytest.raises(ValueError):
        dense.gradients(H, W, [0, 1], np.zeros(2), np.zeros(2), dw_vocab_rows=[10])
