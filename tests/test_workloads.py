"""The seeded input recipes (workloads.py) on CPU: each configuration's response structure,
lengths, rewards and token count as stated in the workload table, determinism under its
seed, the fp32 -> bf16 rounding, the lag noise, whole-group truncation under a cap, and the
temperature-1 sampler's token frequencies."""
import numpy as np
import pytest

import workloads as wl

TOKENS = {"tiny": 331, "qwen3_4b": 360896, "lag64": 1437610, "moe_head": 4350897}


@pytest.mark.parametrize("name", list(TOKENS))
def test_segments_follow_the_recipe(name):
    cfg = wl.CONFIGS[name]
    seg = wl.draw_segments(name)
    R = cfg["n_groups"] * cfg["group_size"]
    assert seg.seg_offsets.shape == (R + 1,) and seg.seg_offsets[0] == 0
    L = np.diff(seg.seg_offsets)
    kind, a, b = cfg["lengths"]
    assert L.min() >= a and L.max() <= b
    assert seg.n_tok == TOKENS[name]
    # contiguous groups: response i in group floor(i / group_size)
    assert np.array_equal(seg.group_ids, (np.arange(R) // cfg["group_size"]).astype(np.int32))
    assert seg.n_groups == cfg["n_groups"]
    if cfg["rewards"][0] == "bernoulli":
        assert set(np.unique(seg.rewards)) <= {0.0, 1.0}
        assert abs(seg.rewards.mean() - cfg["rewards"][1]) < 0.2  # loose: a few hundred draws
    else:
        assert seg.rewards.min() >= 0.0 and seg.rewards.max() < 1.0
    again = wl.draw_segments(name)
    assert np.array_equal(seg.seg_offsets, again.seg_offsets) and np.array_equal(seg.rewards, again.rewards)


def test_loguniform_lengths_cover_their_range():
    rng = np.random.Generator(np.random.PCG64(1))
    L = wl.draw_lengths(rng, 20000, ("loguniform", 128, 2048))
    assert L.min() == 128 and L.max() <= 2048
    # log-uniform: each octave holds about a quarter of the draws
    for lo in (128, 256, 512, 1024):
        frac = np.mean((L >= lo) & (L < 2 * lo))
        assert 0.2 < frac < 0.3, (lo, frac)


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 65280.0], np.float32)
    back = wl.bits_to_f32(wl.bf16_bits(x))
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to the even mantissa (1)
    assert back[0] == 1.0 and back[1] == 1.0
    # 1 + 3 * 2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: ties to 1 + 2^-6
    assert back[2] == np.float32(1.0 + 2 ** -6)
    assert back[3] == 1.0 and back[4] == -2.5 and back[5] == 65280.0


def test_matrices_have_the_stated_scales():
    H, W = wl.draw_matrices(512, 256, 2048, 7)
    h, w = wl.bits_to_f32(H).astype(np.float64), wl.bits_to_f32(W).astype(np.float64)
    assert H.shape == (512, 256) and W.shape == (2048, 256)
    assert abs(h.std() - 1.0) < 0.02 and abs(h.mean()) < 0.02
    assert abs(w.std() - 1.0 / np.sqrt(256)) < 0.02 / np.sqrt(256)
    H2, _ = wl.draw_matrices(512, 256, 2048, 7)
    assert np.array_equal(H, H2)


def test_lag_noise():
    lp = np.zeros(200000)
    e = wl.rollout_logprobs_with_lag(lp, ("normal", 0.05), 3).astype(np.float64)
    assert abs(e.std() - 0.05) < 0.002 and abs(e.mean()) < 0.002
    t = wl.rollout_logprobs_with_lag(lp, ("student_t3", 0.1), 3).astype(np.float64)
    # Student-t with 3 degrees of freedom: variance 3 (scaled by 0.1^2), heavy tails
    assert np.median(np.abs(t)) < 0.1 and np.abs(t).max() > 1.0
    assert np.array_equal(t, wl.rollout_logprobs_with_lag(lp, ("student_t3", 0.1), 3))


def test_token_cap_keeps_whole_groups():
    p = wl.full_config("tiny", device="cpu", n_tok_cap=200)
    gs = wl.CONFIGS["tiny"]["group_size"]
    R = p.seg.seg_offsets.shape[0] - 1
    assert R % gs == 0 and R >= gs
    assert p.n_tok == int(p.seg.seg_offsets[-1])


def test_sampler_draws_tokens_at_temperature_one():
    """Gumbel-max: the frequency of each token for a repeated row matches softmax(z)."""
    import torch
    V, reps = 6, 30000
    z_target = torch.tensor([0.0, 1.0, -1.0, 2.0, 0.5, -3.0])
    # H = e_0 and W[:, 0] = z: the logits of every row are z (exact in bf16)
    H = torch.zeros((reps, 8), dtype=torch.bfloat16)
    H[:, 0] = 1.0
    W = torch.zeros((V, 8), dtype=torch.bfloat16)
    W[:, 0] = z_target.to(torch.bfloat16)
    ids = wl.rollout_sample_ids(H, W, seed=5, chunk=4096)
    freq = np.bincount(ids.numpy(), minlength=V) / reps
    p = torch.softmax(z_target.double(), 0).numpy()
    # binomial standard error at 30000 draws is below 0.003 for every p
    assert np.all(np.abs(freq - p) < 5 * np.sqrt(p * (1 - p) / reps) + 1e-4), (freq, p)
    assert np.array_equal(ids.numpy(), wl.rollout_sample_ids(H, W, seed=5, chunk=4096).numpy())
