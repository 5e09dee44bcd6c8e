"""The loss stage's setup (group reward sums and per-response coefficients) on group layouts
whose runs of equal ids cross the setup kernel's 32-response windows and 256-response blocks
in every way: kappa and the loss against the fp64 oracle, and kappa bit for bit against the
same responses under relabelled group ids that are no longer sorted (which the setup handles
by rescanning every response in index order, the plain serial sum).  Rewards are Gaussian,
so the fp64 group sums depend on the order of the additions."""
import numpy as np
import pytest
import torch

import oracle as orc

pytestmark = pytest.mark.gpu

rng0 = np.random.default_rng(77)
SIZES = {
    "ones": [1] * 300,
    "fives": [5] * 200,
    "thirty_one": [31] * 40,
    "thirty_two": [32] * 40,
    "thirty_three": [33] * 40,
    "sixty_four": [64] * 20,
    "hundred": [100] * 13,
    "big_and_small": [1000, 3, 257, 1, 64, 700, 2],
    "one_group": [3000],
    "few": [3, 4],
    "random": list(rng0.integers(1, 80, size=120)),
}


@pytest.fixture(scope="module")
def rz():
    import invariant_logprobs_reinforce_b200 as rz
    from invariant_logprobs_reinforce_b200 import build
    build.build()
    return rz


def _layout(sizes, seed):
    rng = np.random.default_rng(seed)
    gid = np.repeat(np.arange(len(sizes)), sizes).astype(np.int32)
    R = gid.size
    L = rng.integers(1, 40, size=R)
    off = np.zeros(R + 1, np.int64)
    off[1:] = np.cumsum(L)
    rewards = rng.standard_normal(R).astype(np.float32)
    n = int(off[-1])
    lp = (-rng.exponential(2.0, n)).astype(np.float32)
    lr = (lp + 0.05 * rng.standard_normal(n)).astype(np.float32)
    return gid, off, rewards, lp, lr, len(sizes)


def _call(rz, lp, lr, rewards, off, gid, G, mask=None):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    if mask is None:
        out = rz.rz_segment_loss(t(lp), t(lr), t(rewards), t(off), t(gid), G)
    else:
        out = rz.rz_segment_loss_ex(t(lp), t(lr), t(rewards), t(off), t(gid), G, rz.loss_options(token_mask=t(mask)))
    assert rz.rz_read_device_status(out["workspace"]) == (0, 0)
    return out["loss"].item(), out["kappa"].cpu().numpy()


@pytest.mark.parametrize("name", list(SIZES))
@pytest.mark.parametrize("masked", [False, True])
def test_setup_runs_across_windows(rz, name, masked):
    gid, off, rewards, lp, lr, G = _layout(SIZES[name], 5 + len(name))
    mask = None
    if masked:
        mask = (np.random.default_rng(3).uniform(size=lp.size) < 0.8).astype(np.uint8)
    loss_a, kappa_a = _call(rz, lp, lr, rewards, off, gid, G, mask)
    # the same groups under labels in decreasing order: the unsorted path
    gid_b = (G - 1 - gid).astype(np.int32)
    loss_b, kappa_b = _call(rz, lp, lr, rewards, off, gid_b, G, mask)
    assert np.array_equal(kappa_a.view(np.int32), kappa_b.view(np.int32))
    assert np.float32(loss_a).view(np.int32) == np.float32(loss_b).view(np.int32)
    loss_o, _, kappa_o = orc.loss_from_lp_ex(lp, lr, rewards, off, gid, G, flags=orc.MASK if masked else 0,
                                             mask=mask)
    np.testing.assert_allclose(kappa_a, kappa_o, rtol=1e-5, atol=1e-30)
    scale = float(np.sum(np.abs(kappa_o)))
    assert abs(loss_a - loss_o) <= 1e-4 * max(abs(loss_o), scale)
