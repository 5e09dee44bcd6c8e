"""The loss stage and the ratio statistics at a size where every persistent CTA takes many
4096-token blocks (about 2^23 tokens: seven or more blocks per CTA, so every shared-memory
stage is refilled several times), with a ragged last block: the bulk-copied path (16-byte
aligned inputs) against the path that reads global memory (the same values 4 bytes into a
fresh buffer) bit for bit, with and without a token mask, and both against the fp64
oracle."""
import numpy as np
import pytest
import torch

import oracle as orc

pytestmark = pytest.mark.gpu

N_TOK = (1 << 23) + 777


@pytest.fixture(scope="module")
def rz():
    import invariant_logprobs_reinforce_b200 as rz
    from invariant_logprobs_reinforce_b200 import build
    build.build()
    return rz


@pytest.fixture(scope="module")
def inputs():
    rng = np.random.default_rng(123)
    L = rng.integers(64, 4097, size=N_TOK // 64 + 1)
    c = np.cumsum(L)
    R = int(np.searchsorted(c, N_TOK)) + 1
    L = L[:R].copy()
    L[-1] -= int(c[R - 1] - N_TOK)
    assert L[-1] >= 1 and int(L.sum()) == N_TOK
    off = np.zeros(R + 1, np.int64)
    off[1:] = np.cumsum(L)
    gid = (np.arange(R) // 16).astype(np.int32)
    G = int(gid[-1]) + 1
    rewards = rng.standard_normal(R).astype(np.float32)
    lp = (-rng.exponential(2.0, N_TOK)).astype(np.float32)
    lr = (lp + 0.05 * rng.standard_normal(N_TOK)).astype(np.float32)
    mask = (rng.uniform(size=N_TOK) < 0.85).astype(np.uint8)
    return dict(off=off, gid=gid, G=G, rewards=rewards, lp=lp, lr=lr, mask=mask)


def _t(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _shifted(x, dtype):
    """x 4 bytes into a fresh buffer: 4-byte aligned (what the calls require), not 16-byte."""
    k = 4 // x.element_size()
    buf = torch.zeros(x.numel() + k, dtype=dtype, device="cuda")
    buf[k:] = x
    return buf[k:]


@pytest.mark.parametrize("masked", [False, True])
def test_segment_loss_streamed_equals_global_path_and_oracle(rz, inputs, masked):
    I = inputs
    lp, lr, mask = _t(I["lp"]), _t(I["lr"]), _t(I["mask"])
    r, off, gid = _t(I["rewards"]), _t(I["off"]), _t(I["gid"])
    outs = []
    for a_lp, a_lr, a_m in ((lp, lr, mask), (_shifted(lp, torch.float32), _shifted(lr, torch.float32),
                                               _shifted(mask, torch.uint8))):
        assert (a_lp.data_ptr() % 16 == 0) == (len(outs) == 0)
        opts = rz.loss_options(token_mask=a_m if masked else None)
        out = rz.rz_segment_loss_ex(a_lp, a_lr, r, off, gid, I["G"], opts)
        assert rz.rz_read_device_status(out["workspace"]) == (0, 0)
        outs.append((out["loss"].item(), out["kappa"]))
    assert torch.equal(outs[0][1].view(torch.int32), outs[1][1].view(torch.int32))
    assert np.float32(outs[0][0]).view(np.int32) == np.float32(outs[1][0]).view(np.int32)
    loss_o, _, kappa_o = orc.loss_from_lp_ex(I["lp"], I["lr"], I["rewards"], I["off"], I["gid"], I["G"],
                                             flags=orc.MASK if masked else 0, mask=I["mask"] if masked else None)
    np.testing.assert_allclose(outs[0][1].cpu().numpy(), kappa_o, rtol=1e-5, atol=1e-30)
    scale = float(np.sum(np.abs(kappa_o)))
    assert abs(outs[0][0] - loss_o) <= 1e-4 * max(abs(loss_o), scale)


@pytest.mark.parametrize("masked", [False, True])
def test_ratio_stats_streamed_equals_global_path_and_oracle(rz, inputs, masked):
    I = inputs
    lp, lr, mask, off = _t(I["lp"]), _t(I["lr"]), _t(I["mask"]), _t(I["off"])
    sa, ra = rz.rz_ratio_stats(lp, lr, off, token_mask=mask if masked else None)
    sb, rb = rz.rz_ratio_stats(_shifted(lp, torch.float32), _shifted(lr, torch.float32), off,
                               token_mask=_shifted(mask, torch.uint8) if masked else None)
    assert torch.equal(sa.view(torch.int64), sb.view(torch.int64))
    assert torch.equal(ra.view(torch.int32), rb.view(torch.int32))
    st_o, rm_o = orc.ratio_stats(I["lp"].astype(np.float64), I["lr"].astype(np.float64), I["off"],
                                 mask=I["mask"] if masked else None)
    st = dict(zip(rz.STAT_NAMES, sa.cpu().numpy().tolist()))
    assert st["count"] == st_o["count"]
    for k in ("k1", "k2", "k3"):
        assert abs(st[k] - st_o[k]) <= 1e-9 * abs(st_o[k]) + 1e-15, k
    for k in ("w_min", "w_max", "dev_max", "dev_median"):
        assert abs(st[k] - st_o[k]) <= 2e-6 * max(1.0, abs(st_o[k])) + 1e-7, (k, st[k], st_o[k])
    np.testing.assert_allclose(ra.cpu().numpy(), rm_o, rtol=2e-6)
