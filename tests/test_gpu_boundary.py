"""Boundary behaviour on the GPU: device-checked inputs set status bits and never trap,
argument errors enqueue nothing, optional outputs may be omitted, empty calls are no-ops."""
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


@pytest.fixture(scope="module")
def prob():
    p = wl.custom(2, 3, ("uniform", 30, 80), 256, 3000, seed=301)
    return p, h.to_device(p)


def test_bad_token_ids_flag_and_nan_only_their_rows(rz, prob):
    p, dev = prob
    good_lp, _ = rz.rz_token_logprobs(dev["H"], dev["W"], dev["ids"])
    ids = dev["ids"].clone()
    ids[5] = p.V
    ids[7] = -1
    ws = torch.empty(rz.rz_workspace_bytes_logprobs(p.n_tok, p.d, p.V), dtype=torch.uint8, device="cuda")
    lp, lse = rz.rz_token_logprobs(dev["H"], dev["W"], ids, workspace=ws)
    code, bits = rz.rz_read_device_status(ws)
    assert code == 5  # RZ_ERR_DEVICE_CHECK
    assert bits & 1
    assert torch.isnan(lp[5]) and torch.isnan(lp[7])
    keep = torch.ones(p.n_tok, dtype=torch.bool, device="cuda")
    keep[5] = keep[7] = False
    assert torch.equal(lp[keep].view(torch.int32), good_lp[keep].view(torch.int32))
    # the next call on the same workspace starts from a clean status
    rz.rz_token_logprobs(dev["H"], dev["W"], dev["ids"], workspace=ws)
    assert rz.rz_read_device_status(ws) == (0, 0)


def _loss_status(rz, p, dev, **over):
    args = dict(rewards=dev["rewards"], seg_offsets=dev["seg_offsets"], group_ids=dev["group_ids"],
                n_groups=p.seg.n_groups)
    args.update(over)
    lr = torch.full((p.n_tok,), -8.0, device="cuda")
    out = rz.rz_loss_fwd_bwd(dev["H"], dev["W"], dev["ids"], lr, args["rewards"], args["seg_offsets"],
                             args["group_ids"], args["n_groups"])
    return rz.rz_read_device_status(out["workspace"])


def test_bad_segments_and_groups_are_flagged(rz, prob):
    p, dev = prob
    assert _loss_status(rz, p, dev) == (0, 0)
    off = dev["seg_offsets"].clone()
    off[-1] += 1  # does not end at n_tok
    code, bits = _loss_status(rz, p, dev, seg_offsets=off)
    assert code == 5 and bits & 2
    off = dev["seg_offsets"].clone()
    off[2] = off[1]  # empty response
    code, bits = _loss_status(rz, p, dev, seg_offsets=off)
    assert code == 5 and bits & 2
    gid = dev["group_ids"].clone()
    gid[0] = p.seg.n_groups  # out of range
    code, bits = _loss_status(rz, p, dev, group_ids=gid)
    assert code == 5 and bits & 4


def test_argument_errors_enqueue_nothing(rz, prob):
    p, dev = prob
    lp = torch.full((p.n_tok,), 3.0, device="cuda")
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(rz.RZError) as e:
        rz.rz_token_logprobs(dev["H"], dev["W"], dev["ids"], lp_out=lp, workspace=small)
    assert e.value.code == 3
    buf = torch.empty(p.n_tok * p.d + 1, dtype=torch.bfloat16, device="cuda")
    H_mis = buf[1:].view(p.n_tok, p.d)
    H_mis.copy_(dev["H"])
    with pytest.raises(rz.RZError) as e:
        rz.rz_token_logprobs(H_mis, dev["W"], dev["ids"], lp_out=lp)
    assert e.value.code == 1
    torch.cuda.synchronize()
    assert torch.all(lp == 3.0)


def test_optional_outputs_and_empty_call(rz, prob):
    p, dev = prob
    lp, lse = rz.rz_token_logprobs(dev["H"], dev["W"], dev["ids"], want_lse=False)
    assert lse is None and torch.isfinite(lp).all()
    lr = torch.full((p.n_tok,), -8.0, device="cuda")
    out = rz.rz_loss_fwd_bwd(dev["H"], dev["W"], dev["ids"], lr, dev["rewards"], dev["seg_offsets"],
                             dev["group_ids"], p.seg.n_groups, want_lp=False, want_kappa=False)
    assert out["lp"] is None and torch.isfinite(out["dW"]).all()
    H0 = torch.empty((0, p.d), dtype=torch.bfloat16, device="cuda")
    ids0 = torch.empty((0,), dtype=torch.int32, device="cuda")
    lp0, _ = rz.rz_token_logprobs(H0, dev["W"], ids0)
    assert lp0.numel() == 0


def test_bounded_wait_gives_up_and_reports_timeout(rz):
    """A wait on a barrier nothing arrives on ends after its limit with the timeout status;
    the context stays usable (a normal call follows)."""
    code, bits, waited = rz.rz_selftest_wait_timeout(50_000_000)  # 50 ms
    assert code == 6 and bits & 8  # RZ_ERR_DEVICE_TIMEOUT, RZ_DEV_WAIT_TIMEOUT
    assert 50_000_000 <= waited < 2_000_000_000
    H = torch.randn(10, 64, device="cuda").to(torch.bfloat16)
    W = torch.randn(100, 64, device="cuda").to(torch.bfloat16)
    ids = torch.randint(0, 100, (10,), device="cuda", dtype=torch.int32)
    lp, _ = rz.rz_token_logprobs(H, W, ids)
    assert torch.isfinite(lp).all()
