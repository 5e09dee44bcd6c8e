"""rz_loss_fwd_bwd_streamed: H read from host memory chunk by chunk on a copy stream.  The
kernels are the ones of rz_loss_fwd_bwd_ex, so every output must be bit-identical to the
call with H already on the device; the tests start from a device buffer full of garbage, so
a chunk computed before its copy landed would show."""
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
    # 3 chunks of 16384 tokens and a ragged fourth
    p = wl.custom(7, 8, ("uniform", 700, 1200), 128, 3000, seed=611)
    assert p.n_tok > 3 * 16384
    return p


def _inputs(p):
    dev = h.to_device(p)
    g = torch.Generator(device="cuda")
    g.manual_seed(17)
    dev["lp_roll"] = -4.0 * torch.rand(p.n_tok, generator=g, device="cuda")
    return dev


def _garbage_like(t):
    g = torch.Generator(device="cuda")
    g.manual_seed(99)
    return torch.randn(t.shape, generator=g, device="cuda").mul_(1e3).to(t.dtype)


def _same(a, b):
    for k in ("loss", "lp", "kappa", "dW"):
        assert torch.equal(a[k].view(torch.int32), b[k].view(torch.int32)), k
    assert torch.equal(a["dH"].view(torch.int16), b["dH"].view(torch.int16))


def _call_device(rz, dev, p, options):
    return rz.rz_loss_fwd_bwd_ex(dev["H"], dev["W"], dev["ids"], dev["lp_roll"], dev["rewards"], dev["seg_offsets"],
                                 dev["group_ids"], p.seg.n_groups, options)


def _call_streamed(rz, dev, p, H_host, H_dev, options):
    return rz.rz_loss_fwd_bwd_streamed(H_host, H_dev, dev["W"], dev["ids"], dev["lp_roll"], dev["rewards"],
                                       dev["seg_offsets"], dev["group_ids"], p.seg.n_groups, options)


@pytest.mark.parametrize("pinned", [True, False])
def test_streamed_equals_device_resident(rz, prob, pinned):
    dev = _inputs(prob)
    ref = _call_device(rz, dev, prob, None)
    H_host = dev["H"].cpu()
    if pinned:
        H_host = H_host.pin_memory()
    H_dev = _garbage_like(dev["H"])
    out = _call_streamed(rz, dev, prob, H_host, H_dev, None)
    torch.cuda.synchronize()
    assert rz.rz_read_device_status(out["workspace"]) == (0, 0)
    _same(out, ref)
    assert torch.equal(H_dev.view(torch.int16), dev["H"].view(torch.int16))


def test_streamed_with_gate_waits_for_every_chunk(rz, prob):
    dev = _inputs(prob)
    opts = rz.loss_options(gate=(0.2, 5.0), clip_max=2.0)
    ref = _call_device(rz, dev, prob, opts)
    H_dev = _garbage_like(dev["H"])
    out = _call_streamed(rz, dev, prob, dev["H"].cpu().pin_memory(), H_dev, opts)
    torch.cuda.synchronize()
    _same(out, ref)


def test_back_to_back_calls_reuse_the_device_buffer(rz, prob):
    """The second call's copies must wait for the first call's kernels, which still read
    H_dev; each result equals the device-resident call on its own H."""
    dev = _inputs(prob)
    H1 = dev["H"]
    H2 = _garbage_like(H1).mul_(1e-3)
    ref1 = _call_device(rz, dev, prob, None)
    ref2 = _call_device(rz, dict(dev, H=H2), prob, None)
    h1, h2 = H1.cpu().pin_memory(), H2.cpu().pin_memory()
    H_dev = torch.empty_like(H1)
    out1 = _call_streamed(rz, dev, prob, h1, H_dev, None)
    out2 = _call_streamed(rz, dev, prob, h2, H_dev, None)
    torch.cuda.synchronize()
    _same(out1, ref1)
    _same(out2, ref2)


def test_streamed_rejects_null_host_pointer(rz, prob):
    dev = _inputs(prob)
    lib = rz.lib()
    n, d = dev["H"].shape
    code = lib.rz_loss_fwd_bwd_streamed(None, dev["H"].data_ptr(), dev["W"].data_ptr(), dev["ids"].data_ptr(),
                                        dev["lp_roll"].data_ptr(), dev["rewards"].data_ptr(),
                                        dev["seg_offsets"].data_ptr(), dev["group_ids"].data_ptr(), n,
                                        dev["rewards"].shape[0], prob.seg.n_groups, d, dev["W"].shape[0], None,
                                        None, None, None, None, None, None, 0, None)
    assert code == 1  # RZ_ERR_INVALID_ARG, nothing enqueued


@pytest.mark.parametrize("pinned", [True, False])
def test_host_io_delivers_the_gradients_to_host_memory(rz, prob, pinned):
    """rz_loss_fwd_bwd_host_io: dH chunk by chunk and dW at the end copied to host buffers
    that start as garbage; they must equal the device-resident call bit for bit."""
    dev = _inputs(prob)
    ref = _call_device(rz, dev, prob, None)
    n, d = dev["H"].shape
    V = dev["W"].shape[0]
    H_host = dev["H"].cpu()
    dH_host = torch.full((n, d), 7.0, dtype=torch.bfloat16)
    dW_host = torch.full((V, d), 7.0)
    if pinned:
        H_host, dH_host, dW_host = H_host.pin_memory(), dH_host.pin_memory(), dW_host.pin_memory()
    H_dev = _garbage_like(dev["H"])
    out = rz.rz_loss_fwd_bwd_host_io(H_host, H_dev, dev["W"], dev["ids"], dev["lp_roll"], dev["rewards"],
                                     dev["seg_offsets"], dev["group_ids"], prob.seg.n_groups, dH_host=dH_host,
                                     dW_host=dW_host)
    torch.cuda.current_stream().synchronize()  # the stream's work includes the copies
    assert rz.rz_read_device_status(out["workspace"]) == (0, 0)
    _same(out, ref)
    assert torch.equal(dH_host.view(torch.int16), ref["dH"].cpu().view(torch.int16))
    assert torch.equal(dW_host.view(torch.int32), ref["dW"].cpu().view(torch.int32))


def test_host_io_back_to_back_and_without_host_outputs(rz, prob):
    """Two calls in a row into the same host buffers: the second call's dH must not be
    copied out before its own contraction; and both host outputs may be omitted."""
    dev = _inputs(prob)
    H2 = _garbage_like(dev["H"]).mul_(1e-3)
    ref2 = _call_device(rz, dict(dev, H=H2), prob, None)
    n, d = dev["H"].shape
    V = dev["W"].shape[0]
    dH_host = torch.empty((n, d), dtype=torch.bfloat16).pin_memory()
    dW_host = torch.empty((V, d)).pin_memory()
    H_dev = torch.empty_like(dev["H"])
    for H in (dev["H"], H2):
        out = rz.rz_loss_fwd_bwd_host_io(H.cpu().pin_memory(), H_dev, dev["W"], dev["ids"], dev["lp_roll"],
                                         dev["rewards"], dev["seg_offsets"], dev["group_ids"], prob.seg.n_groups,
                                         dH_host=dH_host, dW_host=dW_host)
    torch.cuda.synchronize()
    _same(out, ref2)
    assert torch.equal(dH_host.view(torch.int16), ref2["dH"].cpu().view(torch.int16))
    assert torch.equal(dW_host.view(torch.int32), ref2["dW"].cpu().view(torch.int32))
    plain = rz.rz_loss_fwd_bwd_host_io(H2.cpu(), H_dev, dev["W"], dev["ids"], dev["lp_roll"], dev["rewards"],
                                       dev["seg_offsets"], dev["group_ids"], prob.seg.n_groups)
    torch.cuda.synchronize()
    _same(plain, ref2)
