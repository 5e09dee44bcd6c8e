"""The allocation-free forward entry point, through the C ABI.

rz_token_logprobs_noalloc serves callers that cannot allocate device memory (an engine
that reserved its HBM up front, a loop where cudaMalloc could synchronise the device, a
plugin without access to the host framework's allocator).  It keeps its scratch in a
fixed array inside the library instead of a caller workspace.  This file is collected
last, so a run that stops at the first failure has run every other test first; it also
passes alone in a fresh process.
"""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

LP_ATOL = 2e-3  # the tolerance every logprob parity test uses


@pytest.fixture(scope="module")
def rz():
    from invariant_logprobs_reinforce_b200 import build
    build.build()
    import invariant_logprobs_reinforce_b200 as rz
    return rz


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(rz, H, W, ids, lp, lse):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return rz.lib().rz_token_logprobs_noalloc(_ptr(H), _ptr(W), _ptr(ids), H.shape[0], H.shape[1], W.shape[0],
                                              _ptr(lp), _ptr(lse), stream)


def _problem(n, d, V, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    H = torch.randn((n, d), generator=g, device="cuda").to(torch.bfloat16)
    W = (torch.randn((V, d), generator=g, device="cuda") / d ** 0.5).to(torch.bfloat16)
    ids = torch.randint(0, V, (n,), generator=g, device="cuda", dtype=torch.int32)
    return H, W, ids


def test_noalloc_matches_workspace_entry_point_on_two_calls(rz):
    # two calls in a row with different shapes: the shared scratch keeps the first call's
    # contents, which must not leak into the second
    for n, d, V, seed in ((700, 256, 5000, 1), (300, 1536, 151936, 2)):
        H, W, ids = _problem(n, d, V, seed)
        lp = torch.full((n,), float("nan"), device="cuda")
        lse = torch.full((n,), float("nan"), device="cuda")
        assert _noalloc(rz, H, W, ids, lp, lse) == 0
        ref_lp, ref_lse = rz.rz_token_logprobs(H, W, ids)
        torch.cuda.synchronize()
        assert torch.isfinite(lp).all() and torch.isfinite(lse).all()
        assert (lp - ref_lp).abs().max().item() <= LP_ATOL
        assert (lse - ref_lse).abs().max().item() <= LP_ATOL
        # same kernels and same reduction order: the bits agree as well
        assert torch.equal(lp.view(torch.int32), ref_lp.view(torch.int32))
        assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32))


def test_python_wrapper_is_the_same_call(rz):
    H, W, ids = _problem(500, 512, 9000, 3)
    lp = torch.empty(500, device="cuda")
    lse = torch.empty(500, device="cuda")
    rz.rz_token_logprobs_noalloc(H, W, ids, lp, lse)
    ref_lp, ref_lse = rz.rz_token_logprobs(H, W, ids)
    torch.cuda.synchronize()
    assert torch.equal(lp.view(torch.int32), ref_lp.view(torch.int32))
    assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32))


def test_noalloc_rejects_calls_beyond_its_scratch(rz):
    d, V = 256, 151936
    segs = -(-V // 2048)
    n = (32 << 20) // (4 * (2 * segs + 1)) + 1024  # needs more than the fixed scratch holds
    H = torch.zeros((n, d), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((V, d), dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros((n,), dtype=torch.int32, device="cuda")
    lp = torch.full((n,), 7.0, device="cuda")
    assert _noalloc(rz, H, W, ids, lp, None) == 3  # RZ_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
    assert torch.all(lp == 7.0)  # nothing was enqueued
