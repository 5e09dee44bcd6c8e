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


def test_noalloc_out_of_range_ids_give_nan_rows_only(rz):
    # the bad-id path sets its status bit in the shared scratch (internal here): the rows
    # with an id outside [0, V) are NaN, every other row is bit-equal to the workspace call
    n, d, V = 400, 512, 9000
    H, W, ids = _problem(n, d, V, 4)
    bad = torch.tensor([7, 200], device="cuda")
    ids[bad[0]] = V
    ids[bad[1]] = -1
    lp = torch.empty(n, device="cuda")
    lse = torch.empty(n, device="cuda")
    assert _noalloc(rz, H, W, ids, lp, lse) == 0
    ref_lp, ref_lse = rz.rz_token_logprobs(H, W, ids)
    torch.cuda.synchronize()
    good = torch.ones(n, dtype=torch.bool, device="cuda")
    good[bad] = False
    assert torch.isnan(lp[bad]).all()
    assert torch.equal(lp[good].view(torch.int32), ref_lp[good].view(torch.int32))
    assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32))
    # and the next call, with valid ids, is clean again
    ids[bad] = 3
    assert _noalloc(rz, H, W, ids, lp, lse) == 0
    ref_lp, _ = rz.rz_token_logprobs(H, W, ids)
    torch.cuda.synchronize()
    assert torch.equal(lp.view(torch.int32), ref_lp.view(torch.int32))


@pytest.mark.parametrize("use_scratch", [True, False])
def test_wait_that_gave_up_gives_nan_not_stale_values(rz, use_scratch):
    # a wait that gives up leaves partials unwritten; the scratch then still holds the
    # previous call's partials of the same rows.  The merge must not turn those into
    # plausible logprobs: every lp and lse of the call comes out NaN.
    n, d, V = 300, 256, 5000
    H, W, ids = _problem(n, d, V, 5)
    lp = torch.empty(n, device="cuda")
    lse = torch.empty(n, device="cuda")
    assert _noalloc(rz, H, W, ids, lp, lse) == 0  # leaves this shape's partials in the scratch
    torch.cuda.synchronize()
    assert torch.isfinite(lp).all()
    lp_t, lse_t, code, bits = rz.rz_selftest_forward_after_timeout(H, W, ids, use_noalloc_scratch=use_scratch)
    torch.cuda.synchronize()
    assert torch.isnan(lp_t).all() and torch.isnan(lse_t).all()
    if not use_scratch:
        assert code == 6 and bits & 8  # RZ_ERR_DEVICE_TIMEOUT, RZ_DEV_WAIT_TIMEOUT
    # the next ordinary call is correct again
    lp2 = torch.empty(n, device="cuda")
    assert _noalloc(rz, H, W, ids, lp2, None) == 0
    torch.cuda.synchronize()
    assert torch.equal(lp2.view(torch.int32), lp.view(torch.int32))
