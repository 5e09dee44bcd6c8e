"""The e4m3 (fp8) forward: quantisation codes bit-exact against the reference, logprobs
against the fp64 oracle on the dequantised operands, and the batch-invariance contract."""
import numpy as np
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


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def test_quantisation_codes_are_bit_exact(rz, oracle):
    g = torch.Generator(device="cuda")
    g.manual_seed(1)
    X = torch.randn((300, 384), generator=g, device="cuda")
    X[7] = 0.0
    X[11] *= 1e4
    X[12] *= 1e-6
    Xb = X.to(torch.bfloat16)
    q, sc = rz.rz_quantize_rows_e4m3(Xb)
    q_o, sc_o = oracle.quantize_rows_e4m3(_bits(Xb))
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), sc_o.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_o)


def _fp8_problem(rz, p):
    dev = h.to_device(p)
    H8, hs = rz.rz_quantize_rows_e4m3(dev["H"])
    W8, ws = rz.rz_quantize_rows_e4m3(dev["W"])
    return dev, H8, hs, W8, ws


@pytest.mark.parametrize("shape", [(2, 4, (16, 64), 256, 4096, 101), (3, 3, (20, 90), 128, 5000, 201),
                                   (1, 2, (1, 3), 384, 7, 202), (2, 3, (10, 40), 256, 3003, 207)])
def test_fp8_logprobs_against_oracle(rz, oracle, shape):
    g_, gs, lengths, d, V, seed = shape
    p = wl.custom(g_, gs, ("uniform",) + tuple(lengths), d, V, seed)
    dev, H8, hs, W8, ws = _fp8_problem(rz, p)
    lp, lse = rz.rz_token_logprobs_fp8(H8, hs, W8, ws, dev["ids"])
    Hd = oracle.decode_e4m3(H8.cpu().numpy()) * hs.cpu().numpy().astype(np.float64)[:, None]
    Wd = oracle.decode_e4m3(W8.cpu().numpy()) * ws.cpu().numpy().astype(np.float64)[:, None]
    lp_o, lse_o = oracle.token_logprobs(Hd, Wd, p.ids)
    assert np.abs(lp.cpu().numpy() - lp_o).max() <= h.LP_ATOL
    assert np.abs(lse.cpu().numpy() - lse_o).max() <= h.LP_ATOL


def test_fp8_same_bits_with_unaligned_column_scales(rz):
    """Column scales at a 4-byte (not 16-byte) aligned address take the scalar loads; the
    logits and so the logprobs must not change by a bit.  V = 3003 leaves a ragged last tile."""
    p = wl.custom(2, 3, ("uniform", 10, 40), 256, 3003, 208)
    dev, H8, hs, W8, ws = _fp8_problem(rz, p)
    buf = torch.zeros(ws.numel() + 1, dtype=torch.float32, device="cuda")
    buf[1:] = ws
    ws_off = buf[1:]
    assert ws.data_ptr() % 16 == 0 and ws_off.data_ptr() % 16 == 4
    lp_a, lse_a = rz.rz_token_logprobs_fp8(H8, hs, W8, ws, dev["ids"])
    lp_b, lse_b = rz.rz_token_logprobs_fp8(H8, hs, W8, ws_off, dev["ids"])
    assert torch.equal(lp_a.view(torch.int32), lp_b.view(torch.int32))
    assert torch.equal(lse_a.view(torch.int32), lse_b.view(torch.int32))


def test_fp8_zero_head(rz):
    H = torch.randn(100, 256, device="cuda").to(torch.bfloat16)
    W = torch.zeros(3000, 256, device="cuda", dtype=torch.bfloat16)
    H8, hs = rz.rz_quantize_rows_e4m3(H)
    W8, ws = rz.rz_quantize_rows_e4m3(W)
    ids = torch.randint(0, 3000, (100,), device="cuda", dtype=torch.int32)
    lp, _ = rz.rz_token_logprobs_fp8(H8, hs, W8, ws, ids)
    assert torch.allclose(lp.double(), torch.full_like(lp.double(), -np.log(3000)), atol=4e-6, rtol=0)


def test_fp8_batch_invariance(rz):
    cfg = wl.CONFIGS["invariance"]
    d, V = cfg["d"], cfg["V"]
    H, W = wl.draw_matrices(1024, d, V, cfg["seed"], device="cuda")
    ids = torch.from_numpy(wl.draw_uniform_ids(1024, V, cfg["seed"])).cuda()
    H8, hs = rz.rz_quantize_rows_e4m3(H)
    W8, ws = rz.rz_quantize_rows_e4m3(W)
    ref, ref_lse = rz.rz_token_logprobs_fp8(H8, hs, W8, ws, ids)
    rng = np.random.default_rng(2)
    lp = torch.empty_like(ref)
    for i in rng.choice(1024, 48, replace=False):  # single rows (decode calls)
        rz.rz_token_logprobs_fp8(H8[i:i + 1], hs[i:i + 1], W8, ws, ids[i:i + 1], lp_out=lp[i:i + 1], want_lse=False)
        torch.cuda.synchronize()
        assert lp[i].view(torch.int32).item() == ref[i].view(torch.int32).item()
    for chunk in (64, 333):  # prefill chunks
        for c0 in range(0, 1024, chunk):
            c1 = min(1024, c0 + chunk)
            rz.rz_token_logprobs_fp8(H8[c0:c1], hs[c0:c1], W8, ws, ids[c0:c1], lp_out=lp[c0:c1], want_lse=False)
        torch.cuda.synchronize()
        assert torch.equal(lp.view(torch.int32), ref.view(torch.int32))
    perm = torch.from_numpy(rng.permutation(1024)).cuda()
    lpp, _ = rz.rz_token_logprobs_fp8(H8[perm].contiguous(), hs[perm].contiguous(), W8, ws, ids[perm].contiguous())
    assert torch.equal(lpp.view(torch.int32), ref[perm].view(torch.int32))
