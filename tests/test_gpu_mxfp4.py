"""The MXFP4 forward through the C ABI: rz_quantize_rows_mxfp4 bit for bit against the
oracle's OCP Microscaling quantiser (E2M1 codes and UE8M0 block scales), and
rz_token_logprobs_mxfp4 against the fp64 oracle's logprobs of the decoded operands (|dlp| <=
2e-3), bitwise batch-invariant across rows alone, prefill chunks and a permutation.

The tensor cores multiply E2M1 values and apply the power-of-two block scales exactly and
accumulate in fp32, so the only difference from the oracle is fp32 accumulation and the
log-sum-exp arithmetic shared with the bf16 forward."""
import math

import numpy as np
import pytest
import torch

import workloads as wl
from oracle import dense, mxfp4
from tests import helpers as h

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rz():
    from invariant_logprobs_reinforce_b200 import build
    build.build()
    import invariant_logprobs_reinforce_b200 as rz
    return rz


def untile_scales(tiled: np.ndarray, rows: int, d: int) -> np.ndarray:
    """[rows, d/32] scale bytes from the tiled layout of include/rz.h."""
    r = np.arange(rows)[:, None]
    k = np.arange(d // 32)[None, :]
    off = ((r // 128) * (d // 128) + k // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + k % 4
    return tiled[off]


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """[rows, d] E2M1 codes from bytes holding element 2j in the low nibble."""
    out = np.empty((packed.shape[0], packed.shape[1] * 2), np.uint8)
    out[:, 0::2] = packed & 0x0F
    out[:, 1::2] = packed >> 4
    return out


def _hard_rows(rows, d, seed):
    """bf16 rows that reach every branch of the quantiser: ordinary blocks over many
    magnitudes, all-zero blocks, blocks of tiny (subnormal) values, exact rounding ties,
    negative zeros and values that saturate."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, d)).astype(np.float32)
    x *= np.exp2(rng.integers(-20, 20, size=(rows, d // 32))).repeat(32, axis=1).astype(np.float32)
    x[0, :32] = 0.0                                  # an all-zero block
    if rows < 4:
        return wl.bf16_bits(x)
    x[1, :32] = np.float32(3e-39) * rng.standard_normal(32).astype(np.float32)  # subnormal block
    # exact ties at the block scale 1 (block maximum 4): 0.25, 0.75, ..., 5 and their negatives
    ties = np.array([4.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, 0.0, -0.0,
                     0.5, 1.0, 1.5, 2.0, 3.0, -4.0, 0.3, -0.1, 0.2, 2.4, 2.6, 3.4, 3.6, 0.74, 0.76, 1.26, 1.74],
                    np.float32)
    x[2, :32] = ties
    x[3, 32:64] = -0.0                               # negative zeros only
    return wl.bf16_bits(x)


@pytest.mark.parametrize("rows,d", [(300, 512), (1, 256), (257, 7168)])
def test_quantiser_matches_the_oracle_bit_for_bit(rz, rows, d):
    bits = _hard_rows(rows, d, 7)
    X = h.bits_to_torch_bf16(bits, "cuda")
    q, sc = rz.rz_quantize_rows_mxfp4(X)
    torch.cuda.synchronize()
    codes_o, scales_o = mxfp4.quantize_rows_mxfp4(bits)
    codes = unpack_codes(q.cpu().numpy())
    scales = untile_scales(sc.cpu().numpy(), rows, d)
    assert np.array_equal(scales, scales_o)
    assert np.array_equal(codes, codes_o)
    # the padding rows up to a multiple of 256 carry zero scales
    pad = (rows + 255) // 256 * 256
    if pad > rows:
        rr = np.arange(rows, pad)[:, None]
        k = np.arange(d // 32)[None, :]
        off = ((rr // 128) * (d // 128) + k // 4) * 512 + (rr % 32) * 16 + ((rr % 128) // 32) * 4 + k % 4
        assert not np.any(sc.cpu().numpy()[off])
    assert sc.numel() == rz.rz_mxfp4_scale_bytes(rows, d)


def _decoded_bits(codes, scales):
    """bf16 bit patterns of the decoded MXFP4 values (exactly representable in bf16)."""
    v = mxfp4.decode_mxfp4(codes, scales)
    b = wl.bf16_bits(v.astype(np.float32))
    assert np.array_equal(dense.bf16_bits_to_f64(b), v)
    return b


def _operands(rz, n, d, V, seed):
    H, W = wl.draw_matrices(n, d, V, seed, device="cuda")
    ids = torch.from_numpy(wl.draw_uniform_ids(n, V, seed)).cuda()
    H4, hs = rz.rz_quantize_rows_mxfp4(H)
    W4, ws = rz.rz_quantize_rows_mxfp4(W)
    return H, W, ids, H4, hs, W4, ws


def oracle_decoded_chunk(bits):
    """The oracle's MXFP4 quantisation of some rows, decoded, as bf16 bits (a process-pool task)."""
    codes, scales = mxfp4.quantize_rows_mxfp4(bits)
    return _decoded_bits(codes, scales)


@pytest.fixture(scope="module")
def pool():
    """Host processes for the oracle, started with spawn (a forked child of a process that has
    used CUDA can hang); the oracle is row-wise, so row ranges go to the workers."""
    import concurrent.futures
    import multiprocessing
    import os
    workers = max(1, min(16, os.cpu_count() or 1))
    with concurrent.futures.ProcessPoolExecutor(workers, mp_context=multiprocessing.get_context("spawn")) as ex:
        yield ex


def _oracle_operand(X, pool, rows_per_call=2048):
    """bf16 bits of the oracle's decoded MXFP4 quantisation of X, row range by row range."""
    bits = X.view(torch.int16).cpu().numpy().view(np.uint16)
    chunks = [bits[r0:r0 + rows_per_call] for r0 in range(0, bits.shape[0], rows_per_call)]
    return np.concatenate(list(pool.map(oracle_decoded_chunk, chunks)), axis=0)


def _oracle_lp(H, W, ids, pool):
    return dense.token_logprobs(_oracle_operand(H, pool), _oracle_operand(W, pool), ids.cpu().numpy())


@pytest.mark.parametrize("n,d,V,seed", [
    (1, 256, 300, 11),          # a single row, one partial vocabulary tile
    (300, 256, 5000, 12),       # three segments, ragged row block and vocabulary tail
    (700, 1536, 9000, 13),      # several row blocks and segments at a real d
    (512, 2560, 151936, 14),    # the Qwen3-4B head
    (256, 7168, 129280, 15),    # the MoE head
])
def test_logprobs_match_the_oracle_on_the_decoded_operands(rz, pool, n, d, V, seed):
    H, W, ids, H4, hs, W4, ws = _operands(rz, n, d, V, seed)
    lp, lse = rz.rz_token_logprobs_mxfp4(H4, hs, W4, ws, ids)
    torch.cuda.synchronize()
    lp_o, lse_o = _oracle_lp(H, W, ids, pool)
    assert np.abs(lp.cpu().numpy() - lp_o).max() <= h.LP_ATOL
    assert np.abs(lse.cpu().numpy() - lse_o).max() <= h.LP_ATOL


def test_zero_head_gives_minus_log_V(rz):
    n, d, V = 200, 512, 5000
    H = torch.randn((n, d), device="cuda").to(torch.bfloat16)
    W = torch.zeros((V, d), dtype=torch.bfloat16, device="cuda")
    ids = torch.randint(0, V, (n,), device="cuda", dtype=torch.int32)
    H4, hs = rz.rz_quantize_rows_mxfp4(H)
    W4, ws = rz.rz_quantize_rows_mxfp4(W)
    lp, lse = rz.rz_token_logprobs_mxfp4(H4, hs, W4, ws, ids)
    assert torch.allclose(lp.double(), torch.full_like(lp.double(), -math.log(V)), atol=4e-6, rtol=0)
    assert torch.allclose(lse.double(), torch.full_like(lse.double(), math.log(V)), atol=4e-6, rtol=0)


def test_batch_invariance_alone_chunks_permuted(rz):
    n, d, V = 2048, 1536, 151936
    H, W, ids, H4, hs, W4, ws = _operands(rz, n, d, V, 21)
    ref, _ = rz.rz_token_logprobs_mxfp4(H4, hs, W4, ws, ids)
    ref_bits = ref.view(torch.int32)
    g = torch.Generator().manual_seed(5)
    # rows alone (each row quantised on its own: a row's codes and scales depend only on the row)
    for r in torch.randperm(n, generator=g)[:24].tolist():
        h4, s1 = rz.rz_quantize_rows_mxfp4(H[r:r + 1])
        lp1, _ = rz.rz_token_logprobs_mxfp4(h4, s1, W4, ws, ids[r:r + 1])
        assert torch.equal(lp1.view(torch.int32), ref_bits[r:r + 1]), r
    # prefill chunks
    for c in (64, 512):
        out = torch.empty(n, device="cuda")
        for c0 in range(0, n, c):
            h4, s1 = rz.rz_quantize_rows_mxfp4(H[c0:c0 + c])
            rz.rz_token_logprobs_mxfp4(h4, s1, W4, ws, ids[c0:c0 + c], lp_out=out[c0:c0 + c], want_lse=False)
        assert torch.equal(out.view(torch.int32), ref_bits), c
    # a permutation of the batch
    perm = torch.randperm(n, generator=g).cuda()
    h4, s1 = rz.rz_quantize_rows_mxfp4(H[perm].contiguous())
    lpp, _ = rz.rz_token_logprobs_mxfp4(h4, s1, W4, ws, ids[perm].contiguous())
    assert torch.equal(lpp.view(torch.int32), ref_bits[perm])
