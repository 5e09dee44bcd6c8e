"""Pins of the MXFP4 reference (oracle/mxfp4.py; CPU only) against the OCP Microscaling
v1.0 definitions written out here independently: the E2M1 bit layout over all 16 codes,
the E8M0 block exponent rule, brute-force nearest rounding with ties to even, hand-worked
ties, saturation, zero blocks, and the quantise-then-decode round trip."""
import math

import numpy as np
import pytest

import workloads as wl
from oracle import mxfp4


def e2m1_by_definition(code: int) -> float:
    """Sign bit 3; exponent bits 2..1 with bias 1; mantissa bit 0.  Exponent 0 is subnormal
    (m * 0.5); otherwise (1 + m / 2) * 2^(e - 1)."""
    s = -1.0 if code & 8 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    return s * (m * 0.5 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1))


VALUES = np.array([e2m1_by_definition(c) for c in range(16)])


def _rows(x):
    return wl.bf16_bits(np.asarray(x, np.float32))


def test_e2m1_table_matches_the_bit_layout():
    codes = np.arange(16, dtype=np.uint8).reshape(1, 16)
    codes = np.concatenate([codes, codes], axis=1)                # one 32-element block
    dec = mxfp4.decode_mxfp4(codes, np.array([[127]], np.uint8))  # scale 2^0
    assert np.array_equal(dec[0, :16], VALUES)
    assert sorted(set(np.abs(VALUES))) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert mxfp4.E2M1_MAX == VALUES.max()


def test_block_exponent_puts_the_block_maximum_in_4_to_8():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((16, 128)) * np.exp2(rng.integers(-30, 30, (16, 128)))
    bits = _rows(X)
    xf = wl.bits_to_f32(bits).astype(np.float64)
    _, sc = mxfp4.quantize_rows_mxfp4(bits)
    Xe = sc.astype(np.int64) - 127
    amax = np.abs(xf).reshape(16, 4, 32).max(axis=2)
    ratio = amax / np.exp2(Xe.astype(np.float64))
    assert np.all((ratio >= 4.0) & (ratio < 8.0))
    # by the definition: X = floor(log2 amax) - 2
    assert np.array_equal(Xe, np.floor(np.log2(amax)).astype(np.int64) - 2)


def test_codes_are_the_nearest_e2m1_value_with_ties_to_even():
    rng = np.random.default_rng(4)
    X = rng.standard_normal((8, 256)) * np.exp2(rng.uniform(-4, 4, (8, 256)))
    bits = _rows(X)
    q, sc = mxfp4.quantize_rows_mxfp4(bits)
    y = wl.bits_to_f32(bits).astype(np.float64) / np.exp2(np.repeat(sc.astype(np.float64) - 127, 32, axis=1))
    mags = np.abs(VALUES[:8])
    dist = np.abs(np.abs(y)[..., None] - mags)
    best = dist.min(axis=-1)
    got = np.abs(VALUES[q])
    assert np.array_equal(np.abs(np.abs(y) - got), best)
    ties = (dist == best[..., None]).sum(-1) > 1
    assert np.all((q[ties] & 1) == 0)
    assert np.array_equal(q >> 3, np.signbit(y).astype(np.uint8))


@pytest.mark.parametrize("x,mag", [
    (0.25, 0.0),   # 0 | 0.5: even code 0
    (0.75, 1.0),   # 0.5 | 1: even code 2
    (1.25, 1.0),   # 1 | 1.5: even code 2
    (1.75, 2.0),   # 1.5 | 2: even code 4
    (2.5, 2.0),    # 2 | 3: even code 4
    (3.5, 4.0),    # 3 | 4: even code 6
    (5.0, 4.0),    # 4 | 6: even code 6
    (7.5, 6.0),    # above the largest value: saturates
    (-5.0, -4.0),
])
def test_hand_worked_ties_and_saturation(x, mag):
    # the block maximum 7.5 gives X = floor(log2 7.5) - 2 = 0: scale 1
    row = np.full((1, 32), 0.5, np.float32)
    row[0, 0] = 7.5
    row[0, 1] = x
    q, sc = mxfp4.quantize_rows_mxfp4(_rows(row))
    assert sc[0, 0] == 127
    assert VALUES[q[0, 1]] == mag


def test_zero_block_and_sign_of_zero():
    row = np.zeros((1, 64), np.float32)
    row[0, 32:] = 1.0
    row[0, 5] = -0.0
    q, sc = mxfp4.quantize_rows_mxfp4(_rows(row))
    assert sc[0, 0] == 0 and sc[0, 1] == 127 - 2  # zero block: X = -127; ones: floor(log2 1) - 2
    assert np.all(q[0, :32] & 7 == 0) and q[0, 5] == 8
    assert np.all(mxfp4.decode_mxfp4(q, sc)[0, 32:] == 1.0)


def test_round_trip_error_is_within_half_a_step():
    """|decode(quantise(x)) - x| is at most half the E2M1 spacing around x / 2^X (0.25,
    0.5 or 1 times the scale), except above 6 where it saturates."""
    rng = np.random.default_rng(8)
    X = rng.standard_normal((4, 512)).astype(np.float32)
    bits = _rows(X)
    xf = wl.bits_to_f32(bits).astype(np.float64)
    q, sc = mxfp4.quantize_rows_mxfp4(bits)
    dec = mxfp4.decode_mxfp4(q, sc)
    s = np.exp2(np.repeat(sc.astype(np.float64) - 127, 32, axis=1))
    y = np.abs(xf) / s
    half = np.where(y < 2, 0.25, np.where(y < 4, 0.5, 1.0))
    within = np.abs(dec - xf) <= half * s
    assert np.all(within | (y > 6.0))
    assert np.all(np.abs(dec[y > 6.0]) == 6.0 * s[y > 6.0])


def test_rejects_rows_that_are_not_whole_blocks():
    with pytest.raises(ValueError):
        mxfp4.quantize_rows_mxfp4(_rows(np.ones((1, 48), np.float32)))


def test_lm_head_from_mxfp4_operands_matches_the_decoded_fp64_head():
    """What an MXFP4 LM-head kernel must reproduce: logprobs of the decoded operands, which
    the fp64 oracle takes as given (its fp64-operand path is pinned separately)."""
    import oracle
    rng = np.random.default_rng(9)
    H = _rows(rng.standard_normal((6, 64)))
    W = _rows(rng.standard_normal((50, 64)) / 8)
    ids = rng.integers(0, 50, 6).astype(np.int32)
    Hq, Hs = mxfp4.quantize_rows_mxfp4(H)
    Wq, Ws = mxfp4.quantize_rows_mxfp4(W)
    Hd, Wd = mxfp4.decode_mxfp4(Hq, Hs), mxfp4.decode_mxfp4(Wq, Ws)
    lp, lse = oracle.token_logprobs(Hd, Wd, ids)
    z = Hd @ Wd.T
    ref_lse = np.array([math.log(np.exp(r - r.max()).sum()) + r.max() for r in z])
    assert np.allclose(lse, ref_lse, rtol=0, atol=1e-12)
    assert np.allclose(lp, z[np.arange(6), ids] - ref_lse, rtol=0, atol=1e-12)
