"""Pins of the oracle's e4m3 helpers and of its fp64-operand path (CPU only).  The helpers
are checked against the OCP 8-bit floating-point definition of E4M3 ("fn" variant: no
infinities, one NaN pattern per sign), written out here bit by bit, and against brute force
over all 256 codes.  The pages name FP8 weights and reduced-precision arithmetic on the
rollout side but fix no format or scaling; the reading is per-row absmax scaling to the
e4m3 range, round to nearest even."""
import math

import numpy as np
import pytest

import oracle
import workloads as wl


def e4m3_by_definition(code: int) -> float:
    """Sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0.  Exponent 0 holds the
    subnormals m * 2^-9; S.1111.111 is NaN; everything else is (1 + m/8) * 2^(e - 7)."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


ALL_CODES = np.arange(256, dtype=np.uint8)
VALUES = np.array([e4m3_by_definition(c) for c in range(256)])
FINITE = ~np.isnan(VALUES)


def test_decode_matches_the_definition_on_all_codes():
    got = oracle.decode_e4m3(ALL_CODES)
    assert np.array_equal(np.isnan(got), np.isnan(VALUES))
    assert np.array_equal(got[FINITE], VALUES[FINITE])
    # landmarks of the format
    assert oracle.decode_e4m3(np.array([0x7E], np.uint8))[0] == 448.0          # largest finite
    assert oracle.decode_e4m3(np.array([0x08], np.uint8))[0] == 2.0 ** -6       # smallest normal
    assert oracle.decode_e4m3(np.array([0x01], np.uint8))[0] == 2.0 ** -9       # smallest subnormal
    assert oracle.E4M3_MAX == VALUES[FINITE].max()


def _bf16_rows(rows):
    return wl.bf16_bits(np.asarray(rows, np.float32))


def test_row_maximum_maps_to_the_largest_code_and_scale_is_absmax_over_448():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((64, 96)).astype(np.float32) * np.exp2(rng.integers(-20, 20, (64, 1)))
    bits = _bf16_rows(X)
    q, sc = oracle.quantize_rows_e4m3(bits)
    xb = wl.bits_to_f32(bits)
    m = np.abs(xb).max(axis=1)
    assert np.array_equal(sc, (m / np.float32(448.0)).astype(np.float32))
    i = np.abs(xb).argmax(axis=1)
    top = q[np.arange(64), i]
    assert np.all((top & 0x7F) == 0x7E)                       # |code| = 448
    assert np.array_equal(top >> 7, (xb[np.arange(64), i] < 0).astype(np.uint8))


def test_codes_are_the_nearest_value_with_ties_to_even():
    rng = np.random.default_rng(11)
    X = rng.standard_normal((32, 128)).astype(np.float32) * np.exp2(rng.uniform(-8, 8, (32, 128)))
    bits = _bf16_rows(X)
    q, sc = oracle.quantize_rows_e4m3(bits)
    y = (wl.bits_to_f32(bits) / sc[:, None]).astype(np.float64)  # the fp32 division, widened exactly
    fin = VALUES[FINITE]
    dist = np.abs(y[..., None] - fin)                              # brute force over every finite code
    best = dist.min(axis=-1)
    got = VALUES[q]
    assert not np.isnan(got).any()
    assert np.array_equal(np.abs(y - got), best)
    # at an exact tie the even mantissa wins
    ties = (dist == best[..., None]).sum(-1) > 1
    ties &= y != 0  # +0 and -0 are both nearest to 0
    assert np.all((q[ties] & 1) == 0)


@pytest.mark.parametrize("x,code", [
    (1.0 + 1 / 16, 0x38),   # halfway between 1 (m = 0) and 1.125 (m = 1): even -> 1
    (1.0 + 3 / 16, 0x3A),   # halfway between 1.125 (m = 1) and 1.25 (m = 2): even -> 1.25
    (-(1.0 + 5 / 16), 0xBA),  # halfway between -1.25 (m = 2) and -1.375 (m = 3): even -> -1.25
    (3 * 2.0 ** -10, 0x02),   # halfway between subnormals 2^-9 (m = 1) and 2^-8 (m = 2): even -> 2^-8
])
def test_hand_worked_ties(x, code):
    # scale 1: the row's maximum is 448
    row = np.array([[448.0, x]], np.float32)
    q, sc = oracle.quantize_rows_e4m3(_bf16_rows(row))
    assert sc[0] == 1.0 and q[0, 0] == 0x7E
    assert q[0, 1] == code, hex(q[0, 1])


def test_zero_row_has_scale_one_and_zero_codes():
    q, sc = oracle.quantize_rows_e4m3(_bf16_rows(np.zeros((2, 64), np.float32)))
    assert np.all(sc == 1.0) and np.all((q & 0x7F) == 0)


def test_fp64_operands_are_used_as_given():
    """The fp8 parity test hands the oracle fp64 operands (decoded codes times scales).  With
    H_t = e_k the logits are the head's column k exactly, so lp and lse have closed forms;
    the head's values are not fp32 or bf16 numbers, so any narrowing of the fp64 input path
    would show."""
    from scipy.special import logsumexp
    rng = np.random.default_rng(5)
    V, d = 40, 8
    W = rng.standard_normal((V, d)) * (1 + 1e-12)   # not representable in fp32
    assert np.any(W.astype(np.float32).astype(np.float64) != W)
    ks = np.array([0, 5, 7], np.int64)
    H = np.zeros((3, d))
    H[np.arange(3), ks] = 1.0
    ids = np.array([3, 39, 0], np.int32)
    lp, lse = oracle.token_logprobs(H, W, ids)
    for t, k in enumerate(ks):
        ref = logsumexp(W[:, k])
        assert abs(lse[t] - ref) <= 1e-14 * max(1.0, abs(ref))
        assert abs(lp[t] - (W[ids[t], k] - ref)) <= 1e-14 * max(1.0, abs(ref))


def test_fp64_and_bf16_bit_operands_agree_on_bf16_values():
    rng = np.random.default_rng(6)
    Hb = wl.bf16_bits(rng.standard_normal((20, 64)).astype(np.float32))
    Wb = wl.bf16_bits((rng.standard_normal((300, 64)) / 8).astype(np.float32))
    ids = rng.integers(0, 300, 20).astype(np.int32)
    a = oracle.token_logprobs(Hb, Wb, ids)
    b = oracle.token_logprobs(wl.bits_to_f32(Hb).astype(np.float64), wl.bits_to_f32(Wb).astype(np.float64), ids)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
