"""MXFP4 operands for an LM head: CPU reference of the quantiser and the decoder.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``.  The pages name MXFP4 weights on
the rollout side ("vLLM says aligned kernels make asynchronous RL stable at lag 64",
section "Zero mismatch expands to newer models") but fix no scheme; the reading here is
the OCP Microscaling (MX) v1.0 format, the one Blackwell's block-scaled tensor-core
instructions consume:

  - a row of d values is cut into blocks of 32 consecutive elements along d;
  - each block shares one scale 2^X stored as E8M0 (the biased exponent X + 127, one byte);
    X = floor(log2(max |x| over the block)) - 2, where 2 is the exponent of E2M1's largest
    value (6 = 1.5 * 2^2), clamped to [-127, 127]; an all-zero block takes X = -127;
  - each element is E2M1 (sign bit 3, exponent bits 2..1 with bias 1, mantissa bit 0:
    magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), the nearest value to x / 2^X with ties to the
    even code, saturating at +-6 (x / 2^X lies in [4, 8), so only the top of a block can
    exceed 6).

Everything is computed in fp64: a bf16 value divided by a power of two is exact there, so
the only rounding is the one to the E2M1 grid.  One 4-bit code is kept per byte here (the
packed layout is the kernel's business).
"""
from __future__ import annotations

import numpy as np

BLOCK = 32
E2M1_MAX = 6.0
E2M1_EMAX = 2          # exponent of the largest E2M1 value
# magnitudes of the eight non-negative codes 0..7, in code order
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _bf16_to_f64(bits):
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def block_exponents(X):
    """Shared exponent X of every 32-element block of the rows of X (fp64, d % 32 == 0):
    floor(log2 amax) - 2, clamped to [-127, 127]; -127 for an all-zero block."""
    rows, d = X.shape
    if d % BLOCK:
        raise ValueError("d must be a multiple of 32")
    amax = np.abs(X).reshape(rows, d // BLOCK, BLOCK).max(axis=2)
    _, e = np.frexp(amax)            # amax = f * 2^e with f in [0.5, 1): floor(log2 amax) = e - 1
    Xe = (e.astype(np.int64) - 1) - E2M1_EMAX
    Xe = np.where(amax > 0, Xe, -127)
    return np.clip(Xe, -127, 127)


def round_to_e2m1(y):
    """E2M1 codes (uint8, sign in bit 3) of the fp64 values y: nearest magnitude, ties to the
    even code, saturating at 6.  A negative zero keeps its sign bit."""
    a = np.abs(y)[..., None]
    dist = np.abs(a - E2M1_MAGNITUDES)
    best = dist.min(axis=-1, keepdims=True)
    tie = dist == best
    # among the nearest codes take the even one (at most two codes tie, and they are adjacent)
    even = tie & (np.arange(8) % 2 == 0)
    mag = np.where(even.any(axis=-1), even.argmax(axis=-1), tie.argmax(axis=-1)).astype(np.uint8)
    return mag | (np.signbit(y).astype(np.uint8) << 3)


def quantize_rows_mxfp4(X_bits):
    """bf16 rows (uint16 bit patterns, [rows, d], d % 32 == 0) -> (E2M1 codes uint8 [rows, d],
    E8M0 scale bytes uint8 [rows, d / 32] = X + 127)."""
    X = _bf16_to_f64(X_bits)
    rows, d = X.shape
    Xe = block_exponents(X)
    scale = np.exp2(np.repeat(Xe, BLOCK, axis=1).astype(np.float64))
    codes = round_to_e2m1(X / scale)
    return codes, (Xe + 127).astype(np.uint8)


def decode_mxfp4(codes, scale_bytes):
    """fp64 values of E2M1 codes [rows, d] with E8M0 block scales [rows, d / 32]."""
    codes = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[codes & 7]
    sign = np.where(codes & 8, -1.0, 1.0)
    Xe = np.asarray(scale_bytes, dtype=np.int64) - 127
    return sign * mag * np.exp2(np.repeat(Xe, BLOCK, axis=1).astype(np.float64))
