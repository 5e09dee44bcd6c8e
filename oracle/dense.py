"""Dense (matrix-form) fp64 oracle for mid-size problems: token logprobs, dH and rows of dW.

TEST INFRASTRUCTURE ONLY: the test suite is the only caller.  The product path (the CUDA
library and its binding) never imports this module, and it imports nothing from the product.

The definitions are those of ``oracle.c`` ("vLLM says aligned kernels make asynchronous RL
stable at lag 64" (ainewsbites.com), section "REINFORCE Zero removes the mismatch first"),
written in matrix form so that a library fp64 matrix product (numpy / BLAS) serves as the
contraction step:

    Z      = H W^T                               (z[t,v] = sum_k H[t,k] W[v,k])
    lse[t] = m_t + log sum_v exp(z[t,v] - m_t),  m_t = max_v z[t,v]
    lp[t]  = z[t, y_t] - lse[t]
    P      = exp(Z - lse)                         (softmax of each row)
    dZ     = kappa (onehot(y) - P)
    dH     = dZ W,      dW[v,:] = sum_t dZ[t,v] H[t,:]

The row-by-row C oracle takes minutes at the real head shapes (d up to 7168, V up to
151936) for a couple of thousand tokens; this form takes seconds.  Token rows are
independent in every quantity except dW, so rows are processed in groups of ``row_block``
tokens to bound memory, and dW is formed once, at the end, from the dZ columns of the
requested vocabulary rows over all tokens (no reduction is split).  The loss stage (w,
kappa, loss) is the C oracle's own ``loss_from_lp``.  Every input is bf16 bit patterns
(uint16), widened exactly to fp64.

Pinned in tests/test_oracle_dense.py against the C oracle (independently written, itself
pinned by closed forms and invariants) and against closed forms of its own.
"""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact fp64 values of bf16 bit patterns (uint16)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _rows(n: int, row_block: int):
    for r0 in range(0, n, row_block):
        yield r0, min(n, r0 + row_block)


def _logits(H64: np.ndarray, W64: np.ndarray, r0: int, r1: int) -> np.ndarray:
    """z[t, v] = sum_k H[t, k] W[v, k] for the rows r0 .. r1 - 1 (fp64 matrix product)."""
    return H64[r0:r1] @ W64.T


def token_logprobs(H_bits, W_bits, ids, row_block: int = 512):
    """(lp, lse) of every row, fp64: the log-softmax of the logits gathered at the token."""
    H64, W64 = bf16_bits_to_f64(H_bits), bf16_bits_to_f64(W_bits)
    ids = np.asarray(ids, dtype=np.int64)
    n, V = H64.shape[0], W64.shape[0]
    if ids.shape != (n,) or np.any(ids < 0) or np.any(ids >= V):
        raise ValueError("token ids must be in [0, V), one per row")
    lp = np.empty(n)
    lse = np.empty(n)
    for r0, r1 in _rows(n, row_block):
        Z = _logits(H64, W64, r0, r1)
        m = Z.max(axis=1)
        l = m + np.log(np.exp(Z - m[:, None]).sum(axis=1))
        lse[r0:r1] = l
        lp[r0:r1] = Z[np.arange(r1 - r0), ids[r0:r1]] - l
    return lp, lse


def gradients(H_bits, W_bits, ids, lse, kappa, dw_vocab_rows=None, row_block: int = 512):
    """(dH [n, d], dW rows [len(dw_vocab_rows), d]) in fp64, given every row's lse and kappa.

    dZ[t, v] = kappa_t ([v == y_t] - exp(z[t, v] - lse_t)); dH = dZ W; dW[v] = sum_t dZ[t, v] H[t].
    dw_vocab_rows None: every vocabulary row.
    """
    H64, W64 = bf16_bits_to_f64(H_bits), bf16_bits_to_f64(W_bits)
    ids = np.asarray(ids, dtype=np.int64)
    n, V = H64.shape[0], W64.shape[0]
    lse = np.asarray(lse, dtype=np.float64)
    kappa = np.asarray(kappa, dtype=np.float64)
    sel = np.arange(V) if dw_vocab_rows is None else np.asarray(dw_vocab_rows, dtype=np.int64)
    if np.any(sel < 0) or np.any(sel >= V):
        raise ValueError("vocabulary rows must be in [0, V)")
    dH = np.empty_like(H64)
    dZ_sel = np.empty((n, sel.shape[0]))
    for r0, r1 in _rows(n, row_block):
        Z = _logits(H64, W64, r0, r1)
        P = np.exp(Z - lse[r0:r1, None])
        onehot = np.zeros_like(P)
        onehot[np.arange(r1 - r0), ids[r0:r1]] = 1.0
        dZ = kappa[r0:r1, None] * (onehot - P)
        dH[r0:r1] = dZ @ W64
        dZ_sel[r0:r1] = dZ[:, sel]
    dW_rows = dZ_sel.T @ H64
    return dH, dW_rows
