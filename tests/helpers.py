"""Shared helpers for the GPU parity tests: move a workloads.Problem to the device,
call the C ABI through the binding, and compare with the oracle under the stated
tolerances (|dlp| <= 2e-3 absolute, loss relative 1e-4 with the cancellation guard,
dH/dW relative Frobenius <= 5e-3)."""
from __future__ import annotations

import numpy as np
import torch

import workloads as wl

LP_ATOL = 2e-3
LOSS_RTOL = 1e-4
GRAD_RFRO = 5e-3


def bits_to_torch_bf16(bits: np.ndarray, device) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def torch_bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def to_device(p: wl.Problem, device="cuda"):
    out = dict(
        H=bits_to_torch_bf16(p.H, device), W=bits_to_torch_bf16(p.W, device),
        ids=torch.from_numpy(np.asarray(p.ids, np.int32)).to(device),
    )
    if p.seg is not None:
        out.update(
            rewards=torch.from_numpy(p.seg.rewards.astype(np.float32)).to(device),
            seg_offsets=torch.from_numpy(p.seg.seg_offsets.astype(np.int64)).to(device),
            group_ids=torch.from_numpy(p.seg.group_ids.astype(np.int32)).to(device),
        )
    return out


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a - b))


def loss_close(gpu_loss: float, ref_loss: float, A: np.ndarray, w_mean: np.ndarray) -> bool:
    """|dloss| <= 1e-4 * max(|loss|, (1/N) sum_i |A_i| mean_t w_t)  (cancellation guard)."""
    scale = float(np.mean(np.abs(A) * w_mean))
    return abs(gpu_loss - ref_loss) <= LOSS_RTOL * max(abs(ref_loss), scale)


def response_means(values: np.ndarray, off: np.ndarray) -> np.ndarray:
    L = np.diff(off)
    resp = np.repeat(np.arange(len(L)), L)
    return np.bincount(resp, weights=values, minlength=len(L)) / L
