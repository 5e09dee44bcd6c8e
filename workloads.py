"""Seeded synthetic inputs for the REINFORCE Zero logprob / loss / gradient path.

This module only draws random inputs; it holds none of the path's arithmetic (no
log-softmax, no ratio, no advantage, no gradient).  It is shared by the tests, the
benchmark and the smoke check, and both the oracle and the CUDA library receive what it
produces as plain arrays.

Workload shapes (the pages train on math-reasoning, agentic tool-use, OSWorld and
SWE-bench-Pro data with Qwen3-4B, a 1.5B model and MoE models; none of that data or
those weights exist here, so seeded synthetic inputs of the same shapes stand in):

  tiny        d=256,  V=4096,   2 groups x 4 responses, lengths U{16..64}
  qwen3_4b    d=2560, V=151936, 64 groups x 8,  lengths log-uniform 128..2048
  invariance  d=1536, V=151936, 4096 fixed rows (batch-invariance stress)
  lag64       d=2560, V=151936, 32 groups x 8,  lengths log-uniform 1024..16384
  moe_head    d=7168, V=129280, 128 groups x 16, lengths U{256..4096}

Values: H ~ N(0,1) and W ~ N(0, 1/d) drawn in fp32 and rounded to bf16 (round to
nearest even).  Responses are contiguous token segments; group g holds responses
g*gs .. g*gs+gs-1.  Rewards are Bernoulli(p) in {0,1} or U[0,1].

Sampled token ids are uniform for ``tiny`` and ``invariance``; for the other shapes the
pages' rollout samples tokens from the policy at temperature 1, which ``rollout_sample_ids``
stands in for with a Gumbel-max draw over bf16 logits computed by torch (the rollout
engine, not the path under test).  ``rollout_logprobs_with_lag`` turns the learner's
logprobs into recorded rollout logprobs by adding the seeded weight-lag noise.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

CONFIGS = {
    "tiny": dict(d=256, V=4096, n_groups=2, group_size=4, lengths=("uniform", 16, 64),
                 rewards=("bernoulli", 0.3), ids="uniform", noise=("normal", 0.05), seed=101),
    "qwen3_4b": dict(d=2560, V=151936, n_groups=64, group_size=8, lengths=("loguniform", 128, 2048),
                     rewards=("bernoulli", 0.29), ids="sampled", noise=("normal", 0.02), seed=102),
    "invariance": dict(d=1536, V=151936, n_rows=4096, ids="uniform", seed=103),
    "lag64": dict(d=2560, V=151936, n_groups=32, group_size=8, lengths=("loguniform", 1024, 16384),
                  rewards=("uniform",), ids="sampled", noise=("student_t3", 0.1), seed=104),
    "moe_head": dict(d=7168, V=129280, n_groups=128, group_size=16, lengths=("uniform", 256, 4096),
                     rewards=("bernoulli", 0.5), ids="sampled", noise=("normal", 0.05), seed=105),
}


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 values -> bf16 bit patterns (uint16), round to nearest even."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bits_to_f32(h: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> their exact fp32 values."""
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def draw_lengths(rng: np.random.Generator, R: int, spec) -> np.ndarray:
    kind, a, b = spec
    if kind == "uniform":
        return rng.integers(a, b + 1, size=R).astype(np.int64)
    if kind == "loguniform":
        L = np.floor(np.exp(rng.uniform(math.log(a), math.log(b), size=R)))
        return np.clip(L, a, b).astype(np.int64)
    raise ValueError(kind)


def draw_rewards(rng: np.random.Generator, R: int, spec) -> np.ndarray:
    if spec[0] == "bernoulli":
        return (rng.uniform(size=R) < spec[1]).astype(np.float32)
    if spec[0] == "uniform":
        return rng.uniform(size=R).astype(np.float32)
    raise ValueError(spec)


@dataclasses.dataclass
class Segments:
    """Responses as contiguous token segments plus their groups and rewards."""
    seg_offsets: np.ndarray  # int64 [R+1]
    group_ids: np.ndarray  # int32 [R]
    rewards: np.ndarray  # float32 [R]
    n_groups: int

    @property
    def n_tok(self) -> int:
        return int(self.seg_offsets[-1])

    @property
    def n_resp(self) -> int:
        return int(self.group_ids.shape[0])


def draw_segments(name: str, seed: Optional[int] = None, n_groups: Optional[int] = None,
                  group_size: Optional[int] = None, lengths=None) -> Segments:
    cfg = CONFIGS[name]
    rng = np.random.Generator(np.random.PCG64(cfg["seed"] if seed is None else seed))
    G = cfg["n_groups"] if n_groups is None else n_groups
    gs = cfg["group_size"] if group_size is None else group_size
    R = G * gs
    L = draw_lengths(rng, R, cfg["lengths"] if lengths is None else lengths)
    off = np.zeros(R + 1, np.int64)
    off[1:] = np.cumsum(L)
    gid = (np.arange(R) // gs).astype(np.int32)
    r = draw_rewards(rng, R, cfg["rewards"])
    return Segments(off, gid, r, G)


def draw_matrices(n: int, d: int, V: int, seed: int, device: str = "cpu"):
    """H [n,d] ~ N(0,1), W [V,d] ~ N(0,1/d), both bf16.

    device='cpu': numpy PCG64, returned as uint16 bit arrays.
    device='cuda...': torch Philox on that device, returned as torch bf16 tensors.
    """
    if device == "cpu":
        rng = np.random.Generator(np.random.PCG64(seed))
        H = bf16_bits(rng.standard_normal((n, d), dtype=np.float32))
        W = bf16_bits(rng.standard_normal((V, d), dtype=np.float32) * np.float32(1.0 / math.sqrt(d)))
        return H, W
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    H = torch.empty((n, d), dtype=torch.bfloat16, device=device)
    W = torch.empty((V, d), dtype=torch.bfloat16, device=device)
    rows = max(1, (1 << 26) // d)  # draw in fp32 slabs of <= 256 MB
    for r0 in range(0, n, rows):
        r1 = min(n, r0 + rows)
        H[r0:r1] = torch.randn((r1 - r0, d), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    for r0 in range(0, V, rows):
        r1 = min(V, r0 + rows)
        W[r0:r1] = (torch.randn((r1 - r0, d), generator=g, device=device, dtype=torch.float32)
                    * (1.0 / math.sqrt(d))).to(torch.bfloat16)
    return H, W


def draw_uniform_ids(n: int, V: int, seed: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed + 7919))
    return rng.integers(0, V, size=n).astype(np.int32)


def rollout_sample_ids(H: torch.Tensor, W: torch.Tensor, seed: int, chunk: int = 2048) -> torch.Tensor:
    """Stand-in for the rollout engine's sampler: tokens drawn at temperature 1.

    Gumbel-max over bf16 logits from torch's matmul (fp32 accumulate); ties go to the
    lowest index (torch.argmax).  Harness-only: the path under test receives the ids as
    input.  Works on any torch device; on CPU only for small shapes.
    """
    g = torch.Generator(device=H.device)
    g.manual_seed(seed + 104729)
    out = torch.empty(H.shape[0], dtype=torch.int32, device=H.device)
    for r0 in range(0, H.shape[0], chunk):
        r1 = min(H.shape[0], r0 + chunk)
        z = torch.matmul(H[r0:r1], W.t()).float()
        u = torch.rand(z.shape, generator=g, device=H.device, dtype=torch.float32)
        u.clamp_(min=1e-30)
        z.sub_(torch.log(-torch.log(u)))  # + Gumbel(0,1)
        out[r0:r1] = torch.argmax(z, dim=1).to(torch.int32)
        del z, u
    return out


def rollout_logprobs_with_lag(lp_learner: np.ndarray, noise, seed: int) -> np.ndarray:
    """Recorded rollout logprobs = learner logprobs + seeded weight-lag noise (fp32).

    noise = ("normal", sigma) or ("student_t3", scale) with t = Z / sqrt(chi2_3 / 3).
    """
    rng = np.random.Generator(np.random.PCG64(seed + 15485863))
    n = lp_learner.shape[0]
    if noise[0] == "normal":
        eps = rng.standard_normal(n) * noise[1]
    elif noise[0] == "student_t3":
        z = rng.standard_normal(n)
        chi2 = rng.chisquare(3, size=n)
        eps = noise[1] * z / np.sqrt(chi2 / 3.0)
    else:
        raise ValueError(noise)
    return (np.asarray(lp_learner, dtype=np.float64) + eps).astype(np.float32)


@dataclasses.dataclass
class Problem:
    """One call's inputs.  H/W are uint16 bf16 bits (CPU) or torch bf16 tensors (device)."""
    H: object
    W: object
    ids: object
    seg: Optional[Segments]
    d: int
    V: int
    noise: Optional[tuple] = None
    seed: int = 0

    @property
    def n_tok(self) -> int:
        return int(self.H.shape[0])


def tiny(seed: Optional[int] = None) -> Problem:
    """The CPU-seconds case: 2 groups x 4 responses, d=256, V=4096, uniform ids."""
    cfg = CONFIGS["tiny"]
    s = cfg["seed"] if seed is None else seed
    seg = draw_segments("tiny", seed=s)
    H, W = draw_matrices(seg.n_tok, cfg["d"], cfg["V"], s)
    ids = draw_uniform_ids(seg.n_tok, cfg["V"], s)
    return Problem(H, W, ids, seg, cfg["d"], cfg["V"], cfg["noise"], s)


def custom(n_groups: int, group_size: int, lengths, d: int, V: int, seed: int,
           rewards=("bernoulli", 0.3), noise=("normal", 0.05)) -> Problem:
    """A small problem of any shape (parity tests at several tiles and ragged tails)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    R = n_groups * group_size
    L = draw_lengths(rng, R, lengths)
    off = np.zeros(R + 1, np.int64)
    off[1:] = np.cumsum(L)
    gid = (np.arange(R) // group_size).astype(np.int32)
    r = draw_rewards(rng, R, rewards)
    seg = Segments(off, gid, r, n_groups)
    H, W = draw_matrices(seg.n_tok, d, V, seed)
    ids = draw_uniform_ids(seg.n_tok, V, seed)
    return Problem(H, W, ids, seg, d, V, noise, seed)


def full_config(name: str, device: str, n_tok_cap: Optional[int] = None) -> Problem:
    """A full-size workload generated on ``device`` (H, W on the device as torch bf16).

    ``n_tok_cap`` keeps only the leading responses whose tokens fit in the cap.
    """
    cfg = CONFIGS[name]
    seed = cfg["seed"]
    seg = draw_segments(name)
    if n_tok_cap is not None and seg.n_tok > n_tok_cap:
        R = int(np.searchsorted(seg.seg_offsets, n_tok_cap, side="right")) - 1
        gs = cfg["group_size"]
        R = max(gs, (R // gs) * gs)  # whole groups only
        seg = Segments(seg.seg_offsets[:R + 1].copy(), seg.group_ids[:R].copy(), seg.rewards[:R].copy(),
                       R // gs)
    H, W = draw_matrices(seg.n_tok, cfg["d"], cfg["V"], seed, device=device)
    if cfg["ids"] == "sampled":
        ids = rollout_sample_ids(H, W, seed)
    else:
        ids = torch.from_numpy(draw_uniform_ids(seg.n_tok, cfg["V"], seed)).to(device)
    return Problem(H, W, ids, seg, cfg["d"], cfg["V"], cfg.get("noise"), seed)
