"""Data-parallel REINFORCE Zero step with a deterministic gradient all-reduce.

The path shards by responses: each rank holds whole groups (so group means stay local),
every rank computes its shard with N set to the global number of responses
(rz_loss_options.n_resp_total), and dW and the loss are summed across ranks.  The sum is
made independent of timing, topology and the collective's algorithm ("vLLM
Train-Inference Consistency Release Notes", section "Achieving Bitwise Consistency",
cross-GPU consistency) by moving data with pure copies and adding in rank order on the
GPU:

    all-to-all    rank s receives slice s of every rank's tensor        (copy)
    rz_sum_shards slice s = sum over ranks r = 0..R-1, in order         (librz kernel)
    all-gather    every rank receives every summed slice                (copy)

torch.distributed (NCCL on GPUs) only moves bytes.  The CUDA sum is the default; a CPU
summation can be injected only for testing the orchestration on CPU ranks.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from . import lib, loss_options, rz_loss_fwd_bwd_ex, rz_sum_shards_f32


def deterministic_all_reduce(x: torch.Tensor, group=None, sum_shards=None) -> torch.Tensor:
    """Sum an fp32 tensor over the ranks of `group`, bit-identical on every rank."""
    if x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("deterministic_all_reduce takes a contiguous fp32 tensor")
    world = dist.get_world_size(group)
    flat = x.reshape(-1)
    count = flat.numel()
    piece = -(-count // world)
    send = torch.zeros(world * piece, dtype=x.dtype, device=x.device)
    send[:count] = flat
    recv = torch.empty(world * piece, dtype=x.dtype, device=x.device)
    dist.all_to_all_single(recv, send, group=group)  # recv[r * piece:(r+1) * piece] = my slice of rank r
    stacked = recv.view(world, piece)
    if sum_shards is None:
        if not x.is_cuda:
            raise RuntimeError("the rank-order sum runs in librz on a CUDA device")
        lib()
        mine = rz_sum_shards_f32(stacked)
    else:
        mine = sum_shards(stacked)
    out = torch.empty(world * piece, dtype=x.dtype, device=x.device)
    dist.all_gather_into_tensor(out, mine.contiguous(), group=group)
    return out[:count].view_as(x)


def global_response_count(n_resp_local: int, device, group=None) -> int:
    """The number of responses over all ranks (integer sum: exact in any order)."""
    t = torch.tensor([n_resp_local], dtype=torch.int64, device=device)
    dist.all_reduce(t, group=group)
    return int(t.item())


def shard_groups(seg_offsets, group_ids, world: int):
    """Split a batch into `world` shards of whole groups, balanced by tokens (host logic).

    Each group's responses must form one contiguous run (the layout the group-mean advantage
    is computed over).  Shard r ends at the group boundary whose token offset is closest to
    (r + 1) n_tok / world, keeping at least one group for every shard after it; needs at
    least `world` groups.  Returns one dict per rank: its token range [tok_lo, tok_hi), its
    response range [resp_lo, resp_hi), its seg_offsets rebased to 0 and its group ids
    renumbered 0 .. n_groups - 1 in order of appearance."""
    off = np.asarray(seg_offsets, dtype=np.int64)
    gid = np.asarray(group_ids, dtype=np.int64)
    R = gid.shape[0]
    if off.shape != (R + 1,) or R == 0:
        raise ValueError("seg_offsets must have n_resp + 1 entries, n_resp >= 1")
    starts = np.flatnonzero(np.r_[True, gid[1:] != gid[:-1]])  # first response of each run
    if np.unique(gid[starts]).shape[0] != starts.shape[0]:
        raise ValueError("a group's responses must be contiguous")
    n_runs = starts.shape[0]
    if n_runs < world:
        raise ValueError(f"{n_runs} groups cannot fill {world} shards")
    bounds = np.r_[starts, R]  # response index of every group boundary
    n_tok = int(off[-1])
    cut = [0]
    for r in range(1, world):
        lo, hi = cut[-1] + 1, n_runs - (world - r)  # boundary indices still allowed
        cand = np.arange(lo, hi + 1)
        target = r * n_tok / world
        cut.append(int(cand[np.argmin(np.abs(off[bounds[cand]] - target))]))
    cut.append(n_runs)
    shards = []
    for r in range(world):
        r0, r1 = int(bounds[cut[r]]), int(bounds[cut[r + 1]])
        t0, t1 = int(off[r0]), int(off[r1])
        local = gid[r0:r1]
        _, first = np.unique(local, return_index=True)
        order = np.argsort(np.argsort(first))  # rank of each distinct id by first appearance
        ids = order[np.searchsorted(np.unique(local), local)].astype(np.int32)
        shards.append(dict(tok_lo=t0, tok_hi=t1, resp_lo=r0, resp_hi=r1, seg_offsets=off[r0:r1 + 1] - t0,
                           group_ids=ids, n_groups=int(first.shape[0])))
    return shards


def dp_loss_fwd_bwd(H, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, n_groups, group=None,
                    options=None, sum_shards=None, workspace=None, n_resp_total=None):
    """One data-parallel step: this rank's shard (whole groups, e.g. from shard_groups) through
    rz_loss_fwd_bwd_ex with N = the global response count, then dW and the loss summed
    deterministically.  dH stays local (its rows are this rank's tokens).  Returns the
    rz_loss_fwd_bwd dict with the global loss and dW.  `workspace` (uint8 CUDA tensor of at
    least rz_workspace_bytes_loss for the shard) is reused when given; `n_resp_total`, when
    the caller already knows it, saves the collective that counts the responses.
    `sum_shards` is for testing the orchestration on CPU ranks only (see
    deterministic_all_reduce)."""
    n_total = (global_response_count(rewards.shape[0], rewards.device, group) if n_resp_total is None
               else int(n_resp_total))
    opts = options if options is not None else loss_options()
    opts.n_resp_total = n_total
    out = rz_loss_fwd_bwd_ex(H, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, n_groups, opts,
                             workspace=workspace)
    out["dW"] = deterministic_all_reduce(out["dW"], group, sum_shards)
    out["loss"] = deterministic_all_reduce(out["loss"], group, sum_shards)
    return out
