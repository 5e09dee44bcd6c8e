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


def dp_loss_fwd_bwd(H, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, n_groups, group=None,
                    options=None):
    """One data-parallel step: this rank's shard (whole groups) through rz_loss_fwd_bwd_ex with
    N = the global response count, then dW and the loss summed deterministically.  dH stays
    local (its rows are this rank's tokens).  Returns the rz_loss_fwd_bwd dict with the
    global loss and dW."""
    n_total = global_response_count(rewards.shape[0], rewards.device, group)
    opts = options if options is not None else loss_options()
    opts.n_resp_total = n_total
    out = rz_loss_fwd_bwd_ex(H, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, n_groups, opts)
    out["dW"] = deterministic_all_reduce(out["dW"], group)
    out["loss"] = deterministic_all_reduce(out["loss"], group)
    return out
