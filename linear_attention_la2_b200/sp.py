"""Sequence parallelism across ranks: each rank holds one contiguous part of
every (b, h) sequence, in rank order (rank r: rows [r N, (r + 1) N) of the
whole). The parts exchange one fp32 d x dv state per (b, h) and part - the
only cross-rank step - and each rank then runs its part from the sum of the
states before it (youleyou.com article, section "小结": sequence-parallel
linear attention; section "Lightning Attention-2简介", point 2: the state is a
running sum, so a part needs only the summed states of the earlier parts).

Forward: S_r = sum over the part of k^T v (la2_kv_state), all-gather of S
over the group, then la2_forward_sp with the states of ranks < r.
Backward: also T_r = sum over the part of q^T dO; dQ needs the states of the
earlier parts, dK and dV the sum of T over the later parts.

The exchange uses torch.distributed (NCCL between GPUs); the gathered states
land in this rank's memory before any kernel reads them.
"""

from __future__ import annotations

from . import la2


def exchange_states(local, group=None):
    """All-gather one [B, H, d, dv] float32 state per rank into a new
    [world, B, H, d, dv] tensor in rank order."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    flat = torch.empty(world * local.numel(), dtype=local.dtype, device=local.device)
    dist.all_gather_into_tensor(flat, local.contiguous().view(-1), group=group)
    return flat.view((world,) + tuple(local.shape))


def prefix_suffix(gathered, rank):
    """The states before rank `rank` and after it (contiguous slices)."""
    return gathered[:rank], gathered[rank + 1:]


def forward(q, k, v, group=None, block: int = 64, stream=None):
    """This rank's part of the causal output; q, k, v are its part [B,H,N,.]."""
    import torch.distributed as dist

    rank = dist.get_rank(group)
    gathered = exchange_states(la2.kv_state(k, v, stream=stream), group)
    before, _ = prefix_suffix(gathered, rank)
    return la2.forward_sp(q, k, v, before, block=block, stream=stream)


def backward(q, k, v, do, group=None, block: int = 64, stream=None):
    """This rank's part of (dQ, dK, dV) of the whole sequence's <dO, O>."""
    import torch.distributed as dist

    rank = dist.get_rank(group)
    kv = exchange_states(la2.kv_state(k, v, stream=stream), group)
    qdo = exchange_states(la2.kv_state(q, do, stream=stream), group)
    before, _ = prefix_suffix(kv, rank)
    _, after = prefix_suffix(qdo, rank)
    return la2.backward_sp(q, k, v, do, before, after, block=block, stream=stream)
