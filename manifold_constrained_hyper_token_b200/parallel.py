"""Data parallelism over tokens for the mHC layer.

Tokens are independent and the layer's parameters (phi, b, alpha) are shared,
so a batch shards over ranks by tokens with no exchange in the forward pass;
the backward's only exchange is a sum over ranks of the parameter gradients
(grad_phi [nC, n^2+2n], grad_b [n^2+2n], grad_alpha [1] or [3] with per-group
alpha), kept in one flat
buffer so that it is a single all-reduce.  These helpers are the host side of
that scheme; the per-rank compute is the library's kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def token_shard(T: int, rank: int, world: int) -> tuple[int, int]:
    """[start, end) of rank's contiguous share of T tokens (sizes differ by at most 1)."""
    base, extra = divmod(int(T), int(world))
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def param_grad_buffer(n: int, C: int, device, dtype=torch.float32, alpha_groups: int = 1):
    """One flat buffer and its (grad_phi, grad_b, grad_alpha) views.  grad_alpha has
    one entry for a shared alpha and three (pre, post, res) when alpha_groups == 3."""
    K, M = n * C, n * n + 2 * n
    na = 3 if alpha_groups == 3 else 1
    flat = torch.empty(K * M + M + na, dtype=dtype, device=device)
    return flat, flat[:K * M].view(K, M), flat[K * M:K * M + M], flat[K * M + M:]


def allreduce_param_grads(flat: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the flat parameter-gradient buffer over all ranks, in place."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    return flat


def max_over_ranks(value: float, device, group=None) -> float:
    """The maximum of a per-rank float (e.g. a device-measured time) over ranks."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
