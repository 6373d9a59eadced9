"""Data-parallel plumbing: one process per GPU, tokens sharded across ranks.

Every (token, slot) of the operator is independent of every other token, so
a batch splits across ranks by tokens with no data-path collective; weights
are replicated.  Only the benchmark's timing uses a collective (max over
ranks).
"""
from __future__ import annotations


def token_shard(n_tokens_total: int, rank: int, world: int) -> tuple[int, int]:
    """(first token, token count) of `rank`'s contiguous share of a batch.

    Shares differ by at most one token; earlier ranks take the remainder."""
    if world < 1 or not (0 <= rank < world) or n_tokens_total < 0:
        raise ValueError("bad shard request")
    base, rem = divmod(n_tokens_total, world)
    t0 = rank * base + min(rank, rem)
    return t0, base + (1 if rank < rem else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar across the default process group (identity
    when torch.distributed is not initialised)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
