"""Expert parallelism: the experts are cut into contiguous ranges, one per
rank; every rank computes the slots routed to its own experts, for every
token, and one all-to-all returns each slot's output row to the rank that
owns the token.

The PR #283 article ("ik_llama.cpp 的 CUDA 更优 MoE 实现", section 3.3) notes
that MoE had no row split across GPUs, against vLLM's tensor parallelism.
This module is the other split the expert-sorted tables make natural: the
row-id pass groups the slots by expert, so a contiguous expert range owns a
contiguous range of sorted positions [expert_bounds[e0], expert_bounds[e1]).

Step, per rank (tokens sharded as by dist.token_shard, weights of the rank's
experts only):
  1. all-gather the token shards' activations and ids (every rank sees all
     tokens);
  2. take the slots t*k+s whose expert lies in this rank's range, in
     ascending slot order, and compute their rows with `compute` - one
     expert per row (k = 1), the expert renumbered into the local range;
  3. all-to-all: the rows go to the owners of their tokens.  Ascending slot
     order is already ordered by owner (token shards are contiguous and
     ascending in rank), and a receiver lists its own slots per source rank
     in the same order, so no indices travel with the rows;
  4. the owner writes each received row to dst[t - t0][s].
Each slot's row is computed by exactly one rank from the same weights and
activation row as without the split, and the exchange moves bits without
arithmetic.  The combine of a token's k rows then runs on its owner, in
ascending s, as it would unsharded.

Only torch.distributed collectives and index bookkeeping run here; the rows
themselves come from `compute` (the library's entry points on a GPU).
"""
from __future__ import annotations

from typing import Callable

import torch
import torch.distributed as dist

from .dist import token_shard


def expert_range(n_experts: int, rank: int, world: int) -> tuple[int, int]:
    """[e0, e1) of `rank`'s contiguous share of the experts (sizes differ by at
    most one, earlier ranks take the remainder)."""
    e0, n = token_shard(n_experts, rank, world)
    return e0, e0 + n


def owned_slot_range(expert_bounds, e0: int, e1: int) -> tuple[int, int]:
    """Sorted positions [p0, p1) of the slots of experts [e0, e1), read from the
    row-id pass's expert_bounds (n_experts + 1 exclusive prefix offsets)."""
    return int(expert_bounds[e0]), int(expert_bounds[e1])


def local_slots(ids_all: torch.Tensor, e0: int, e1: int) -> torch.Tensor:
    """Flat slot indices t*k+s (ascending) whose expert is in [e0, e1)."""
    flat = ids_all.reshape(-1)
    return torch.nonzero((flat >= e0) & (flat < e1), as_tuple=False).reshape(-1)


def _all_gather_rows(x: torch.Tensor, counts: list[int], group=None) -> torch.Tensor:
    """Concatenate every rank's rows (row counts `counts`, in rank order)."""
    world = len(counts)
    m = max(counts)
    pad = torch.zeros((m,) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    pad[: x.shape[0]] = x
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:c] for p, c in zip(parts, counts)], dim=0)


def ep_forward(x_local: torch.Tensor, ids_local: torch.Tensor, n_tokens_total: int, n_experts: int,
               n_out: int, compute: Callable[[torch.Tensor, torch.Tensor], torch.Tensor], group=None) -> torch.Tensor:
    """The expert-parallel step for this rank.

    x_local [T_r][n_in] and ids_local [T_r][k] (global expert ids) are this
    rank's token shard (token_shard(n_tokens_total, rank, world)).
    compute(x_rows [n][n_in], ids_rows [n][1] int32, local expert numbers) ->
    rows [n][n_out] float32 runs the operator for one expert per row with this
    rank's weights (experts expert_range(...) renumbered from 0).
    Returns dst [T_r][k][n_out] float32 for this rank's tokens."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    t0, T_r = token_shard(n_tokens_total, rank, world)
    if x_local.shape[0] != T_r or ids_local.shape[0] != T_r:
        raise ValueError("x_local / ids_local must hold this rank's token shard")
    k = ids_local.shape[1]
    counts = [token_shard(n_tokens_total, r, world)[1] for r in range(world)]
    x_all = _all_gather_rows(x_local, counts, group)
    ids_all = _all_gather_rows(ids_local, counts, group)
    e0, e1 = expert_range(n_experts, rank, world)

    # 2. rows of this rank's experts, ascending slot order
    mine = local_slots(ids_all, e0, e1)
    tok = torch.div(mine, k, rounding_mode="floor")
    if mine.numel():
        rows = compute(x_all.index_select(0, tok).contiguous(),
                       (ids_all.reshape(-1).index_select(0, mine) - e0).to(torch.int32).reshape(-1, 1).contiguous())
        rows = rows.reshape(mine.numel(), n_out).to(torch.float32)
    else:
        rows = torch.empty((0, n_out), dtype=torch.float32, device=x_local.device)

    # 3. send to token owners: split sizes by owner (contiguous token ranges)
    starts = [token_shard(n_tokens_total, r, world)[0] for r in range(world)] + [n_tokens_total]
    send = [int(((tok >= starts[r]) & (tok < starts[r + 1])).sum()) for r in range(world)]
    my_ids = ids_local.reshape(-1)
    recv_sel = []
    for q in range(world):
        a, b = expert_range(n_experts, q, world)
        recv_sel.append(torch.nonzero((my_ids >= a) & (my_ids < b), as_tuple=False).reshape(-1))
    recv = [int(s.numel()) for s in recv_sel]
    out_rows = torch.empty((sum(recv), n_out), dtype=torch.float32, device=x_local.device)
    dist.all_to_all_single(out_rows, rows.contiguous(), recv, send, group=group)

    # 4. place the rows at their slots
    dst = torch.empty((T_r * k, n_out), dtype=torch.float32, device=x_local.device)
    dst.index_copy_(0, torch.cat(recv_sel), out_rows)
    return dst.reshape(T_r, k, n_out)
