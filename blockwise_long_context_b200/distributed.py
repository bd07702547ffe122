"""LV-XAttn's exchange across GPUs: stationary key/value shards, gathered partials.

LV-XAttn review page, "The reading" and Figure 3 / Algorithm 1: every worker
keeps one block K_i, V_i of the long visual key/value sequence, and the
queries' partial outputs and log-sum-exp statistics (O_i, L_i) of all workers
are combined by the rescaling of the merge ("What carries the argument").

Here every rank computes its shard's block partials for all query rows with
``lvx_attn_fwd_partials`` (the library's kernels), the ranks exchange them in
one all-gather over ``torch.distributed`` (NCCL over NVLink between GPUs), and
every rank merges all partials with ``lvx_merge_partials``.  This is the
all-gather form of the exchange, and its result is replicated on every rank.

``xattn_forward_ring`` is the ring form: the query rows are sharded too, each
rank's query block travels around the ring (its transfer overlapping the
partial computed on the block held), and each partial goes straight back to
the query block's owner, which merges the W partials of its rows once.  The
pages rescale the travelling (O, L) at every hop; merging all partials at the
owner moves the same bytes (one partial per round per rank) and gives the
same result up to the order of the rescaling.  Each rank ends with the output
of its own query rows.

Only the transfers are communication; every compute step runs in the
library's CUDA kernels, and there is no CPU path.
"""

from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import binding as lvx


def shard_bounds(S_KV: int, world: int, rank: int) -> Tuple[int, int]:
    """Keys [lo, hi) of rank ``rank``: the same partition as the key/value
    blocks, shard i = [i * ceil(S_KV / world), min((i + 1) * ceil(S_KV / world), S_KV))."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    per = -(-S_KV // world)
    lo = min(rank * per, S_KV)
    return lo, min(lo + per, S_KV)


def _world(group) -> Tuple[int, int]:
    if not (dist.is_available() and dist.is_initialized()):
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def gather_partials(o_loc: torch.Tensor, l_loc: torch.Tensor,
                    group=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """All-gather of every rank's partials along the block axis, rank-major.

    o_loc [n, B, H, S_Q, d], l_loc [n, B, H, S_Q] (float32, same n on every
    rank) -> [world * n, ...] in rank order, so the merge sees the same order
    on every rank and every rank computes the same bits."""
    world, _ = _world(group)
    if world == 1:
        return o_loc, l_loc
    o_all = o_loc.new_empty((world * o_loc.shape[0],) + tuple(o_loc.shape[1:]))
    l_all = l_loc.new_empty((world * l_loc.shape[0],) + tuple(l_loc.shape[1:]))
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(o_all, o_loc.contiguous(), group=group)
        dist.all_gather_into_tensor(l_all, l_loc.contiguous(), group=group)
    else:
        dist.all_gather(list(o_all.chunk(world)), o_loc.contiguous(), group=group)
        dist.all_gather(list(l_all.chunk(world)), l_loc.contiguous(), group=group)
    return o_all, l_all


def xattn_forward_sharded(q: torch.Tensor, k_shard: torch.Tensor, v_shard: torch.Tensor,
                          group=None, n_local_blocks: int = 1, scale: float = 0.0,
                          stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Cross-attention of all query rows over a key/value sequence sharded across
    the ranks of ``group`` (rank r holds keys ``shard_bounds(S_KV, world, r)``).

    q [B, S_Q, H, d] (replicated), k_shard / v_shard [B, S_KV_r, H_kv, d] (this
    rank's shard, cut into ``n_local_blocks`` blocks) -> out [B, S_Q, H, d],
    lse [B, H, S_Q] float32, the same on every rank.  Non-causal."""
    if not q.is_cuda:
        raise RuntimeError("xattn_forward_sharded runs in the CUDA library; q must be on a GPU")
    B, S_Q, H, d = q.shape
    o_loc = torch.empty(n_local_blocks, B, H, S_Q, d, dtype=torch.float32, device=q.device)
    l_loc = torch.empty(n_local_blocks, B, H, S_Q, dtype=torch.float32, device=q.device)
    lvx.lvx_attn_fwd_partials(q, k_shard, v_shard, o_loc, l_loc, scale, stream)
    o_all, l_all = gather_partials(o_loc, l_loc, group)
    out = torch.empty_like(q)
    lse = torch.empty(B, H, S_Q, dtype=torch.float32, device=q.device)
    lvx.lvx_merge_partials(o_all, l_all, out, lse, stream)
    return out, lse


def run_xattn_ring(q, k, v, partial_fn, merge_fn, exchange):
    """LV-XAttn's rotation of the query blocks (LV-XAttn review page, "What
    carries the argument"; Figure 3 / Algorithm 1).  This rank keeps k, v
    [B, S_kv_r, H_kv, d]; q [B, S_r, H, d] is its query block.  In round s it
    holds the query block of rank (r - s) mod W, starts passing it on, computes
    that block's partial against k, v with ``partial_fn`` (signature as in
    ``ring.run_ring_forward``) and sends the partial to the block's owner,
    receiving its own block's partial from rank (r + s) mod W.  ``merge_fn``
    merges the W partials of this rank's rows."""
    world, rank = exchange.world, exchange.rank
    B, S_r, H, d = q.shape
    q_len = exchange.lengths(S_r, q.device)
    o_parts = torch.zeros((world, B, H, S_r, d), dtype=torch.float32, device=q.device)
    l_parts = torch.full((world, B, H, S_r), float("-inf"), dtype=torch.float32, device=q.device)
    q_cur, in_flight = q, []
    for s in range(world):
        owner = (rank - s) % world
        handle = None
        if s + 1 < world:
            handle = exchange.start([q_cur], q_len[(rank - s - 1) % world])
        if s == 0:
            partial_fn(q_cur, k, v, o_parts[0:1], l_parts[0:1], False)
        else:
            S_o = q_cur.shape[1]
            o_p = torch.zeros((1, B, H, S_o, d), dtype=torch.float32, device=q.device)
            l_p = torch.full((1, B, H, S_o), float("-inf"), dtype=torch.float32, device=q.device)
            partial_fn(q_cur, k, v, o_p, l_p, False)
            in_flight.append(exchange.exchange([o_p, l_p], owner, [o_parts[s], l_parts[s]],
                                               (rank + s) % world))
        if handle is not None:
            q_cur = exchange.finish(handle)[0]
    for h in in_flight:
        exchange.finish(h)
    return merge_fn(o_parts, l_parts)


def xattn_forward_ring(q, k_shard, v_shard, group=None, scale: float = 0.0, stream=None):
    """Cross-attention with the query rows and the key/value sequence both
    sharded across the ranks of ``group`` (rank r holds rows
    ``shard_bounds(S, W, r)`` of each) -> out [B, S_r, H, d], lse [B, H, S_r]
    float32 for this rank's query rows.  Non-causal."""
    if not q.is_cuda:
        raise RuntimeError("xattn_forward_ring runs in the CUDA library; q must be on a GPU")
    from .ring import RingExchange, kernel_merge, kernel_partial
    return run_xattn_ring(q, k_shard, v_shard, kernel_partial(scale, stream),
                          kernel_merge(q, stream), RingExchange(group))
