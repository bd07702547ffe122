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

Backward (the pages leave it unspecified: LV-XAttn review page, referee
report, major comment 1; this is the textbook gradient with the global
log-sum-exp, as in the single-GPU backward).  In the ring form the key/value
shard stays where it is, and so do the float32 accumulators of its dK, dV;
each query block travels again, with its dO, O and log-sum-exp and a float32
dQ accumulator.  In round s rank r adds the contributions of the block it
holds against its own shard (``lvx_attn_bwd_accumulate``: dQ into the
travelling accumulator, dK and dV into its own), then passes the accumulator
on; after the last round one more hop brings every dQ home.  In the
all-gather form every rank holds all query rows: it computes its shard's dK,
dV locally and its contribution to every row's dQ, and one all-reduce sums
the dQ contributions.

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


def run_xattn_ring(q, k, v, partial_fn, merge_fn, exchange, n_local: int = 1):
    """LV-XAttn's rotation of the query blocks (LV-XAttn review page, "What
    carries the argument"; Figure 3 / Algorithm 1).  This rank keeps k, v
    [B, S_kv_r, H_kv, d]; q [B, S_r, H, d] is its query block.  In round s it
    holds the query block of rank (r - s) mod W, starts passing it on, computes
    that block's partial against k, v with ``partial_fn`` (signature as in
    ``ring.run_ring_forward``) and sends the partial to the block's owner,
    receiving its own block's partial from rank (r + s) mod W.  ``merge_fn``
    merges the W partials of this rank's rows.  With ``n_local`` > 1 each
    round's partial is that many block partials of the key/value shard (more
    CTAs per round when the query blocks are short), W * n_local in all."""
    world, rank = exchange.world, exchange.rank
    B, S_r, H, d = q.shape
    q_len = exchange.lengths(S_r, q.device)
    nl = n_local
    o_parts = torch.zeros((world * nl, B, H, S_r, d), dtype=torch.float32, device=q.device)
    l_parts = torch.full((world * nl, B, H, S_r), float("-inf"), dtype=torch.float32, device=q.device)
    q_cur, in_flight = q, []
    for s in range(world):
        owner = (rank - s) % world
        handle = None
        if s + 1 < world:
            handle = exchange.start([q_cur], q_len[(rank - s - 1) % world])
        if s == 0:
            partial_fn(q_cur, k, v, o_parts[0:nl], l_parts[0:nl], False)
        else:
            S_o = q_cur.shape[1]
            o_p = torch.zeros((nl, B, H, S_o, d), dtype=torch.float32, device=q.device)
            l_p = torch.full((nl, B, H, S_o), float("-inf"), dtype=torch.float32, device=q.device)
            partial_fn(q_cur, k, v, o_p, l_p, False)
            in_flight.append(exchange.exchange([o_p, l_p], owner, [o_parts[s * nl:(s + 1) * nl],
                                                                   l_parts[s * nl:(s + 1) * nl]],
                                               (rank + s) % world))
        if handle is not None:
            q_cur = exchange.finish(handle)[0]
    for h in in_flight:
        exchange.finish(h)
    return merge_fn(o_parts, l_parts)


def xattn_forward_ring(q, k_shard, v_shard, group=None, scale: float = 0.0, stream=None,
                       n_local_blocks: int = 1):
    """Cross-attention with the query rows and the key/value sequence both
    sharded across the ranks of ``group`` (rank r holds rows
    ``shard_bounds(S, W, r)`` of each) -> out [B, S_r, H, d], lse [B, H, S_r]
    float32 for this rank's query rows.  Non-causal.  ``n_local_blocks``: block
    partials per round (see ``run_xattn_ring``)."""
    if not q.is_cuda:
        raise RuntimeError("xattn_forward_ring runs in the CUDA library; q must be on a GPU")
    from .ring import RingExchange, kernel_merge, kernel_partial
    return run_xattn_ring(q, k_shard, v_shard, kernel_partial(scale, stream),
                          kernel_merge(q, stream), RingExchange(group), n_local_blocks)


def _recv_like(t: torch.Tensor, n: int, seq_dim: int = 1) -> torch.Tensor:
    shape = list(t.shape)
    shape[seq_dim] = n
    return torch.empty(shape, dtype=t.dtype, device=t.device)


def run_xattn_ring_backward(q, k, v, out, lse, do, grad_fn, exchange):
    """LV-XAttn's backward in the ring form.  This rank keeps k, v
    [B, S_kv_r, H_kv, d] and the float32 accumulators of their gradients; its
    query block q [B, S_r, H, d] with out, do (same shape) and lse [B, H, S_r]
    travels as in the forward, with a float32 dq accumulator.  In round s the
    rank holds the block of rank (r - s) mod W and ``grad_fn(q, k, v, out, lse,
    do, diagonal, dq, dk, dv)`` (as in ``ring.run_ring_backward``) adds that
    block's contributions; the block's other tensors move on before the
    compute, its dq accumulator after it, and after the last round each
    accumulator is back with its owner.  Returns float32 (dq [B, S_r, H, d],
    dk, dv [B, S_kv_r, H_kv, d])."""
    world, rank = exchange.world, exchange.rank
    q_len = exchange.lengths(q.shape[1], q.device)
    f32 = lambda t: torch.zeros(t.shape, dtype=torch.float32, device=t.device)
    dk, dv = f32(k), f32(v)
    cur = [q, do, out, lse.transpose(1, 2).contiguous()]   # lse travels as [B, S, H]
    dq = f32(q)
    for s in range(world):
        handle = None
        if s + 1 < world:   # the next block: rank (r - s - 1)'s, from the previous rank
            n_in = q_len[(rank - s - 1) % world]
            handle = exchange.exchange(cur, (rank + 1) % world, [_recv_like(t, n_in) for t in cur],
                                       (rank - 1) % world)
        grad_fn(cur[0], k, v, cur[2], cur[3].transpose(1, 2).contiguous(), cur[1], False, dq, dk,
                dv)
        if world > 1:
            # the accumulator follows its block; after the last round it goes home
            n_in = q_len[(rank - s - 1) % world]
            dq = exchange.finish(exchange.exchange([dq], (rank + 1) % world,
                                                   [_recv_like(dq, n_in)], (rank - 1) % world))[0]
        if handle is not None:
            cur = exchange.finish(handle)
    return dq, dk, dv


def xattn_backward_ring(q, k_shard, v_shard, out, lse, do, group=None, scale: float = 0.0,
                        stream=None):
    """Gradients of ``xattn_forward_ring``: this rank's query rows and key/value
    shard (rows cut with ``shard_bounds``) -> dq [B, S_r, H, d], dk, dv
    [B, S_kv_r, H_kv, d] in the input dtype, from the forward's out and lse of
    this rank's rows.  Non-causal."""
    if not q.is_cuda:
        raise RuntimeError("xattn_backward_ring runs in the CUDA library; q must be on a GPU")
    from .ring import RingExchange, kernel_block_grad
    dq, dk, dv = run_xattn_ring_backward(q, k_shard, v_shard, out, lse, do,
                                         kernel_block_grad(scale, stream), RingExchange(group))
    return dq.to(q.dtype), dk.to(k_shard.dtype), dv.to(v_shard.dtype)


def run_xattn_sharded_backward(q, k, v, out, lse, do, grad_fn, group=None):
    """The backward of the all-gather form: every rank holds all query rows
    and one key/value shard.  ``grad_fn`` (as above) adds the shard's
    contributions to float32 dq, dk, dv; one all-reduce sums dq over the
    ranks.  Returns float32 (dq [B, S_Q, H, d], dk, dv of the shard)."""
    f32 = lambda t: torch.zeros(t.shape, dtype=torch.float32, device=t.device)
    dq, dk, dv = f32(q), f32(k), f32(v)
    grad_fn(q, k, v, out, lse, do, False, dq, dk, dv)
    world, _ = _world(group)
    if world > 1:
        dist.all_reduce(dq, op=dist.ReduceOp.SUM, group=group)
    return dq, dk, dv


def xattn_backward_sharded(q, k_shard, v_shard, out, lse, do, group=None, scale: float = 0.0,
                           stream=None):
    """Gradients of ``xattn_forward_sharded`` -> dq [B, S_Q, H, d] (the same on
    every rank), dk, dv of this rank's shard, in the input dtype."""
    if not q.is_cuda:
        raise RuntimeError("xattn_backward_sharded runs in the CUDA library; q must be on a GPU")
    from .ring import kernel_block_grad
    dq, dk, dv = run_xattn_sharded_backward(q, k_shard, v_shard, out, lse, do,
                                            kernel_block_grad(scale, stream), group)
    return dq.to(q.dtype), dk.to(k_shard.dtype), dv.to(v_shard.dtype)
