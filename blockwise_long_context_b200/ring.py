"""Ring Attention (pass-KV) across ranks: the scheme LV-XAttn is compared with.

Ring Attention with Blockwise Transformers page, abstract; LV-XAttn review
page, "What carries the argument" and "Core claim": every worker holds one
block of the queries and one block of the keys and values.  The key/value
blocks travel around the ring; at each of the W steps a worker computes the
blockwise attention of its queries against the block it holds while that
block moves on to the next worker.  The partial outputs are combined by the
same rescaling as the merge of the block partials.

Layout: rank r of W holds rows ``shard_bounds(S, W, r)`` of Q and of K, V.
For self-attention with the causal mask (the plainest reading, as for the
single-GPU kernels: key j is visible to query row i iff j <= i), at step s
rank r holds the block of rank src = (r - s) mod W; the pair is computed in
full if src < r, with the diagonal mask if src == r, and skipped if src > r
(its partial is the empty (0, -inf)).  Without the mask every pair is
computed (cross-attention whose query and key sequences are both sharded).

Backward: each block's dK, dV accumulators travel with it; a step adds the
contribution of the local query rows, computed with their global
log-sum-exp and D = rowsum(dO o O) (the blockwise form of the exact
gradient).  After W steps and W passes of the accumulators each is back with
the block's owner.  The pages leave the backward unspecified (LV-XAttn review
page, referee report, major comment 1); this is the textbook gradient, as in
the single-GPU backward.

Only the exchange is communication (point-to-point over ``torch.distributed``:
NCCL over NVLink between GPUs, gloo on CPU); by default every compute step
runs in the library's CUDA kernels.  The drivers take the step functions as
arguments so the exchange can be exercised on its own.
"""

from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from . import binding as lvx
from .distributed import shard_bounds

__all__ = ["shard_bounds", "ring_schedule", "RingExchange", "run_ring_forward",
           "run_ring_backward", "ring_attention_forward", "ring_attention_backward"]

FULL, DIAG, SKIP = "full", "diag", "skip"


def ring_schedule(rank: int, world: int, step: int, causal: bool) -> Tuple[int, str]:
    """(src, mode): the rank whose key/value block rank ``rank`` holds at ``step``,
    and whether that pair is computed in full, with the diagonal mask, or skipped."""
    if not (0 <= rank < world and 0 <= step < world):
        raise ValueError("need 0 <= rank, step < world")
    src = (rank - step) % world
    if not causal:
        return src, FULL
    return src, (FULL if src < rank else DIAG if src == rank else SKIP)


class RingExchange:
    """Sends tensors to the next rank and receives the incoming block's tensors
    from the previous one, as one batch of point-to-point operations."""

    def __init__(self, group=None):
        self.group = group
        if dist.is_available() and dist.is_initialized():
            self.world, self.rank = dist.get_world_size(group), dist.get_rank(group)
        else:
            self.world, self.rank = 1, 0

    def _global(self, r: int) -> int:
        return dist.get_global_rank(self.group, r) if self.group is not None else r

    def lengths(self, n: int, device) -> List[int]:
        """Every rank's ``n`` (its shard length), in rank order."""
        if self.world == 1:
            return [n]
        mine = torch.tensor([n], dtype=torch.int64, device=device)
        all_n = [torch.empty_like(mine) for _ in range(self.world)]
        dist.all_gather(all_n, mine, group=self.group)
        return [int(t.item()) for t in all_n]

    def exchange(self, sends: Sequence[torch.Tensor], dst: int,
                 recvs: Sequence[torch.Tensor], src: int):
        """Starts sending ``sends`` to rank ``dst`` and receiving into ``recvs``
        (contiguous, preallocated) from rank ``src``, as one batch; returns a
        handle for ``finish``.  Every rank must post its matching half."""
        # empty tensors are not sent: both sides know every shard's length, so
        # they leave out the same transfers
        sends = [t.contiguous() for t in sends if t.numel() > 0]
        ops = [dist.P2POp(dist.isend, t, self._global(dst), self.group) for t in sends]
        ops += [dist.P2POp(dist.irecv, r, self._global(src), self.group) for r in recvs
                if r.numel() > 0]
        works = dist.batch_isend_irecv(ops) if ops else []
        return list(recvs), works, sends   # the send buffers stay referenced until finish

    def start(self, tensors: Sequence[torch.Tensor], seq_len: Optional[int] = None):
        """Sends ``tensors`` to the next rank; the ones received from the previous
        rank have the same shapes except dimension 1, which is ``seq_len`` (the
        length of the incoming block)."""
        if self.world == 1:
            return list(tensors), []
        recv = []
        for t in tensors:
            shape = list(t.shape)
            if seq_len is not None:
                shape[1] = seq_len
            recv.append(torch.empty(shape, dtype=t.dtype, device=t.device))
        return self.exchange(tensors, (self.rank + 1) % self.world, recv,
                             (self.rank - 1) % self.world)

    @staticmethod
    def finish(handle) -> List[torch.Tensor]:
        recv, works = handle[0], handle[1]
        for w in works:
            w.wait()
        return recv

    def pass_on(self, tensors: Sequence[torch.Tensor], seq_len: Optional[int] = None
                ) -> List[torch.Tensor]:
        return self.finish(self.start(tensors, seq_len))


PartialFn = Callable[[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor, bool], None]
MergeFn = Callable[[torch.Tensor, torch.Tensor], Tuple[torch.Tensor, torch.Tensor]]
GradFn = Callable[..., Tuple[torch.Tensor, torch.Tensor, torch.Tensor]]


def run_ring_forward(q, k, v, partial_fn: PartialFn, merge_fn: MergeFn, exchange: RingExchange,
                     causal: bool = False):
    """q [B, S_r, H, d], k, v [B, S_kv_r, H_kv, d]: this rank's blocks.
    ``partial_fn(q, k_blk, v_blk, O [1,B,H,S_r,d], L [1,B,H,S_r], diagonal)`` writes
    one block partial; ``merge_fn(O_parts, L_parts)`` returns (out, lse).  The next
    block's transfer is started before the current block's partial is computed."""
    world, rank = exchange.world, exchange.rank
    B, S_r, H, d = q.shape
    kv_len = exchange.lengths(k.shape[1], k.device)   # shards may differ in length
    o_parts = torch.zeros((world, B, H, S_r, d), dtype=torch.float32, device=q.device)
    l_parts = torch.full((world, B, H, S_r), float("-inf"), dtype=torch.float32, device=q.device)
    k_cur, v_cur = k, v
    for step in range(world):
        _, mode = ring_schedule(rank, world, step, causal)
        handle = None
        if step + 1 < world:
            nxt = ring_schedule(rank, world, step + 1, causal)[0]
            handle = exchange.start([k_cur, v_cur], kv_len[nxt])
        if mode != SKIP:
            partial_fn(q, k_cur, v_cur, o_parts[step:step + 1], l_parts[step:step + 1], mode == DIAG)
        if handle is not None:
            k_cur, v_cur = exchange.finish(handle)
    return merge_fn(o_parts, l_parts)


def run_ring_backward(q, k, v, out, lse, do, grad_fn: GradFn, exchange: RingExchange,
                      causal: bool = False):
    """Gradients of this rank's blocks: (dq [B,S_r,H,d], dk, dv [B,S_kv_r,H_kv,d]) in
    float32.  ``grad_fn(q, k_blk, v_blk, out, lse, do, diagonal)`` returns one block
    pair's contributions (dq_part, dk_part, dv_part) with the global ``lse``."""
    world, rank = exchange.world, exchange.rank
    kv_len = exchange.lengths(k.shape[1], k.device)
    dq = torch.zeros(q.shape, dtype=torch.float32, device=q.device)
    dk_acc = torch.zeros(k.shape, dtype=torch.float32, device=k.device)
    dv_acc = torch.zeros(v.shape, dtype=torch.float32, device=v.device)
    k_cur, v_cur = k, v
    for step in range(world):
        _, mode = ring_schedule(rank, world, step, causal)
        # the block (and accumulators) this rank holds next: after the last step,
        # the accumulators of its own block come home
        nxt = ring_schedule(rank, world, step + 1, causal)[0] if step + 1 < world else rank
        handle = exchange.start([k_cur, v_cur], kv_len[nxt]) if step + 1 < world else None
        if mode != SKIP:
            dq_p, dk_p, dv_p = grad_fn(q, k_cur, v_cur, out, lse, do, mode == DIAG)
            dq += dq_p
            dk_acc += dk_p
            dv_acc += dv_p
        # the accumulators travel with their block; the last pass returns them home
        dk_acc, dv_acc = exchange.pass_on([dk_acc, dv_acc], kv_len[nxt])
        if handle is not None:
            k_cur, v_cur = exchange.finish(handle)
    return dq, dk_acc, dv_acc


def kernel_partial(scale: float = 0.0, stream=None) -> PartialFn:
    """One block partial with the library's forward kernels."""
    def fn(q, k_blk, v_blk, o, l, diagonal):
        if q.shape[1] == 0 or k_blk.shape[1] == 0:
            return                      # an empty block: the partial stays (0, -inf)
        # one step's slice of the partials is 16-byte aligned only if its size is;
        # the library wants aligned pointers, so short shards go through a copy
        oo = o if o.data_ptr() % 16 == 0 else torch.empty_like(o)
        ll = l if l.data_ptr() % 16 == 0 else torch.empty_like(l)
        lvx.lvx_attn_fwd_partials(q, k_blk, v_blk, oo, ll, scale, stream, causal=diagonal)
        if oo is not o:
            o.copy_(oo)
        if ll is not l:
            l.copy_(ll)
    return fn


def kernel_merge(like: torch.Tensor, stream=None) -> MergeFn:
    """The library's merge kernel, output in ``like``'s dtype and shape."""
    def fn(o_parts, l_parts):
        B, S_r, H, _ = like.shape
        out = torch.empty_like(like)
        lse = torch.empty(B, H, S_r, dtype=torch.float32, device=like.device)
        if S_r > 0:
            lvx.lvx_merge_partials(o_parts, l_parts, out, lse, stream)
        return out, lse
    return fn


def kernel_block_grad(scale: float = 0.0) -> GradFn:
    """One block pair's gradient contributions with the library's fused backward
    (it recomputes P from the given global log-sum-exp and D from out and do)."""
    def fn(q, k_blk, v_blk, out, lse, do, diagonal):
        if q.shape[1] == 0 or k_blk.shape[1] == 0:
            z = lambda t: torch.zeros(t.shape, dtype=torch.float32, device=t.device)
            return z(q), z(k_blk), z(v_blk)
        dq, dk, dv = lvx.attention_backward(q, k_blk, v_blk, out, lse, do, causal=diagonal,
                                            scale=scale)
        return dq.float(), dk.float(), dv.float()
    return fn


def _require_cuda(t: torch.Tensor, what: str) -> None:
    if not t.is_cuda:
        raise RuntimeError(f"{what} runs in the CUDA library; its inputs must be on a GPU")


def ring_attention_forward(q, k, v, group=None, causal: bool = False, scale: float = 0.0,
                           stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Attention of this rank's query rows over the key/value sequence sharded
    across the ranks of ``group`` -> out [B, S_r, H, d], lse [B, H, S_r] float32."""
    _require_cuda(q, "ring_attention_forward")
    return run_ring_forward(q, k, v, kernel_partial(scale, stream), kernel_merge(q, stream),
                            RingExchange(group), causal)


def ring_attention_backward(q, k, v, out, lse, do, group=None, causal: bool = False,
                            scale: float = 0.0) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """dq, dk, dv of this rank's blocks (input dtype), from the ring forward's
    out and lse."""
    _require_cuda(q, "ring_attention_backward")
    dq, dk, dv = run_ring_backward(q, k, v, out, lse, do, kernel_block_grad(scale),
                                   RingExchange(group), causal)
    return dq.to(q.dtype), dk.to(k.dtype), dv.to(v.dtype)
