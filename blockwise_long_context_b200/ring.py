"""Ring Attention (pass-KV) across ranks: the scheme LV-XAttn is compared with.

Ring Attention with Blockwise Transformers page, abstract; LV-XAttn review
page, "What carries the argument" and "Core claim": every worker holds one
block of the queries and one block of the keys and values.  The key/value
blocks travel around the ring; at each of the W steps a worker computes the
blockwise attention of its queries against the block it holds while that
block moves on to the next worker.  The partial outputs are combined by the
same rescaling as the merge of the block partials.

Layouts: the sequence is cut into chunks with ``shard_bounds``.  Contiguous:
W chunks, rank r holds chunk r.  Zigzag: 2W chunks, rank r holds chunks r and
2W - 1 - r (its local tensors are the two concatenated; ``rank_bounds``
gives the rows).  At step s rank r holds the chunks of rank (r - s) mod W.
For self-attention with the causal mask (the plainest reading, as for the
single-GPU kernels: key j is visible to query row i iff j <= i), a query
chunk is computed against an earlier key chunk in full, against its own
chunk with the diagonal mask, and not against a later one (that partial is
the empty (0, -inf)).  With the contiguous layout the last rank then does
W - 1 full blocks and the diagonal while the first does only its diagonal;
the zigzag layout gives every rank the same work at every step.  Without
the mask every pair is computed (cross-attention whose query and key
sequences are both sharded).

Backward: each chunk's dK, dV accumulators (float32) travel with it; a step
adds the contribution of the local query rows, computed with their global
log-sum-exp and D = rowsum(dO o O) (the blockwise form of the exact
gradient), with ``lvx_attn_bwd_accumulate``, which adds in float32 without
rounding each part to the input dtype.  After W steps and W passes of the
accumulators each is back with the chunk's owner.  The pages leave the backward unspecified (LV-XAttn review
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

__all__ = ["shard_bounds", "rank_bounds", "chunks_of", "pair_mode", "ring_schedule",
           "RingExchange", "run_ring_forward", "run_ring_backward", "ring_attention_forward",
           "ring_attention_backward"]

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

    def start(self, tensors: Sequence[torch.Tensor], seq_len=None):
        """Sends ``tensors`` to the next rank; the ones received from the previous
        rank have the same shapes except dimension 1, which is ``seq_len`` (the
        length of the incoming block; one length, or one per tensor)."""
        if self.world == 1:
            return list(tensors), []
        lens = seq_len if isinstance(seq_len, (list, tuple)) else [seq_len] * len(tensors)
        recv = []
        for t, n in zip(tensors, lens):
            shape = list(t.shape)
            if n is not None:
                shape[1] = n
            recv.append(torch.empty(shape, dtype=t.dtype, device=t.device))
        return self.exchange(tensors, (self.rank + 1) % self.world, recv,
                             (self.rank - 1) % self.world)

    @staticmethod
    def finish(handle) -> List[torch.Tensor]:
        recv, works = handle[0], handle[1]
        for w in works:
            w.wait()
        return recv

    def pass_on(self, tensors: Sequence[torch.Tensor], seq_len=None) -> List[torch.Tensor]:
        return self.finish(self.start(tensors, seq_len))


PartialFn = Callable[[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor, bool], None]
MergeFn = Callable[[torch.Tensor, torch.Tensor], Tuple[torch.Tensor, torch.Tensor]]
GradFn = Callable[..., None]


CONTIGUOUS, ZIGZAG = "contiguous", "zigzag"


def chunks_of(rank: int, world: int, layout: str = CONTIGUOUS) -> List[int]:
    """The chunks of the sequence rank ``rank`` holds, in the order it holds them:
    contiguous, one chunk of W (chunk r); zigzag, two of 2W (chunks r and
    2W - 1 - r), which gives every rank the same causal work at every step."""
    if layout == CONTIGUOUS:
        return [rank]
    if layout == ZIGZAG:
        return [rank, 2 * world - 1 - rank]
    raise ValueError(f"unknown layout {layout!r}")


def rank_bounds(S: int, world: int, rank: int, layout: str = CONTIGUOUS) -> List[Tuple[int, int]]:
    """Rows [lo, hi) of a length-S sequence that rank ``rank`` holds, chunk by
    chunk; its local tensors are these rows concatenated in this order."""
    n = world if layout == CONTIGUOUS else 2 * world
    return [shard_bounds(S, n, c) for c in chunks_of(rank, world, layout)]


def pair_mode(cq: int, ck: int, causal: bool) -> str:
    """Query chunk ``cq`` against key chunk ``ck``: in full, with the diagonal
    mask, or skipped (every key of a later chunk is masked)."""
    if not causal or ck < cq:
        return FULL
    return DIAG if ck == cq else SKIP


class _Chunks:
    """Chunk lengths of a sequence sharded over the ranks (all ranks agree: the
    total length comes from the gathered local lengths)."""

    def __init__(self, local_len: int, exchange: "RingExchange", layout: str, device):
        world = exchange.world
        self.total = sum(exchange.lengths(local_len, device))
        self.n = world if layout == CONTIGUOUS else 2 * world
        self.world, self.layout = world, layout

    def lens(self, rank: int) -> List[int]:
        return [hi - lo for lo, hi in rank_bounds(self.total, self.world, rank, self.layout)]


def _split(t: torch.Tensor, lens: Sequence[int], dim: int = 1) -> List[torch.Tensor]:
    out, o = [], 0
    for n in lens:
        out.append(t.narrow(dim, o, n).contiguous())
        o += n
    if o != t.shape[dim]:
        raise ValueError("local rows do not match the layout's chunks (cut them with rank_bounds)")
    return out


def run_ring_forward(q, k, v, partial_fn: PartialFn, merge_fn: MergeFn, exchange: RingExchange,
                     causal: bool = False, layout: str = CONTIGUOUS):
    """q [B, S_r, H, d], k, v [B, S_kv_r, H_kv, d]: this rank's rows (its chunks,
    concatenated).  ``partial_fn(q, k_blk, v_blk, O [1,B,H,S,d], L [1,B,H,S],
    diagonal)`` writes one chunk pair's partial; ``merge_fn(O_parts, L_parts)``
    returns (out, lse) for one query chunk.  The next block's transfer is started
    before the current block's partials are computed."""
    world, rank = exchange.world, exchange.rank
    B, _, H, d = q.shape
    qc = _Chunks(q.shape[1], exchange, layout, q.device)
    kc = _Chunks(k.shape[1], exchange, layout, k.device)
    mine = chunks_of(rank, world, layout)
    nloc = len(mine)
    q_ch = _split(q, qc.lens(rank))
    k_cur, v_cur = _split(k, kc.lens(rank)), _split(v, kc.lens(rank))
    o_parts = [torch.zeros((world * nloc, B, H, t.shape[1], d), dtype=torch.float32, device=q.device)
               for t in q_ch]
    l_parts = [torch.full((world * nloc, B, H, t.shape[1]), float("-inf"), dtype=torch.float32,
                          device=q.device) for t in q_ch]
    for step in range(world):
        theirs = chunks_of((rank - step) % world, world, layout)
        handle = None
        if step + 1 < world:
            nxt = kc.lens((rank - step - 1) % world)
            handle = exchange.start(k_cur + v_cur, nxt + nxt)
        for iq, cq in enumerate(mine):
            for ik, ck in enumerate(theirs):
                mode = pair_mode(cq, ck, causal)
                if mode != SKIP:
                    slot = step * nloc + ik
                    partial_fn(q_ch[iq], k_cur[ik], v_cur[ik], o_parts[iq][slot:slot + 1],
                               l_parts[iq][slot:slot + 1], mode == DIAG)
        if handle is not None:
            recv = exchange.finish(handle)
            k_cur, v_cur = recv[:nloc], recv[nloc:]
    merged = [merge_fn(o, l) for o, l in zip(o_parts, l_parts)]
    if nloc == 1:
        return merged[0]
    return torch.cat([m[0] for m in merged], dim=1), torch.cat([m[1] for m in merged], dim=2)


def run_ring_backward(q, k, v, out, lse, do, grad_fn: GradFn, exchange: RingExchange,
                      causal: bool = False, layout: str = CONTIGUOUS):
    """Gradients of this rank's rows: (dq [B,S_r,H,d], dk, dv [B,S_kv_r,H_kv,d]) in
    float32.  ``grad_fn(q, k_blk, v_blk, out, lse, do, diagonal, dq, dk, dv)`` adds
    one chunk pair's contributions, computed with the global ``lse``, to the
    float32 accumulators dq, dk, dv."""
    world, rank = exchange.world, exchange.rank
    qc = _Chunks(q.shape[1], exchange, layout, q.device)
    kc = _Chunks(k.shape[1], exchange, layout, k.device)
    mine = chunks_of(rank, world, layout)
    nloc = len(mine)
    ql = qc.lens(rank)
    q_ch, out_ch, do_ch = _split(q, ql), _split(out, ql), _split(do, ql)
    lse_ch = _split(lse, ql, dim=2)
    k_cur, v_cur = _split(k, kc.lens(rank)), _split(v, kc.lens(rank))
    f32 = lambda t: torch.zeros(t.shape, dtype=torch.float32, device=t.device)
    dq = [f32(t) for t in q_ch]
    dk_acc, dv_acc = [f32(t) for t in k_cur], [f32(t) for t in v_cur]
    for step in range(world):
        theirs = chunks_of((rank - step) % world, world, layout)
        # the block (and accumulators) this rank holds next: after the last step,
        # the accumulators of its own chunks come home
        nxt = kc.lens((rank - step - 1) % world) if step + 1 < world else kc.lens(rank)
        handle = exchange.start(k_cur + v_cur, nxt + nxt) if step + 1 < world else None
        for iq, cq in enumerate(mine):
            for ik, ck in enumerate(theirs):
                mode = pair_mode(cq, ck, causal)
                if mode == SKIP:
                    continue
                grad_fn(q_ch[iq], k_cur[ik], v_cur[ik], out_ch[iq], lse_ch[iq], do_ch[iq],
                        mode == DIAG, dq[iq], dk_acc[ik], dv_acc[ik])
        # the accumulators travel with their block; the last pass returns them home
        recv = exchange.pass_on(dk_acc + dv_acc, nxt + nxt)
        dk_acc, dv_acc = recv[:nloc], recv[nloc:]
        if handle is not None:
            recv = exchange.finish(handle)
            k_cur, v_cur = recv[:nloc], recv[nloc:]
    cat = lambda ts: ts[0] if len(ts) == 1 else torch.cat(ts, dim=1)
    return cat(dq), cat(dk_acc), cat(dv_acc)


def kernel_partial(scale: float = 0.0, stream=None) -> PartialFn:
    """One block partial with the library's forward kernels."""
    def fn(q, k_blk, v_blk, o, l, diagonal):
        if q.shape[1] == 0 or k_blk.shape[1] == 0:
            return                      # an empty block: the partial stays (0, -inf)
        if o.shape[0] > k_blk.shape[1]:   # more slots than keys: the rest stay (0, -inf)
            o, l = o[:k_blk.shape[1]], l[:k_blk.shape[1]]
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
    """The library's merge kernel, output in ``like``'s dtype (shape from the partials)."""
    def fn(o_parts, l_parts):
        _, B, H, S_r, d = o_parts.shape
        out = torch.empty((B, S_r, H, d), dtype=like.dtype, device=like.device)
        lse = torch.empty(B, H, S_r, dtype=torch.float32, device=like.device)
        if S_r > 0:
            lvx.lvx_merge_partials(o_parts, l_parts, out, lse, stream)
        return out, lse
    return fn


def kernel_block_grad(scale: float = 0.0, stream=None) -> GradFn:
    """One block pair's gradient contributions with the library's fused backward
    (it recomputes P from the given global log-sum-exp and D from out and do),
    added in float32 to the accumulators by the kernels themselves
    (``lvx_attn_bwd_accumulate``): no part is rounded to the input dtype."""
    def fn(q, k_blk, v_blk, out, lse, do, diagonal, dq, dk, dv):
        if q.shape[1] == 0 or k_blk.shape[1] == 0:
            return
        lvx.lvx_attn_bwd_accumulate(q, k_blk, v_blk, out, lse, do, dq, dk, dv, causal=diagonal,
                                    scale=scale, stream=stream)
    return fn


def _require_cuda(t: torch.Tensor, what: str) -> None:
    if not t.is_cuda:
        raise RuntimeError(f"{what} runs in the CUDA library; its inputs must be on a GPU")


def ring_attention_forward(q, k, v, group=None, causal: bool = False, scale: float = 0.0,
                           stream=None, layout: str = CONTIGUOUS) -> Tuple[torch.Tensor, torch.Tensor]:
    """Attention of this rank's query rows over the key/value sequence sharded
    across the ranks of ``group`` (rows cut with ``rank_bounds``) ->
    out [B, S_r, H, d], lse [B, H, S_r] float32."""
    _require_cuda(q, "ring_attention_forward")
    return run_ring_forward(q, k, v, kernel_partial(scale, stream), kernel_merge(q, stream),
                            RingExchange(group), causal, layout)


def ring_attention_backward(q, k, v, out, lse, do, group=None, causal: bool = False,
                            scale: float = 0.0, layout: str = CONTIGUOUS
                            ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """dq, dk, dv of this rank's rows (input dtype), from the ring forward's
    out and lse."""
    _require_cuda(q, "ring_attention_backward")
    dq, dk, dv = run_ring_backward(q, k, v, out, lse, do, kernel_block_grad(scale),
                                   RingExchange(group), causal, layout)
    return dq.to(q.dtype), dk.to(k.dtype), dv.to(v.dtype)
