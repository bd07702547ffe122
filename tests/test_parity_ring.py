"""Ring Attention on the GPU: the library's kernels at every ring step.

The ring's ranks are emulated one after another on one GPU (no kernel waits
for another rank).  For each rank and step, ``chunks_of`` names the chunks it
holds and the key/value chunks it has at that step, ``pair_mode`` says
whether a chunk pair is computed in full, with the diagonal mask or skipped,
and the step functions the distributed driver uses (``kernel_partial``,
``kernel_merge``, ``kernel_block_grad``) compute it.  Both layouts are run:
contiguous, and zigzag (rank r holds chunks r and 2W - 1 - r of 2W).  The
assembled outputs and gradients are compared with the fp64 oracle's full
attention; uneven shards (1000 keys over 3 ranks) and empty shards and
chunks are covered.  A one-rank NCCL group runs the distributed driver
itself; the exchange over several ranks is covered on CPU by
``tests/test_ring_gloo.py``.
"""

import os
import socket

import numpy as np
import pytest
import torch

import oracle
from blockwise_long_context_b200 import inputs
from blockwise_long_context_b200.ring import (DIAG, SKIP, chunks_of, kernel_block_grad,
                                              kernel_merge, kernel_partial, pair_mode, shard_bounds)
from tests._parity import compare

pytestmark = pytest.mark.gpu


def _problem(B, H, H_kv, d, S_Q, S_KV):
    w = inputs.WORKLOADS["C2"].scaled(B=B, H=H, H_kv=H_kv, d=d, S_Q=S_Q, S_KV=S_KV, n_blocks=1,
                                      causal=False, backward=True, d_embed=0)
    return inputs.make(w, tensors=("q", "k", "v", "do"))


def _emulate(host, W, causal, layout="contiguous"):
    """Every rank's ring steps, one after another, chunk pair by chunk pair; the
    results are put back in global row order."""
    dev = {n: t.cuda() for n, t in host.items()}
    B, S_Q, H, d = dev["q"].shape
    S_KV = dev["k"].shape[1]
    nC = W if layout == "contiguous" else 2 * W
    qb = [shard_bounds(S_Q, nC, c) for c in range(nC)]
    kb = [shard_bounds(S_KV, nC, c) for c in range(nC)]
    cut = lambda t, lo, hi: t[:, lo:hi].contiguous()
    q = [cut(dev["q"], *b) for b in qb]
    do = [cut(dev["do"], *b) for b in qb]
    k = [cut(dev["k"], *b) for b in kb]
    v = [cut(dev["v"], *b) for b in kb]
    partial, grad = kernel_partial(), kernel_block_grad()
    outs, lses = [None] * nC, [None] * nC
    for r in range(W):
        mine = chunks_of(r, W, layout)
        for cq in mine:
            n = W * len(mine)
            o_parts = torch.zeros((n, B, H, q[cq].shape[1], d), dtype=torch.float32, device="cuda")
            l_parts = torch.full((n, B, H, q[cq].shape[1]), float("-inf"), device="cuda")
            for st in range(W):
                for ik, ck in enumerate(chunks_of((r - st) % W, W, layout)):
                    mode = pair_mode(cq, ck, causal)
                    if mode != SKIP:
                        slot = st * len(mine) + ik
                        partial(q[cq], k[ck], v[ck], o_parts[slot:slot + 1], l_parts[slot:slot + 1],
                                mode == DIAG)
            outs[cq], lses[cq] = kernel_merge(q[cq])(o_parts, l_parts)
    f32 = lambda t: torch.zeros(t.shape, dtype=torch.float32, device="cuda")
    dq, dk, dv = [f32(t) for t in q], [f32(t) for t in k], [f32(t) for t in v]
    for r in range(W):
        for st in range(W):
            for cq in chunks_of(r, W, layout):
                for ck in chunks_of((r - st) % W, W, layout):
                    mode = pair_mode(cq, ck, causal)
                    if mode == SKIP:
                        continue
                    grad(q[cq], k[ck], v[ck], outs[cq], lses[cq], do[cq], mode == DIAG,
                         dq[cq], dk[ck], dv[ck])
    torch.cuda.synchronize()
    from blockwise_long_context_b200 import binding as lvx
    lvx.lvx_last_device_error()
    cat = lambda ts, dim=1: torch.cat(ts, dim=dim)
    return (cat(outs), cat(lses, 2), cat(dq).to(torch.bfloat16), cat(dk).to(torch.bfloat16),
            cat(dv).to(torch.bfloat16))


CASES = [
    # name,               B, H, H_kv, d,  S_Q,  S_KV, W, causal, layout
    ("causal_w3_uneven",   1, 4, 2,  128, 1000, 1000, 3, True,  "contiguous"),
    ("causal_w4_d64",      1, 2, 1,   64,  512,  512, 4, True,  "contiguous"),
    ("cross_w3",           1, 4, 2,  128,  300, 1000, 3, False, "contiguous"),
    ("cross_w2_d64",       2, 2, 2,   64,  130,  777, 2, False, "contiguous"),
    ("causal_empty_shard", 1, 2, 2,  128,    9,    9, 4, True,  "contiguous"),   # 3, 3, 3, 0
    ("zigzag_w4",          1, 4, 2,  128, 1000, 1000, 4, True,  "zigzag"),
    ("zigzag_w3_d64",      2, 2, 1,   64,  700,  700, 3, True,  "zigzag"),
    ("zigzag_empty_chunks", 1, 2, 2, 128,    9,    9, 4, True,  "zigzag"),   # 2,2,2,2,1,0,0,0
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_emulated_ring_matches_attention(case):
    name, B, H, H_kv, d, S_Q, S_KV, W, causal, layout = case
    host = _problem(B, H, H_kv, d, S_Q, S_KV)
    out, lse, dq, dk, dv = _emulate(host, W, causal, layout)
    q, k, v, do = (host[t].double().numpy() for t in ("q", "k", "v", "do"))
    o_ref, l_ref = oracle.attention_fwd(q, k, v, causal=causal)
    dq_r, dk_r, dv_r = oracle.attention_bwd(q, k, v, do, causal=causal)
    compare(out, o_ref, "bf16", f"{name}: O")
    compare(lse, l_ref, "bf16", f"{name}: LSE", rel_rms=1e-4)
    compare(dq, dq_r, "bf16", f"{name}: dQ")
    compare(dk, dk_r, "bf16", f"{name}: dK")
    compare(dv, dv_r, "bf16", f"{name}: dV")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("causal,layout", [(True, "contiguous"), (False, "contiguous"),
                                           (True, "zigzag")])
def test_ring_driver_in_a_one_rank_nccl_group(causal, layout):
    import datetime
    import torch.distributed as dist
    from blockwise_long_context_b200.ring import ring_attention_backward, ring_attention_forward
    host = _problem(1, 4, 2, 128, 384, 384 if causal else 640)
    dev = {n: t.cuda() for n, t in host.items()}
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0),
                            timeout=datetime.timedelta(seconds=60))
    try:
        out, lse = ring_attention_forward(dev["q"], dev["k"], dev["v"], causal=causal,
                                          layout=layout)
        dq, dk, dv = ring_attention_backward(dev["q"], dev["k"], dev["v"], out, lse, dev["do"],
                                             causal=causal, layout=layout)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    q, k, v, do = (host[t].double().numpy() for t in ("q", "k", "v", "do"))
    o_ref, l_ref = oracle.attention_fwd(q, k, v, causal=causal)
    dq_r, dk_r, dv_r = oracle.attention_bwd(q, k, v, do, causal=causal)
    compare(out, o_ref, "bf16", "ring nccl: O")
    compare(lse, l_ref, "bf16", "ring nccl: LSE", rel_rms=1e-4)
    compare(dq, dq_r, "bf16", "ring nccl: dQ")
    compare(dk, dk_r, "bf16", "ring nccl: dK")
    compare(dv, dv_r, "bf16", "ring nccl: dV")
