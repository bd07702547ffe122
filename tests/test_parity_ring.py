"""Ring Attention on the GPU: the library's kernels at every ring step.

The ring's ranks are emulated one after another on one GPU (no kernel waits
for another rank): for each rank and step, ``ring_schedule`` names the
key/value block held and whether the pair is computed in full, with the
diagonal mask or skipped, and the same step functions the distributed driver
uses (``kernel_partial``, ``kernel_merge``, ``kernel_block_grad``) compute
it.  The assembled outputs and gradients are compared with the fp64 oracle's
full attention.  Uneven shards (1000 keys over 3 ranks) and an empty trailing
shard are covered.  A one-rank NCCL group runs the distributed driver itself;
the exchange over several ranks is covered on CPU by
``tests/test_ring_gloo.py``.
"""

import os
import socket

import numpy as np
import pytest
import torch

import oracle
from blockwise_long_context_b200 import inputs
from blockwise_long_context_b200.ring import (DIAG, SKIP, kernel_block_grad, kernel_merge,
                                              kernel_partial, ring_schedule, shard_bounds)
from tests._parity import compare

pytestmark = pytest.mark.gpu


def _problem(B, H, H_kv, d, S_Q, S_KV):
    w = inputs.WORKLOADS["C2"].scaled(B=B, H=H, H_kv=H_kv, d=d, S_Q=S_Q, S_KV=S_KV, n_blocks=1,
                                      causal=False, backward=True, d_embed=0)
    return inputs.make(w, tensors=("q", "k", "v", "do"))


def _emulate(host, W, causal):
    dev = {n: t.cuda() for n, t in host.items()}
    S_Q, S_KV = dev["q"].shape[1], dev["k"].shape[1]
    qb = [shard_bounds(S_Q, W, r) for r in range(W)]
    kb = [shard_bounds(S_KV, W, r) for r in range(W)]
    cut = lambda t, lo, hi: t[:, lo:hi].contiguous()
    q = [cut(dev["q"], *qb[r]) for r in range(W)]
    do = [cut(dev["do"], *qb[r]) for r in range(W)]
    k = [cut(dev["k"], *kb[r]) for r in range(W)]
    v = [cut(dev["v"], *kb[r]) for r in range(W)]
    partial, grad = kernel_partial(), kernel_block_grad()
    outs, lses = [], []
    for r in range(W):
        B, S_r, H, d = q[r].shape
        o_parts = torch.zeros((W, B, H, S_r, d), dtype=torch.float32, device="cuda")
        l_parts = torch.full((W, B, H, S_r), float("-inf"), dtype=torch.float32, device="cuda")
        for s in range(W):
            src, mode = ring_schedule(r, W, s, causal)
            if mode != SKIP:
                partial(q[r], k[src], v[src], o_parts[s:s + 1], l_parts[s:s + 1], mode == DIAG)
        out_r, lse_r = kernel_merge(q[r])(o_parts, l_parts)
        outs.append(out_r); lses.append(lse_r)
    dq = [torch.zeros(t.shape, dtype=torch.float32, device="cuda") for t in q]
    dk = [torch.zeros(t.shape, dtype=torch.float32, device="cuda") for t in k]
    dv = [torch.zeros(t.shape, dtype=torch.float32, device="cuda") for t in v]
    for r in range(W):
        for s in range(W):
            src, mode = ring_schedule(r, W, s, causal)
            if mode == SKIP:
                continue
            gq, gk, gv = grad(q[r], k[src], v[src], outs[r], lses[r], do[r], mode == DIAG)
            dq[r] += gq; dk[src] += gk; dv[src] += gv
    torch.cuda.synchronize()
    from blockwise_long_context_b200 import binding as lvx
    lvx.lvx_last_device_error()
    cat = lambda ts, dim=1: torch.cat(ts, dim=dim)
    return (cat(outs), cat(lses, 2), cat(dq).to(torch.bfloat16), cat(dk).to(torch.bfloat16),
            cat(dv).to(torch.bfloat16))


CASES = [
    # name,               B, H, H_kv, d,  S_Q,  S_KV, W, causal
    ("causal_w3_uneven",   1, 4, 2,  128, 1000, 1000, 3, True),
    ("causal_w4_d64",      1, 2, 1,   64,  512,  512, 4, True),
    ("cross_w3",           1, 4, 2,  128,  300, 1000, 3, False),
    ("cross_w2_d64",       2, 2, 2,   64,  130,  777, 2, False),
    ("causal_empty_shard", 1, 2, 2,  128,    9,    9, 4, True),   # shards 3, 3, 3, 0
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_emulated_ring_matches_attention(case):
    name, B, H, H_kv, d, S_Q, S_KV, W, causal = case
    host = _problem(B, H, H_kv, d, S_Q, S_KV)
    out, lse, dq, dk, dv = _emulate(host, W, causal)
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


@pytest.mark.parametrize("causal", [True, False])
def test_ring_driver_in_a_one_rank_nccl_group(causal):
    import datetime
    import torch.distributed as dist
    from blockwise_long_context_b200.ring import ring_attention_backward, ring_attention_forward
    host = _problem(1, 4, 2, 128, 384, 384 if causal else 640)
    dev = {n: t.cuda() for n, t in host.items()}
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0),
                            timeout=datetime.timedelta(seconds=60))
    try:
        out, lse = ring_attention_forward(dev["q"], dev["k"], dev["v"], causal=causal)
        dq, dk, dv = ring_attention_backward(dev["q"], dev["k"], dev["v"], out, lse, dev["do"],
                                             causal=causal)
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
