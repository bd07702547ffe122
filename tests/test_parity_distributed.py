"""GPU parity of the per-shard partials and of LV-XAttn's forward and backward across ranks.

``lvx_attn_fwd_partials`` computes one key/value shard's block partials
(O_i, L_i) without merging them; ``distributed.xattn_forward_sharded`` runs
it on every rank, all-gathers the partials and merges them with
``lvx_merge_partials`` (LV-XAttn review page, "The reading" and Figure 3 /
Algorithm 1).  Runs here get one GPU, so the several ranks are emulated in
one process -- each shard's partials computed separately and concatenated in
rank order, which is what the all-gather produces -- and the real
torch.distributed path runs with a one-rank NCCL group.  Every result is
checked against the fp64 oracle's unsplit attention, and the backward (query
blocks with their dQ accumulators travelling, dK/dV staying with the
stationary shard; or, in the all-gather form, dQ contributions summed over
the ranks) against the oracle's gradient.
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from blockwise_long_context_b200 import binding as lvx
from blockwise_long_context_b200 import inputs
from blockwise_long_context_b200.distributed import shard_bounds, xattn_forward_sharded
from tests._parity import compare

pytestmark = pytest.mark.gpu


def _problem(B, H, H_kv, d, S_Q, S_KV, dtype="bf16", seed_cfg=1):
    base = inputs.WORKLOADS["C0" if dtype == "f32" else "C1"]
    w = base.scaled(B=B, H=H, H_kv=H_kv, d=d, S_Q=S_Q, S_KV=S_KV, n_blocks=1, causal=False,
                    dtype=dtype)
    host = inputs.make(w)
    return w, host


def _oracle(host):
    q, k, v = (host[t].double().numpy() for t in ("q", "k", "v"))
    return oracle.attention_fwd(q, k, v)


@pytest.mark.parametrize("dtype,d,n", [("bf16", 128, 1), ("bf16", 128, 3), ("bf16", 64, 2),
                                       ("f32", 64, 2)])
def test_shard_partials_match_oracle_partials(dtype, d, n):
    w, host = _problem(2, 4, 2, d, 200, 700, dtype)
    dev = {t: x.cuda() for t, x in host.items()}
    O = torch.empty(n, w.B, w.H, w.S_Q, w.d, dtype=torch.float32, device="cuda")
    L = torch.empty(n, w.B, w.H, w.S_Q, dtype=torch.float32, device="cuda")
    lvx.lvx_attn_fwd_partials(dev["q"], dev["k"], dev["v"], O, L)
    lvx.lvx_last_device_error()
    torch.cuda.synchronize()
    q, k, v = (host[t].double().numpy() for t in ("q", "k", "v"))
    O_r, L_r = oracle.block_partials(q, k, v, n)
    compare(O, np.transpose(O_r, (0, 1, 3, 2, 4)), w.dtype, f"partials {dtype} d={d} n={n}: O")
    compare(L, L_r, w.dtype, f"partials {dtype} d={d} n={n}: L",
            rel_rms=1e-4 if dtype == "bf16" else 1e-6)


@pytest.mark.parametrize("world,n_local,S_KV", [(2, 1, 1024), (3, 2, 1000), (8, 1, 4099)])
def test_sharded_forward_emulated_ranks(world, n_local, S_KV):
    """Each emulated rank computes its shard's partials; concatenated in rank
    order (the all-gather's layout) and merged they give attention over the
    whole key/value sequence."""
    w, host = _problem(1, 8, 2, 128, 300, S_KV)
    dev = {t: x.cuda() for t, x in host.items()}
    Os, Ls = [], []
    for r in range(world):
        lo, hi = shard_bounds(S_KV, world, r)
        O = torch.empty(n_local, w.B, w.H, w.S_Q, w.d, dtype=torch.float32, device="cuda")
        L = torch.empty(n_local, w.B, w.H, w.S_Q, dtype=torch.float32, device="cuda")
        lvx.lvx_attn_fwd_partials(dev["q"], dev["k"][:, lo:hi].contiguous(),
                                  dev["v"][:, lo:hi].contiguous(), O, L)
        Os.append(O); Ls.append(L)
    out = torch.empty_like(dev["q"])
    lse = torch.empty(w.B, w.H, w.S_Q, dtype=torch.float32, device="cuda")
    lvx.lvx_merge_partials(torch.cat(Os), torch.cat(Ls), out, lse)
    lvx.lvx_last_device_error()
    torch.cuda.synchronize()
    o_ref, l_ref = _oracle(host)
    compare(out, o_ref, "bf16", f"sharded x{world}: O")
    compare(lse, l_ref, "bf16", f"sharded x{world}: LSE", rel_rms=1e-4)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_sharded_forward_through_torch_distributed():
    """The real path: NCCL process group (one rank on this GPU), partials,
    all-gather, merge."""
    import torch.distributed as dist
    w, host = _problem(2, 4, 4, 128, 256, 2048)
    dev = {t: x.cuda() for t, x in host.items()}
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        lo, hi = shard_bounds(w.S_KV, 1, 0)
        out, lse = xattn_forward_sharded(dev["q"], dev["k"][:, lo:hi], dev["v"][:, lo:hi],
                                         n_local_blocks=4)
        lvx.lvx_last_device_error()
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    o_ref, l_ref = _oracle(host)
    compare(out, o_ref, "bf16", "torch.distributed: O")
    compare(lse, l_ref, "bf16", "torch.distributed: LSE", rel_rms=1e-4)


@pytest.mark.parametrize("world,S_Q,S_KV", [(2, 300, 1024), (3, 300, 1000), (4, 9, 999)])
def test_ring_form_emulated_ranks(world, S_Q, S_KV):
    """LV-XAttn's ring form with the query rows sharded too: in round s rank r
    computes the partial of rank (r - s)'s query block against its own shard,
    with the same step functions the distributed driver uses; each owner merges
    its W partials.  (4, 9, ...) leaves one rank without query rows."""
    from blockwise_long_context_b200.ring import kernel_merge, kernel_partial
    w, host = _problem(1, 8, 2, 128, S_Q, S_KV)
    dev = {t: x.cuda() for t, x in host.items()}
    qb = [shard_bounds(S_Q, world, r) for r in range(world)]
    kb = [shard_bounds(S_KV, world, r) for r in range(world)]
    q = [dev["q"][:, lo:hi].contiguous() for lo, hi in qb]
    k = [dev["k"][:, lo:hi].contiguous() for lo, hi in kb]
    v = [dev["v"][:, lo:hi].contiguous() for lo, hi in kb]
    partial = kernel_partial()
    parts = []
    for o in range(world):
        S_o = q[o].shape[1]
        parts.append((torch.zeros(world, w.B, w.H, S_o, w.d, dtype=torch.float32, device="cuda"),
                      torch.full((world, w.B, w.H, S_o), float("-inf"), device="cuda")))
    for r in range(world):
        for s in range(world):
            o = (r - s) % world
            partial(q[o], k[r], v[r], parts[o][0][s:s + 1], parts[o][1][s:s + 1], False)
    outs, lses = zip(*(kernel_merge(q[o])(*parts[o]) for o in range(world)))
    lvx.lvx_last_device_error()
    torch.cuda.synchronize()
    o_ref, l_ref = _oracle(host)
    compare(torch.cat(outs, 1), o_ref, "bf16", f"ring form x{world}: O")
    compare(torch.cat(lses, 2), l_ref, "bf16", f"ring form x{world}: LSE", rel_rms=1e-4)


def test_ring_form_through_torch_distributed():
    """xattn_forward_ring through a one-rank NCCL group."""
    import torch.distributed as dist
    from blockwise_long_context_b200.distributed import xattn_forward_ring
    w, host = _problem(2, 4, 2, 128, 256, 1500)
    dev = {t: x.cuda() for t, x in host.items()}
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        out, lse = xattn_forward_ring(dev["q"], dev["k"], dev["v"])
        lvx.lvx_last_device_error()
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    o_ref, l_ref = _oracle(host)
    compare(out, o_ref, "bf16", "ring form, torch.distributed: O")
    compare(lse, l_ref, "bf16", "ring form, torch.distributed: LSE", rel_rms=1e-4)


def _oracle_bwd(host):
    q, k, v, do = (host[t].double().numpy() for t in ("q", "k", "v", "do"))
    return oracle.attention_bwd(q, k, v, do)


def _bwd_problem(S_Q, S_KV, H=8, H_kv=2):
    base = inputs.WORKLOADS["C2"]
    w = base.scaled(B=1, H=H, H_kv=H_kv, d=128, S_Q=S_Q, S_KV=S_KV, n_blocks=1, causal=False,
                    d_embed=0)
    return w, inputs.make(w, tensors=("q", "k", "v", "do"))


@pytest.mark.parametrize("world,S_Q,S_KV", [(2, 300, 1024), (3, 256, 1000), (4, 12, 999)])
def test_xattn_backward_emulated_ranks(world, S_Q, S_KV):
    """The ring form's backward with the step the distributed driver uses: for
    every (query block o, key/value shard r) pair, in ring order, the block's
    contributions are added to o's travelling float32 dQ accumulator and to
    r's stationary dK, dV accumulators.  (4, 12, ...) gives shards of 3 rows."""
    from blockwise_long_context_b200.ring import kernel_block_grad
    w, host = _bwd_problem(S_Q, S_KV)
    dev = {t: x.cuda() for t, x in host.items()}
    out, lse = lvx.attention_forward(dev["q"], dev["k"], dev["v"], 1)
    qb = [shard_bounds(S_Q, world, r) for r in range(world)]
    kb = [shard_bounds(S_KV, world, r) for r in range(world)]
    rows = lambda t, b: t[:, b[0]:b[1]].contiguous()
    q, o_, do = ([rows(t, b) for b in qb] for t in (dev["q"], out, dev["do"]))
    ls = [lse[:, :, lo:hi].contiguous() for lo, hi in qb]
    k, v = ([rows(t, b) for b in kb] for t in (dev["k"], dev["v"]))
    f32 = lambda t: torch.zeros(t.shape, dtype=torch.float32, device="cuda")
    dq, dk, dv = [f32(t) for t in q], [f32(t) for t in k], [f32(t) for t in v]
    grad = kernel_block_grad()
    for s in range(world):
        for r in range(world):
            o = (r - s) % world
            grad(q[o], k[r], v[r], o_[o], ls[o], do[o], False, dq[o], dk[r], dv[r])
    lvx.lvx_last_device_error()
    torch.cuda.synchronize()
    dq_r, dk_r, dv_r = _oracle_bwd(host)
    compare(torch.cat(dq, 1), dq_r, "bf16", f"xattn backward x{world}: dQ")
    compare(torch.cat(dk, 1), dk_r, "bf16", f"xattn backward x{world}: dK")
    compare(torch.cat(dv, 1), dv_r, "bf16", f"xattn backward x{world}: dV")


@pytest.mark.parametrize("form", ["ring", "allgather"])
def test_xattn_backward_through_torch_distributed(form):
    """xattn_backward_ring / xattn_backward_sharded through a one-rank NCCL
    group, after the matching forward."""
    import torch.distributed as dist
    from blockwise_long_context_b200.distributed import (xattn_backward_ring,
                                                         xattn_backward_sharded, xattn_forward_ring)
    w, host = _bwd_problem(256, 1500, H=4, H_kv=2)
    dev = {t: x.cuda() for t, x in host.items()}
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        if form == "ring":
            out, lse = xattn_forward_ring(dev["q"], dev["k"], dev["v"])
            dq, dk, dv = xattn_backward_ring(dev["q"], dev["k"], dev["v"], out, lse, dev["do"])
        else:
            out, lse = xattn_forward_sharded(dev["q"], dev["k"], dev["v"], n_local_blocks=2)
            dq, dk, dv = xattn_backward_sharded(dev["q"], dev["k"], dev["v"], out, lse, dev["do"])
        lvx.lvx_last_device_error()
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    dq_r, dk_r, dv_r = _oracle_bwd(host)
    compare(dq, dq_r, "bf16", f"{form}, torch.distributed: dQ")
    compare(dk, dk_r, "bf16", f"{form}, torch.distributed: dK")
    compare(dv, dv_r, "bf16", f"{form}, torch.distributed: dV")
