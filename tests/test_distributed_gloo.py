"""LV-XAttn's exchange across ranks, on CPU with the gloo backend.

The distributed forward keeps one key/value shard per rank, gathers every
rank's block partials (O_i, L_i) and merges them.  These tests check the host
side of that on CPU: the shard partition, and that the partials of each
rank's shard, gathered over two and three gloo ranks by ``gather_partials``
(the function the GPU path uses), merge to exact attention on every rank;
and that in the ring form (``run_xattn_ring``: query rows sharded too, query
blocks travelling, partials returned to their owner) every rank ends with
exact attention for its own rows, over two to four ranks.
The partials and the merge here come from the fp64 oracle -- the library's
kernels need a GPU; ``tests/test_parity_distributed.py`` runs those.
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("S_KV,world", [(1000, 2), (1000, 3), (7, 3), (64, 8), (5, 5)])
def test_shards_partition_the_keys(S_KV, world):
    sys.path.insert(0, ROOT)
    from blockwise_long_context_b200.distributed import shard_bounds
    bounds = [shard_bounds(S_KV, world, r) for r in range(world)]
    assert bounds[0][0] == 0 and bounds[-1][1] == S_KV
    for (lo, hi), (lo2, _) in zip(bounds, bounds[1:]):
        assert lo <= hi == lo2
    per = -(-S_KV // world)
    assert all(hi - lo <= per for lo, hi in bounds)


def _to_kernel_layout(O, L):
    """oracle partials O [n, B, R, H, d], L [n, B, H, R] -> kernel layout
    O [n, B, H, R, d], L [n, B, H, R] (float32 tensors, as the GPU path gathers)."""
    return (torch.from_numpy(np.ascontiguousarray(np.transpose(O, (0, 1, 3, 2, 4)))).float(),
            torch.from_numpy(np.ascontiguousarray(L)).float())


def _worker(rank, world, port, n_local, results):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import oracle
    from blockwise_long_context_b200.distributed import gather_partials, shard_bounds
    rng = np.random.default_rng(7)                 # the same full problem on every rank
    B, S_Q, H, H_kv, d, S_KV = 2, 5, 4, 2, 8, 23
    q = rng.standard_normal((B, S_Q, H, d))
    k = rng.standard_normal((B, S_KV, H_kv, d))
    v = rng.standard_normal((B, S_KV, H_kv, d))
    lo, hi = shard_bounds(S_KV, world, rank)
    O, L = oracle.block_partials(q, k[:, lo:hi], v[:, lo:hi], n_local)
    o_loc, l_loc = _to_kernel_layout(O, L)
    o_all, l_all = gather_partials(o_loc, l_loc)
    assert o_all.shape[0] == world * n_local and l_all.shape[0] == world * n_local
    # back to the oracle layout, merged by the oracle
    O_all = np.transpose(o_all.double().numpy(), (0, 1, 3, 2, 4))
    out, lse = oracle.merge_partials(O_all, l_all.double().numpy())
    o_ref, l_ref = oracle.attention_fwd(q, k, v)
    results[rank] = (float(np.abs(out - o_ref).max()), float(np.abs(lse - l_ref).max()),
                     o_all.double().numpy().sum())
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,n_local", [(2, 1), (3, 2)])
def test_gathered_shard_partials_merge_to_attention(world, n_local):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.spawn(_worker, args=(world, port, n_local, results), nprocs=world, join=True)
        res = dict(results)
    assert sorted(res) == list(range(world))
    for rank, (eo, el, _) in res.items():
        # float32 partials (as gathered on GPUs) against the fp64 definition
        assert eo < 1e-5 and el < 1e-5, (rank, eo, el)
    # every rank gathered the same tensors
    sums = {r: v[2] for r, v in res.items()}
    assert len(set(sums.values())) == 1


def _ring_worker(rank, world, port, n_local, results):
    """LV-XAttn's ring form: query rows and keys both sharded, query blocks
    travelling, partials sent back to their owner and merged there."""
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import oracle
    from blockwise_long_context_b200.distributed import run_xattn_ring, shard_bounds
    from blockwise_long_context_b200.ring import RingExchange
    rng = np.random.default_rng(9)
    B, S_Q, H, H_kv, d, S_KV = 2, 11, 4, 2, 8, 31      # uneven shards for 2 and 3 ranks
    if world == 4:
        S_Q = 9                                        # query shards 3, 3, 3, 0
    q = rng.standard_normal((B, S_Q, H, d))
    k = rng.standard_normal((B, S_KV, H_kv, d))
    v = rng.standard_normal((B, S_KV, H_kv, d))
    qlo, qhi = shard_bounds(S_Q, world, rank)
    klo, khi = shard_bounds(S_KV, world, rank)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).float()

    def partial(qq, kk, vv, o, l, diagonal):
        if qq.shape[1] == 0 or kk.shape[1] == 0:
            return
        n = min(o.shape[0], kk.shape[1])     # slots past the shard's keys stay (0, -inf)
        O, L = oracle.block_partials(qq.double().numpy(), kk.double().numpy(), vv.double().numpy(), n)
        o[:n].copy_(torch.from_numpy(np.transpose(O, (0, 1, 3, 2, 4))))
        l[:n].copy_(torch.from_numpy(L))

    def merge(o, l):
        out, lse = oracle.merge_partials(np.transpose(o.double().numpy(), (0, 1, 3, 2, 4)),
                                         l.double().numpy())
        return torch.from_numpy(out), torch.from_numpy(lse)

    out, lse = run_xattn_ring(t(q[:, qlo:qhi]), t(k[:, klo:khi]), t(v[:, klo:khi]), partial, merge,
                              RingExchange(), n_local)
    o_ref, l_ref = oracle.attention_fwd(*(t(a).double().numpy() for a in (q, k, v)))
    err = lambda a, b: float(np.abs(a - b).max()) if b.size else 0.0   # empty shard: nothing
    results[rank] = (err(out.numpy(), o_ref[:, qlo:qhi]), err(lse.numpy(), l_ref[:, :, qlo:qhi]))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,n_local", [(2, 1), (3, 1), (4, 1), (3, 4)])
def test_ring_form_query_blocks_travel_and_partials_merge_at_their_owner(world, n_local):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.spawn(_ring_worker, args=(world, port, n_local, results), nprocs=world, join=True)
        res = dict(results)
    assert sorted(res) == list(range(world))
    for rank, (eo, el) in res.items():
        assert eo < 1e-5 and el < 1e-5, (rank, eo, el)


def _block_grad(q, k, v, out, lse, do, scale):
    """Textbook blockwise gradient of one (query block, key shard) pair with the
    rows' global log-sum-exp, written out here (fp64): P = exp(s q.k - lse),
    dV = P^T dO, dP = dO V^T, D = rowsum(dO o O), dS = P o (dP - D),
    dQ = s dS K, dK = s dS^T Q."""
    B, Sq, H, d = q.shape
    grp = H // k.shape[2]
    dq = np.zeros(q.shape); dk = np.zeros(k.shape); dv = np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            g = h // grp
            P = np.exp(scale * q[b, :, h] @ k[b, :, g].T - lse[b, h][:, None])
            dv[b, :, g] += P.T @ do[b, :, h]
            dS = P * (do[b, :, h] @ v[b, :, g].T - (do[b, :, h] * out[b, :, h]).sum(-1)[:, None])
            dq[b, :, h] = scale * dS @ k[b, :, g]
            dk[b, :, g] += scale * dS.T @ q[b, :, h]
    return dq, dk, dv


def _bwd_worker(rank, world, port, form, results):
    """LV-XAttn's backward across ranks with CPU block steps: the ring form
    (query blocks and their dQ accumulators travel, dK/dV stay with the
    stationary shard) and the all-gather form (all query rows on every rank,
    dQ contributions all-reduced)."""
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import oracle
    from blockwise_long_context_b200.distributed import (run_xattn_ring_backward,
                                                         run_xattn_sharded_backward, shard_bounds)
    from blockwise_long_context_b200.ring import RingExchange
    rng = np.random.default_rng(13)
    B, S_Q, H, H_kv, d, S_KV = 2, 11, 4, 2, 8, 31      # uneven shards for 2 and 3 ranks
    if world == 4:
        S_Q = 9                                        # query shards 3, 3, 3, 0
    q = rng.standard_normal((B, S_Q, H, d))
    k = rng.standard_normal((B, S_KV, H_kv, d))
    v = rng.standard_normal((B, S_KV, H_kv, d))
    do = rng.standard_normal((B, S_Q, H, d))
    scale = 1.0 / np.sqrt(d)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).float()
    qf, kf, vf, dof = (t(a).double().numpy() for a in (q, k, v, do))   # the float32 inputs
    o_ref, l_ref = oracle.attention_fwd(qf, kf, vf)
    dq_ref, dk_ref, dv_ref = oracle.attention_bwd(qf, kf, vf, dof)

    def grad(qq, kk, vv, oo, ll, dd, diagonal, dq_acc, dk_acc, dv_acc):
        assert not diagonal
        if qq.shape[1] == 0 or kk.shape[1] == 0:
            return
        parts = _block_grad(qq.double().numpy(), kk.double().numpy(), vv.double().numpy(),
                            oo.double().numpy(), ll.double().numpy(), dd.double().numpy(), scale)
        for acc, part in zip((dq_acc, dk_acc, dv_acc), parts):
            acc += torch.from_numpy(part).float()

    klo, khi = shard_bounds(S_KV, world, rank)
    if form == "ring":
        qlo, qhi = shard_bounds(S_Q, world, rank)
        dq, dk, dv = run_xattn_ring_backward(
            t(q[:, qlo:qhi]), t(k[:, klo:khi]), t(v[:, klo:khi]), t(o_ref[:, qlo:qhi]),
            t(l_ref[:, :, qlo:qhi]), t(do[:, qlo:qhi]), grad, RingExchange())
    else:
        qlo, qhi = 0, S_Q
        dq, dk, dv = run_xattn_sharded_backward(t(q), t(k[:, klo:khi]), t(v[:, klo:khi]), t(o_ref),
                                                t(l_ref), t(do), grad)
    rel = lambda a, b: (float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30)) if b.size
                        else 0.0)   # a rank with an empty shard has nothing to compare
    results[rank] = dict(dq=rel(dq.double().numpy(), dq_ref[:, qlo:qhi]),
                         dk=rel(dk.double().numpy(), dk_ref[:, klo:khi]),
                         dv=rel(dv.double().numpy(), dv_ref[:, klo:khi]),
                         shapes=(tuple(dq.shape), tuple(dk.shape)))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("form", ["ring", "allgather"])
def test_xattn_backward_across_ranks_matches_the_gradient(world, form):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.spawn(_bwd_worker, args=(world, port, form, results), nprocs=world, join=True)
        res = dict(results)
    assert sorted(res) == list(range(world))
    for rank, errs in res.items():
        for name in ("dq", "dk", "dv"):
            # float32 accumulation and transfers against the fp64 gradient
            assert errs[name] < 1e-5, (form, rank, name, errs)
