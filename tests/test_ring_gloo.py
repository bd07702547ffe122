"""Ring Attention's exchange across ranks, on CPU with the gloo backend.

``run_ring_forward`` / ``run_ring_backward`` (the drivers the GPU path uses)
move each key/value block, and in the backward its dK/dV accumulators, around
two to four gloo ranks (with four, one rank's shard is empty).  The per-block steps here are CPU stand-ins: the
forward partial is the oracle's block partial, and the block gradient is the
textbook blockwise gradient with the global log-sum-exp (written out below).
The assembled outputs and gradients must equal the oracle's full attention
and its gradient.  The library's kernels need a GPU;
``tests/test_parity_ring.py`` runs those.
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


@pytest.mark.parametrize("world", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_schedule_visits_every_block_once(world, causal):
    sys.path.insert(0, ROOT)
    from blockwise_long_context_b200.ring import ring_schedule
    for rank in range(world):
        seen = [ring_schedule(rank, world, s, causal) for s in range(world)]
        assert sorted(src for src, _ in seen) == list(range(world))
        for src, mode in seen:
            want = "full" if not causal or src < rank else ("diag" if src == rank else "skip")
            assert mode == want, (rank, src, mode)
    # step s: rank r holds the block that rank r-1 held at step s-1
    for s in range(1, world):
        for rank in range(world):
            assert ring_schedule(rank, world, s, causal)[0] == \
                ring_schedule((rank - 1) % world, world, s - 1, causal)[0]


@pytest.mark.parametrize("world", [2, 3, 4, 8])
def test_zigzag_balances_causal_work(world):
    """With the zigzag layout every rank computes the same causal work at every
    step (two chunk-squares: two full pairs, or one full pair and two diagonal
    halves); with the contiguous layout the last rank computes W - 1 full blocks
    and the diagonal while rank 0 computes only its diagonal."""
    sys.path.insert(0, ROOT)
    from blockwise_long_context_b200.ring import chunks_of, pair_mode
    weight = {"full": 1.0, "diag": 0.5, "skip": 0.0}
    for s in range(world):
        per_rank = []
        for r in range(world):
            theirs = chunks_of((r - s) % world, world, "zigzag")
            per_rank.append(sum(weight[pair_mode(cq, ck, True)]
                                for cq in chunks_of(r, world, "zigzag") for ck in theirs))
        assert per_rank == [2.0] * world, (s, per_rank)
    totals = [sum(weight[pair_mode(r, (r - s) % world, True)] for s in range(world))
              for r in range(world)]
    assert totals == [r + 0.5 for r in range(world)]
    # the zigzag chunks of all ranks tile the sequence once
    for S in (9, 23, 64, 1000):
        from blockwise_long_context_b200.ring import rank_bounds
        rows = sorted(i for r in range(world) for lo, hi in rank_bounds(S, world, r, "zigzag")
                      for i in range(lo, hi))
        assert rows == list(range(S))


def _block_grad(q, k, v, out, lse, do, diagonal, scale):
    """Textbook blockwise gradient of one (query block, key block) pair with the
    rows' global log-sum-exp: P = exp(s q.k - lse), dV = P^T dO, dP = dO V^T,
    D = rowsum(dO o O), dS = P o (dP - D), dQ = s dS K, dK = s dS^T Q (fp64)."""
    B, Sq, H, d = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    grp = H // Hkv
    dq = np.zeros(q.shape); dk = np.zeros(k.shape); dv = np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            g = h // grp
            s = scale * q[b, :, h] @ k[b, :, g].T
            if diagonal:
                s = np.where(np.arange(Sk)[None, :] <= np.arange(Sq)[:, None], s, -np.inf)
            P = np.exp(s - lse[b, h][:, None])
            dv[b, :, g] += P.T @ do[b, :, h]
            dP = do[b, :, h] @ v[b, :, g].T
            D = (do[b, :, h] * out[b, :, h]).sum(-1)
            dS = P * (dP - D[:, None])
            dq[b, :, h] = scale * dS @ k[b, :, g]
            dk[b, :, g] += scale * dS.T @ q[b, :, h]
    return dq, dk, dv


def _rows(a, bounds):
    """This rank's rows: its chunks, concatenated in order."""
    return np.concatenate([a[:, lo:hi] for lo, hi in bounds], axis=1)


def _worker(rank, world, port, causal, layout, results):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import oracle
    from blockwise_long_context_b200.ring import (RingExchange, rank_bounds, run_ring_backward,
                                                  run_ring_forward)
    rng = np.random.default_rng(21)                  # the same full problem on every rank
    B, H, H_kv, d = 2, 4, 2, 8
    S_Q, S_KV = (23, 23) if causal else (13, 29)
    if world == 4:                                   # a trailing shard is empty: 3, 3, 3, 0
        S_Q, S_KV = (9, 9) if causal else (9, 29)
    q = rng.standard_normal((B, S_Q, H, d))
    k = rng.standard_normal((B, S_KV, H_kv, d))
    v = rng.standard_normal((B, S_KV, H_kv, d))
    do = rng.standard_normal((B, S_Q, H, d))
    scale = 1.0 / np.sqrt(d)
    qb, kb = rank_bounds(S_Q, world, rank, layout), rank_bounds(S_KV, world, rank, layout)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).float()
    q_r, do_r = t(_rows(q, qb)), t(_rows(do, qb))
    k_r, v_r = t(_rows(k, kb)), t(_rows(v, kb))

    def partial(qq, kk, vv, o, l, diagonal):
        if qq.shape[1] == 0 or kk.shape[1] == 0:
            return
        O, L = oracle.block_partials(qq.double().numpy(), kk.double().numpy(), vv.double().numpy(),
                                     1, causal=diagonal)
        o.copy_(torch.from_numpy(np.transpose(O, (0, 1, 3, 2, 4))))
        l.copy_(torch.from_numpy(L))

    def merge(o, l):
        out, lse = oracle.merge_partials(np.transpose(o.double().numpy(), (0, 1, 3, 2, 4)),
                                         l.double().numpy())
        return torch.from_numpy(out), torch.from_numpy(lse)

    ex = RingExchange()
    out_r, lse_r = run_ring_forward(q_r, k_r, v_r, partial, merge, ex, causal, layout)

    def grad(qq, kk, vv, oo, ll, dd, diagonal, dq_acc, dk_acc, dv_acc):
        parts = _block_grad(qq.double().numpy(), kk.double().numpy(), vv.double().numpy(),
                            oo.double().numpy(), ll.double().numpy(), dd.double().numpy(),
                            diagonal, scale)
        for acc, part in zip((dq_acc, dk_acc, dv_acc), parts):
            acc += torch.from_numpy(part).float()

    dq_r, dk_r, dv_r = run_ring_backward(q_r, k_r, v_r, out_r, lse_r, do_r, grad, ex, causal, layout)

    qf, kf, vf, dof = (t(a).double().numpy() for a in (q, k, v, do))   # the float32 inputs
    o_ref, l_ref = oracle.attention_fwd(qf, kf, vf, causal=causal)
    dq_ref, dk_ref, dv_ref = oracle.attention_bwd(qf, kf, vf, dof, causal=causal)
    rel = lambda a, b: (float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30)) if b.size
                        else 0.0)   # the rank with an empty shard has nothing to compare
    lse_rows = np.concatenate([l_ref[:, :, lo:hi] for lo, hi in qb], axis=2)
    results[rank] = dict(
        out=rel(out_r.numpy(), _rows(o_ref, qb)), lse=rel(lse_r.numpy(), lse_rows),
        dq=rel(dq_r.double().numpy(), _rows(dq_ref, qb)),
        dk=rel(dk_r.double().numpy(), _rows(dk_ref, kb)),
        dv=rel(dv_r.double().numpy(), _rows(dv_ref, kb)))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
def test_ring_forward_and_backward_match_attention(world, causal, layout):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.spawn(_worker, args=(world, port, causal, layout, results), nprocs=world, join=True)
        res = dict(results)
    assert sorted(res) == list(range(world))
    for rank, errs in res.items():
        # float32 accumulation and transfers against the fp64 definition
        for name, e in errs.items():
            assert e < 1e-5, (rank, name, e)
