"""Pins for the fp64 oracle: it is checked against things other than itself.

Each test ties the oracle to a closed form, an invariant of softmax
attention, brute force on tiny inputs, hand-derived fixtures under
tests/golden/, or an independent library routine (torch's fp64
scaled_dot_product_attention and autograd).  The last group plants
plausible mistakes in the oracle and checks that a pin catches each one.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


def _qkv(B=2, S_Q=5, S_KV=13, H=4, H_kv=2, d=8, seed=0, std=1.0):
    q = _rand((B, S_Q, H, d), seed, std)
    k = _rand((B, S_KV, H_kv, d), seed + 1, std)
    v = _rand((B, S_KV, H_kv, d), seed + 2, std)
    return q, k, v


# ---------------------------------------------------------------- closed forms

def test_golden_two_keys():
    with open(os.path.join(GOLDEN, "two_key_closed_form.json")) as f:
        g = json.load(f)
    q = np.array(g["q"])[None, :, None, :]
    k = np.array(g["k"])[None, :, None, :]
    v = np.array(g["v"])[None, :, None, :]
    do = np.array(g["do"])[None, :, None, :]
    o, lse = oracle.attention_fwd(q, k, v, scale=g["scale"])
    np.testing.assert_allclose(o[0, :, 0], g["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], g["lse"], rtol=0, atol=1e-14)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, scale=g["scale"])
    np.testing.assert_allclose(dq[0, :, 0], g["dq"], atol=1e-14)
    np.testing.assert_allclose(dk[0, :, 0], g["dk"], atol=1e-14)
    np.testing.assert_allclose(dv[0, :, 0], g["dv"], atol=1e-14)


def test_golden_causal_uniform():
    with open(os.path.join(GOLDEN, "causal_uniform_closed_form.json")) as f:
        g = json.load(f)
    v = np.array(g["v"])[None, :, None, :]
    S, d = v.shape[1], v.shape[3]
    q = np.zeros((1, S, 1, d))
    k = _rand((1, S, 1, d), 3)
    o, lse = oracle.attention_fwd(q, k, v, causal=True)
    np.testing.assert_allclose(o[0, :, 0], g["o"], atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], g["lse"], atol=1e-14)


def test_single_key_returns_its_value():
    q, k, v = _qkv(S_KV=1)
    o, lse = oracle.attention_fwd(q, k, v)
    for b in range(2):
        for h in range(4):
            g = h // 2
            np.testing.assert_allclose(o[b, :, h], np.broadcast_to(v[b, 0, g], o[b, :, h].shape), atol=1e-14)
            np.testing.assert_allclose(lse[b, h], q[b, :, h] @ k[b, 0, g] / math.sqrt(8), atol=1e-13)


def test_identical_keys_give_mean_of_values():
    q, k, v = _qkv(S_KV=9)
    k[:] = k[:, :1]
    o, lse = oracle.attention_fwd(q, k, v)
    for b in range(2):
        for h in range(4):
            g = h // 2
            np.testing.assert_allclose(o[b, :, h], np.broadcast_to(v[b, :, g].mean(0), o[b, :, h].shape), atol=1e-13)
            np.testing.assert_allclose(lse[b, h], q[b, :, h] @ k[b, 0, g] / math.sqrt(8) + math.log(9), atol=1e-13)


def test_dominant_key_far_above_the_rest():
    """Logits spread over hundreds of natural-log units (the regime the GPU
    parity cases with rising logits and far-below arguments use): a key whose
    logit exceeds every other by > 100 returns its value, and the LSE is that
    logit plus a term below e^-100; two equal spikes return the mean of their
    values with LSE = spike + ln 2 (closed forms)."""
    d, S = 8, 40
    q = np.zeros((1, 1, 1, d)); q[0, 0, 0, 0] = 1.0
    k = np.zeros((1, S, 1, d)); k[0, :, 0, 0] = np.linspace(-300.0, 0.0, S)
    v = _rand((1, S, 1, d), 7)
    sc = 1.0
    k[0, 17, 0, 0] = 150.0                       # 150 above the next largest logit (0)
    out, lse = oracle.attention_fwd(q, k, v, scale=sc)
    assert np.abs(out[0, 0, 0] - v[0, 17, 0]).max() < 1e-60
    assert abs(lse[0, 0, 0] - 150.0) < 1e-12
    k[0, 23, 0, 0] = 150.0                       # a second, equal spike
    out, lse = oracle.attention_fwd(q, k, v, scale=sc)
    assert np.abs(out[0, 0, 0] - 0.5 * (v[0, 17, 0] + v[0, 23, 0])).max() < 1e-14
    assert abs(lse[0, 0, 0] - (150.0 + math.log(2.0))) < 1e-12
    # and the n-block merge stays exact when the blocks' maxima differ by 150 to 370
    # natural-log units
    O, L = oracle.block_partials(q, k, v, 4, scale=sc)
    out_m, lse_m = oracle.merge_partials(O, L)
    assert np.abs(out_m - out).max() < 1e-14 and np.abs(lse_m - lse).max() < 1e-12


def test_rows_sum_to_one():
    q, k, v = _qkv(S_Q=7, S_KV=31)
    for causal in (False, True):
        qq = q if not causal else _qkv(S_Q=31, S_KV=31)[0]
        for h in range(4):
            P = oracle.attention_probs(qq, k, causal=causal, b=1, h=h)
            np.testing.assert_allclose(P.sum(1), 1.0, atol=1e-14)
            assert (P >= 0).all()


def test_brute_force_python_loops():
    """Scalar Python evaluation of the attention definition on a tiny case."""
    q, k, v = _qkv(B=1, S_Q=3, S_KV=4, H=2, H_kv=1, d=3, seed=11)
    sc = 0.37
    o, lse = oracle.attention_fwd(q, k, v, scale=sc)
    for h in range(2):
        for r in range(3):
            logits = [sc * sum(q[0, r, h, c] * k[0, j, 0, c] for c in range(3)) for j in range(4)]
            z = sum(math.exp(x) for x in logits)
            want = [sum(math.exp(logits[j]) * v[0, j, 0, c] for j in range(4)) / z for c in range(3)]
            assert o[0, r, h].tolist() == pytest.approx(want, abs=1e-14)
            assert lse[0, h, r] == pytest.approx(math.log(z), abs=1e-14)


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("n", [1, 2, 3, 4, 7, 13])
def test_merge_of_block_partials_equals_unsplit(n):
    q, k, v = _qkv()
    O, L = oracle.block_partials(q, k, v, n)
    om, lm = oracle.merge_partials(O, L)
    o, lse = oracle.attention_fwd(q, k, v)
    np.testing.assert_allclose(om, o, atol=1e-12)
    np.testing.assert_allclose(lm, lse, atol=1e-12)


@pytest.mark.parametrize("n", [1, 2, 3, 5, 8])
def test_causal_block_merge_equals_unsplit(n):
    q, k, v = _qkv(S_Q=17, S_KV=17)
    O, L = oracle.block_partials(q, k, v, n, causal=True)
    om, lm = oracle.merge_partials(O, L)
    o, lse = oracle.attention_fwd(q, k, v, causal=True)
    np.testing.assert_allclose(om, o, atol=1e-12)
    np.testing.assert_allclose(lm, lse, atol=1e-12)
    # blocks entirely after a row are the merge identity (0, -inf)
    bounds = oracle.kv_block_bounds(17, n)
    for i, (lo, hi) in enumerate(bounds):
        for r in range(17):
            if lo > r or lo >= hi:
                assert np.all(L[i, :, :, r] == -np.inf)
                assert np.all(O[i, :, r] == 0)


def test_block_bounds_cover_sequence():
    for S in (1, 5, 13, 64, 1000):
        for n in range(1, min(S, 9) + 1):
            b = oracle.kv_block_bounds(S, n)
            assert len(b) == n and b[0][0] == 0
            covered = [j for lo, hi in b for j in range(lo, hi)]
            assert covered == list(range(S))
    assert oracle.kv_block_bounds(5, 4) == [(0, 2), (2, 4), (4, 5), (5, 5)]


def test_merge_identity_and_all_empty():
    O = np.zeros((2, 1, 3, 1, 4)); L = np.full((2, 1, 1, 3), -np.inf)
    om, lm = oracle.merge_partials(O, L)
    assert np.all(om == 0) and np.all(lm == -np.inf)
    q, k, v = _qkv()
    O1, L1 = oracle.block_partials(q, k, v, 1)
    O2 = np.concatenate([O1, np.zeros_like(O1)]); L2 = np.concatenate([L1, np.full_like(L1, -np.inf)])
    om, lm = oracle.merge_partials(O2, L2)
    np.testing.assert_allclose(om, O1[0], atol=1e-15)
    np.testing.assert_allclose(lm, L1[0], atol=1e-15)


def test_permutation_invariance_of_kv_pairs():
    q, k, v = _qkv(S_KV=19)
    perm = np.random.default_rng(5).permutation(19)
    o1, l1 = oracle.attention_fwd(q, k, v)
    o2, l2 = oracle.attention_fwd(q, k[:, perm], v[:, perm])
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


def test_causal_first_and_last_rows():
    q, k, v = _qkv(S_Q=11, S_KV=11)
    o, lse = oracle.attention_fwd(q, k, v, causal=True)
    o_nc, lse_nc = oracle.attention_fwd(q, k, v, causal=False)
    for h in range(4):
        np.testing.assert_allclose(o[:, 0, h], v[:, 0, h // 2], atol=1e-14)
    np.testing.assert_allclose(o[:, -1], o_nc[:, -1], atol=1e-14)
    np.testing.assert_allclose(lse[:, :, -1], lse_nc[:, :, -1], atol=1e-14)


def test_gqa_equals_mha_on_repeated_kv():
    q, k, v = _qkv(H=6, H_kv=2)
    kr = np.repeat(k, 3, axis=2); vr = np.repeat(v, 3, axis=2)
    o1, l1 = oracle.attention_fwd(q, k, v)
    o2, l2 = oracle.attention_fwd(q, kr, vr)
    np.testing.assert_allclose(o1, o2, atol=1e-14)
    np.testing.assert_allclose(l1, l2, atol=1e-14)
    do = _rand(o1.shape, 9)
    dq1, dk1, dv1 = oracle.attention_bwd(q, k, v, do)
    dq2, dk2, dv2 = oracle.attention_bwd(q, kr, vr, do)
    np.testing.assert_allclose(dq1, dq2, atol=1e-13)
    np.testing.assert_allclose(dk1, dk2.reshape(2, 13, 2, 3, 8).sum(3), atol=1e-13)
    np.testing.assert_allclose(dv1, dv2.reshape(2, 13, 2, 3, 8).sum(3), atol=1e-13)


def test_row_and_head_selection():
    q, k, v = _qkv(S_Q=9, S_KV=9)
    rows = [0, 4, 8]
    for causal in (False, True):
        o, lse = oracle.attention_fwd(q, k, v, causal=causal)
        os_, ls_ = oracle.attention_fwd(q, k, v, causal=causal, rows=rows, heads=[1, 3])
        np.testing.assert_allclose(os_, o[:, rows][:, :, [1, 3]], atol=1e-15)
        np.testing.assert_allclose(ls_, lse[:, [1, 3]][:, :, rows], atol=1e-15)


# ---------------------------------------------------------------- gradients

def test_gradient_matches_central_differences():
    q, k, v = _qkv(B=1, S_Q=3, S_KV=5, H=2, H_kv=1, d=4, seed=21)
    do = _rand((1, 3, 2, 4), 22)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do)

    def f(q_, k_, v_):
        return float((oracle.attention_fwd(q_, k_, v_)[0] * do).sum())

    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy(); xp[idx] += eps
            xm = x.copy(); xm[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            args[name] = xp; fp = f(args["q"], args["k"], args["v"])
            args[name] = xm; fm = f(args["q"], args["k"], args["v"])
            num[idx] = (fp - fm) / (2 * eps)
        rel = np.abs(num - g).max() / np.abs(g).max()
        assert rel < 1e-7, (name, rel)


def test_gradient_invariants():
    q, k, v = _qkv(S_KV=17)
    do = _rand(q.shape, 31)
    for causal in (False, True):
        if causal:
            q, k, v = _qkv(S_Q=17, S_KV=17, seed=3)
            do = _rand(q.shape, 32)
        dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal=causal)
        # rows of P sum to 1  =>  sum_j dV_j = sum over the group's query rows of dO
        grp = do.reshape(do.shape[0], do.shape[1], 2, 2, 8).sum(axis=(1, 3))
        np.testing.assert_allclose(dv.sum(1), grp, atol=1e-12)
        # rows of dS sum to 0  =>  sum_j dK_j = 0
        np.testing.assert_allclose(dk.sum(1), 0.0, atol=1e-12)


def test_bwd_keys_matches_full_backward():
    q, k, v = _qkv(S_Q=9, S_KV=21)
    do = _rand(q.shape, 41)
    for causal in (False,):
        dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal=causal)
        keys = [0, 7, 20]
        dks, dvs = oracle.attention_bwd_keys(q, k, v, do, keys, [1], causal=causal, row_chunk=4)
        np.testing.assert_allclose(dks[:, :, 0], dk[:, keys, 1], atol=1e-13)
        np.testing.assert_allclose(dvs[:, :, 0], dv[:, keys, 1], atol=1e-13)
    q, k, v = _qkv(S_Q=21, S_KV=21)
    do = _rand(q.shape, 42)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal=True)
    dks, dvs = oracle.attention_bwd_keys(q, k, v, do, [3, 20], [0, 1], causal=True, row_chunk=5)
    np.testing.assert_allclose(dks, dk[:, [3, 20]], atol=1e-13)
    np.testing.assert_allclose(dvs, dv[:, [3, 20]], atol=1e-13)


def test_bwd_rows_matches_full_backward():
    for causal, (S_Q, S_KV) in ((False, (9, 21)), (True, (21, 21))):
        q, k, v = _qkv(S_Q=S_Q, S_KV=S_KV)
        do = _rand(q.shape, 43)
        dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal=causal)
        rows = [0, 5, S_Q - 1]
        np.testing.assert_allclose(oracle.attention_bwd_rows(q, k, v, do, rows, causal=causal),
                                   dq[:, rows], atol=1e-13)


def test_bwd_keys_tail_rows_exact_under_causal_mask():
    q, k, v = _qkv(S_Q=40, S_KV=40)
    do = _rand(q.shape, 44)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal=True)
    keys = np.arange(30, 40)
    dks, dvs = oracle.attention_bwd_keys(q, k, v, do, keys, [0, 1], causal=True, rows=np.arange(30, 40))
    np.testing.assert_allclose(dks, dk[:, keys], atol=1e-13)
    np.testing.assert_allclose(dvs, dv[:, keys], atol=1e-13)


# ---------------------------------------------------------------- library cross-check

@pytest.mark.parametrize("causal,H,H_kv,S_Q,S_KV", [(False, 4, 2, 5, 13), (True, 4, 4, 9, 9), (False, 6, 1, 3, 7)])
def test_against_torch_sdpa_and_autograd(causal, H, H_kv, S_Q, S_KV):
    q, k, v = _qkv(S_Q=S_Q, S_KV=S_KV, H=H, H_kv=H_kv, seed=51)
    do = _rand(q.shape, 52)
    o, lse = oracle.attention_fwd(q, k, v, causal=causal)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal=causal)
    tq = torch.tensor(q).permute(0, 2, 1, 3).requires_grad_()
    tk = torch.tensor(k).permute(0, 2, 1, 3).requires_grad_()
    tv = torch.tensor(v).permute(0, 2, 1, 3).requires_grad_()
    rep = H // H_kv
    to = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(rep, 1), tv.repeat_interleave(rep, 1), is_causal=causal)
    to.backward(torch.tensor(do).permute(0, 2, 1, 3))
    np.testing.assert_allclose(o, to.detach().permute(0, 2, 1, 3).numpy(), atol=1e-13)
    np.testing.assert_allclose(dq, tq.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12)
    # LSE against torch's logsumexp of the masked logits
    s = torch.einsum("bhrc,bhjc->bhrj", tq.detach(), tk.detach().repeat_interleave(rep, 1)) / math.sqrt(8)
    if causal:
        s = s.masked_fill(torch.ones(S_Q, S_KV, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), atol=1e-13)


def test_kv_recompute_exact_on_integers():
    rng = np.random.default_rng(7)
    y = rng.integers(-3, 4, size=(2, 5, 6)).astype(np.float64)
    wk = rng.integers(-2, 3, size=(6, 4)).astype(np.float64)
    wv = rng.integers(-2, 3, size=(6, 4)).astype(np.float64)
    K, V = oracle.kv_recompute(y, wk, wv)
    for b in range(2):
        for s in range(5):
            for c in range(4):
                assert K[b, s, c] == sum(int(y[b, s, e]) * int(wk[e, c]) for e in range(6))
                assert V[b, s, c] == sum(int(y[b, s, e]) * int(wv[e, c]) for e in range(6))
    Ks, Vs = oracle.kv_recompute(y, wk, wv, rows=[1, 4])
    np.testing.assert_array_equal(Ks, K[:, [1, 4]])


def test_kv_recompute_bwd_matches_central_differences():
    rng = np.random.default_rng(17)
    y = rng.standard_normal((6, 5)); wk = rng.standard_normal((5, 4)); wv = rng.standard_normal((5, 4))
    dk = rng.standard_normal((6, 4)); dv = rng.standard_normal((6, 4))
    dy, dwk, dwv = oracle.kv_recompute_bwd(y, wk, wv, dk, dv)

    def f(y_, wk_, wv_):
        K, V = oracle.kv_recompute(y_, wk_, wv_)
        return float((K * dk).sum() + (V * dv).sum())

    eps = 1e-6
    for x, g, name in ((y, dy, "y"), (wk, dwk, "wk"), (wv, dwv, "wv")):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp = x.copy(); xp[idx] += eps
            xm = x.copy(); xm[idx] -= eps
            args = {"y": y, "wk": wk, "wv": wv}
            args[name] = xp; fp = f(args["y"], args["wk"], args["wv"])
            args[name] = xm; fm = f(args["y"], args["wk"], args["wv"])
            num[idx] = (fp - fm) / (2 * eps)
        np.testing.assert_allclose(num, g, rtol=1e-7, atol=1e-7)


def test_kv_recompute_bwd_exact_on_integers_and_batches():
    rng = np.random.default_rng(18)
    y = rng.integers(-3, 4, size=(2, 5, 6)).astype(np.float64)
    wk = rng.integers(-2, 3, size=(6, 4)).astype(np.float64)
    wv = rng.integers(-2, 3, size=(6, 4)).astype(np.float64)
    dk = rng.integers(-2, 3, size=(2, 5, 4)).astype(np.float64)
    dv = rng.integers(-2, 3, size=(2, 5, 4)).astype(np.float64)
    dy, dwk, dwv = oracle.kv_recompute_bwd(y, wk, wv, dk, dv)
    for e in range(6):
        for c in range(4):
            assert dwk[e, c] == sum(int(y[b, s, e]) * int(dk[b, s, c]) for b in range(2) for s in range(5))
            assert dwv[e, c] == sum(int(y[b, s, e]) * int(dv[b, s, c]) for b in range(2) for s in range(5))
    for b in range(2):
        for s in range(5):
            for e in range(6):
                assert dy[b, s, e] == sum(int(dk[b, s, c]) * int(wk[e, c]) + int(dv[b, s, c]) * int(wv[e, c])
                                          for c in range(4))
    dys, _, _ = oracle.kv_recompute_bwd(y, wk, wv, dk, dv, rows=[0, 3])
    np.testing.assert_array_equal(dys, dy[:, [0, 3]])


# ---------------------------------------------------------------- planted mistakes

def _pins_fail(monkeypatch, name, bad):
    monkeypatch.setattr(oa, name, bad)
    failed = 0
    for t in (test_against_torch_sdpa_and_autograd,):
        for args in [(False, 4, 2, 5, 13), (True, 4, 4, 9, 9)]:
            try:
                t(*args)
            except AssertionError:
                failed += 1
    return failed


def test_planted_wrong_gqa_mapping_is_caught(monkeypatch):
    assert _pins_fail(monkeypatch, "_kv_head", lambda h, H, H_kv: h % H_kv) > 0


def test_planted_wrong_scale_is_caught(monkeypatch):
    assert _pins_fail(monkeypatch, "_default_scale", lambda d, s: 1.0 / d) > 0


def test_planted_causal_off_by_one_is_caught(monkeypatch):
    def bad(qh, kg, scale, causal, rows, key_offset):
        s = scale * (qh @ kg.T)
        if causal:
            keys = key_offset + np.arange(kg.shape[0])
            s = np.where(keys[None, :] < rows[:, None] + 2, s, -np.inf)
        return s
    monkeypatch.setattr(oa, "_logits", bad)
    with pytest.raises(AssertionError):
        test_golden_causal_uniform()
