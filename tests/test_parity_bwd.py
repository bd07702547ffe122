"""Backward parity: dQ, dK, dV from the CUDA path against the fp64 oracle.

The GPU backward recomputes P from its own forward's log-sum-exp; the
oracle computes the textbook gradient from its own fp64 forward.  Small
cases compare every element; full-size workloads compare dQ on sampled rows
and dK, dV on sampled keys of one key/value head (the oracle evaluates each
query row's full softmax to get them), plus the gradient invariants
sum_j dV_j = sum_r dO_r (per group) and sum_j dK_j = 0, which hold for any
size.
"""

import numpy as np
import pytest
import torch

import oracle
from blockwise_long_context_b200 import inputs
from blockwise_long_context_b200 import binding as lvx
from tests._parity import compare, sample_rows

pytestmark = pytest.mark.gpu

SMALL = [
    # name,            B, H, H_kv, d,  S_Q, S_KV, causal, dtype
    ("bf16_d128_gqa",    1, 4, 2,  128, 300, 1000, False, "bf16"),
    ("bf16_d64",         2, 2, 2,   64, 257,  777, False, "bf16"),
    ("bf16_causal",      1, 2, 2,  128, 700,  700, True,  "bf16"),
    ("bf16_causal_d64",  1, 4, 1,   64, 333,  333, True,  "bf16"),
    ("bf16_tiny",        1, 1, 1,  128,   1,    1, False, "bf16"),
    ("bf16_d96_simt",    1, 2, 1,   96, 100,  300, False, "bf16"),
    ("f32_small",        1, 2, 1,   64, 128,  256, False, "f32"),
    ("f32_causal",       1, 1, 1,   32,  70,   70, True,  "f32"),
]


def _workload(B, H, H_kv, d, S_Q, S_KV, causal, dtype):
    base = inputs.WORKLOADS["C0" if dtype == "f32" else "C2"]
    return base.scaled(B=B, H=H, H_kv=H_kv, d=d, S_Q=S_Q, S_KV=S_KV, causal=causal, dtype=dtype,
                       n_blocks=1 if S_KV < 8 else 4, backward=True, d_embed=0)


def _run(w, host):
    dev = {k: t.cuda() for k, t in host.items()}
    out, lse = lvx.attention_forward(dev["q"], dev["k"], dev["v"], w.n_blocks, w.causal)
    dq, dk, dv = lvx.attention_backward(dev["q"], dev["k"], dev["v"], out, lse, dev["do"], w.causal)
    lvx.lvx_last_device_error()
    torch.cuda.synchronize()
    return out, lse, dq, dk, dv


def _invariants(w, host, dk, dv, tol=1e-2):
    grp = w.H // w.H_kv
    do = host["do"].double().numpy()
    want_dv = do.reshape(w.B, w.S_Q, w.H_kv, grp, w.d).sum(axis=(1, 3))
    got_dv = dv.double().cpu().numpy().sum(axis=1)
    rel = np.linalg.norm(got_dv - want_dv) / np.linalg.norm(want_dv)
    assert rel <= tol, f"sum_j dV_j != sum_r dO_r: rel {rel:.2e}"
    dk64 = dk.double().cpu().numpy()
    # relative to the summed magnitudes, with an absolute floor for cases where
    # dK itself is rounding noise (e.g. a single key, where dS = 0 exactly)
    scale = max(np.linalg.norm(np.abs(dk64).sum(axis=1)), 1e-3)
    rel_k = np.linalg.norm(dk64.sum(axis=1)) / scale
    assert rel_k <= tol, f"sum_j dK_j != 0: {rel_k:.2e}"


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_backward_small(case):
    name, *shape = case
    w = _workload(*shape)
    host = inputs.make(w, tensors=("q", "k", "v", "do"))
    out, lse, dq, dk, dv = _run(w, host)
    q, k, v, do = (host[t].double().numpy() for t in ("q", "k", "v", "do"))
    dq_r, dk_r, dv_r = oracle.attention_bwd(q, k, v, do, causal=w.causal)
    compare(dq, dq_r, w.dtype, f"{name}: dQ")
    compare(dk, dk_r, w.dtype, f"{name}: dK")
    compare(dv, dv_r, w.dtype, f"{name}: dV")
    _invariants(w, host, dk, dv, tol=1e-2 if w.dtype == "bf16" else 1e-5)


def test_backward_far_below_the_maximum():
    """Keys whose logits lie far below the row's log-sum-exp: P = exp2(x) with
    x < -126 (log2 units), where the kernel's FMA-pipe exponential is at its
    clamp.  Query head 0 sees a spike at key 262 ~88 natural-log units above
    every other key, so most of its arguments are there; head 1 sees the
    same keys through a logit ramp of ~2 per 128-key tile, which gives the
    compared tensors gradients of ordinary size."""
    rng = np.random.default_rng(12)
    B, H, H_kv, d, S_Q, S_KV = 1, 2, 1, 128, 130, 1000
    q = rng.standard_normal((B, S_Q, H, d)) * 0.5
    k = rng.standard_normal((B, S_KV, H_kv, d)) * 0.5
    v = rng.standard_normal((B, S_KV, H_kv, d))
    do = rng.standard_normal((B, S_Q, H, d)) * 0.05   # dV of the spike key stays ~1
    q[:, :, 0, 0], q[:, :, 1, 0] = 16.0, 4.0
    q[:, :, 0, 1], q[:, :, 1, 1] = 16.0, 0.0
    k[0, :, 0, 0] = 6.0 * ((np.arange(S_KV) % 500) // 128)
    k[0, :, 0, 1] = 0.0
    k[0, 262, 0, 1] = 80.0
    host = {name: torch.from_numpy(t).to(torch.bfloat16)
            for name, t in (("q", q), ("k", k), ("v", v), ("do", do))}
    w = _workload(B, H, H_kv, d, S_Q, S_KV, False, "bf16")
    out, lse, dq, dk, dv = _run(w, host)
    for name, t in (("dQ", dq), ("dK", dk), ("dV", dv)):
        assert torch.isfinite(t.float()).all(), f"{name} not finite"
    q, k, v, do = (host[t].double().numpy() for t in ("q", "k", "v", "do"))
    dq_r, dk_r, dv_r = oracle.attention_bwd(q, k, v, do)
    compare(dq, dq_r, "bf16", "far below: dQ")
    compare(dk, dk_r, "bf16", "far below: dK")
    compare(dv, dv_r, "bf16", "far below: dV")
    _invariants(w, host, dk, dv)


@pytest.mark.parametrize("cfg", ["C2", "C4", "C3"])
def test_backward_full_size_sampled(cfg):
    """dQ on 256 sampled rows of every head and batch (first, last and block-edge
    rows included); dK, dV on 1024 sampled keys of every KV head of batch 0
    (C3: its tail keys, see below); the gradient invariants over everything."""
    w = inputs.WORKLOADS[cfg]
    host = inputs.make(w, tensors=("q", "k", "v", "do"))
    out, lse, dq, dk, dv = _run(w, host)
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    q, k, v, do = (host[t].double().numpy() for t in ("q", "k", "v", "do"))
    # dQ on sampled rows of every head: needs only those rows' softmax
    rows = sample_rows(w.S_Q, w.n_blocks, count=256)
    dq_ref = oracle.attention_bwd_rows(q, k, v, do, rows, causal=w.causal)
    compare(dq[:, rows], dq_ref, "bf16", f"{cfg}: dQ (sampled rows)")
    B0 = 0
    if cfg == "C3":
        # causal tail keys j >= S-256 get gradient only from rows r >= S-256 (all
        # keys of a scaled-down C3 are compared in test_backward_c3_scaled_down)
        keys = np.arange(w.S_KV - 256, w.S_KV)
        heads = list(range(w.H_kv))
        dk_r, dv_r = oracle.attention_bwd_keys(q, k, v, do, keys, heads, causal=True, batches=[B0],
                                               rows=np.arange(w.S_Q - 256, w.S_Q))
    else:
        keys = sample_rows(w.S_KV, w.n_blocks, count=1056, seed=1)   # >= 1024 after the union
        heads = list(range(w.H_kv))
        dk_r, dv_r = oracle.attention_bwd_keys(q, k, v, do, keys, heads, causal=w.causal,
                                               batches=[B0])
    compare(dk[B0][keys][:, heads], dk_r[0], "bf16", f"{cfg}: dK (sampled keys, every KV head)")
    compare(dv[B0][keys][:, heads], dv_r[0], "bf16", f"{cfg}: dV (sampled keys, every KV head)")
    _invariants(w, host, dk, dv)


def test_backward_c3_scaled_down():
    """C3's shape (H = 32, d = 128, n = 8, causal) at S = 16384 on the GPU, with
    dQ, dK and dV compared in full: every row, key and head (the fp64 oracle
    evaluates one head at a time, a few seconds each), plus the gradient
    invariants."""
    w = inputs.WORKLOADS["C3"].scaled(S_Q=16384, S_KV=16384)
    host = inputs.make(w, tensors=("q", "k", "v", "do"))
    out, lse, dq, dk, dv = _run(w, host)
    for h in range(w.H):
        sl = {t: host[t][:, :, h:h + 1].double().numpy() for t in ("q", "k", "v", "do")}
        dq_r, dk_r, dv_r = oracle.attention_bwd(sl["q"], sl["k"], sl["v"], sl["do"], causal=True)
        compare(dq[:, :, h:h + 1], dq_r, "bf16", f"C3 at S=16384, head {h}: dQ")
        compare(dk[:, :, h:h + 1], dk_r, "bf16", f"C3 at S=16384, head {h}: dK")
        compare(dv[:, :, h:h + 1], dv_r, "bf16", f"C3 at S=16384, head {h}: dV")
    _invariants(w, host, dk, dv)


ACCUM = [
    # name,                B, H, H_kv, d,  S_Q, S_KV, causal, dtype   (path)
    ("tc_d128_gqa",         1, 4, 2,  128, 300, 1000, False, "bf16"),  # tensor cores
    ("tc_causal",           1, 2, 2,  128, 700,  700, True,  "bf16"),
    ("tc_d64",              2, 2, 1,   64, 256,  777, False, "bf16"),
    ("simt_rows_not_4k",    1, 2, 1,  128, 130,  513, False, "bf16"),  # S_Q % 4 != 0: CUDA cores
    ("simt_d96",            1, 2, 1,   96, 100,  300, False, "bf16"),
    ("simt_f32",            1, 2, 1,   64, 128,  256, False, "f32"),
]


@pytest.mark.parametrize("case", ACCUM, ids=[c[0] for c in ACCUM])
def test_backward_accumulate_adds_to_float32(case):
    """lvx_attn_bwd_accumulate adds the gradients to float32 arrays: starting
    from nonzero arrays A and calling it twice gives A + 2 * gradient."""
    name, *shape = case
    w = _workload(*shape)
    host = inputs.make(w, tensors=("q", "k", "v", "do"))
    dev = {t: x.cuda() for t, x in host.items()}
    out, lse = lvx.attention_forward(dev["q"], dev["k"], dev["v"], w.n_blocks, w.causal)
    g = torch.Generator(device="cuda").manual_seed(3)
    start = [torch.randn(t.shape, generator=g, device="cuda") for t in (dev["q"], dev["k"], dev["v"])]
    acc = [t.clone() for t in start]
    ws = lvx.bwd_workspace(dev["q"], dev["k"], w.causal)
    for _ in range(2):
        lvx.lvx_attn_bwd_accumulate(dev["q"], dev["k"], dev["v"], out, lse, dev["do"], *acc,
                                    causal=w.causal, workspace=ws)
    lvx.lvx_last_device_error()
    torch.cuda.synchronize()
    q, k, v, do = (host[t].double().numpy() for t in ("q", "k", "v", "do"))
    refs = oracle.attention_bwd(q, k, v, do, causal=w.causal)
    for nm, a, s0, r in zip(("dQ", "dK", "dV"), acc, start, refs):
        got = (a - s0).double().cpu().numpy() / 2.0
        compare(got, r, w.dtype, f"accumulate {name}: {nm}")
