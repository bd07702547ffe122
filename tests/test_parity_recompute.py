"""Parity of attention with K, V regenerated from the visual features one key
block at a time (lvx_attn_fwd_recompute, lvx_attn_bwd_recompute).

The definition is the composition of the oracle's pieces: K = y W_k,
V = y W_v (fp64), exact attention and its textbook gradient, and the
gradients of the projection, dy = dK W_k^T + dV W_v^T, dW = y^T dK.
Small cases compare every element against that; the forward must also equal
the path that materialises K and V (lvx_kv_recompute + lvx_attn_fwd) bit for
bit, since the same kernels compute the same tiles.  The weight gradients are
sums over every key, so (as for lvx_kv_recompute_bwd) both sides are divided
by the oracle's RMS before the bf16 bar is applied; dy and dW here pass through
one more bf16 rounding than lvx_kv_recompute_bwd's outputs (dK, dV enter the
projection GEMMs as bf16), so their normalised bars are twice the attention
bars, max-abs 4e-2 and mean-abs 4e-3 (two roundings of relative size up to
2^-9 instead of one), with the relative RMS bar of 1e-2 unchanged.  At the full visual-
feature workload (y [65536, 4096], W [4096, 1024], S_Q = 2048) dQ is compared
on sampled query rows and dy on sampled key rows; the full dW needs every
key's gradient, so there it is compared with the materialising path.
"""

import numpy as np
import pytest
import torch

import oracle
from blockwise_long_context_b200 import binding as lvx
from blockwise_long_context_b200 import inputs
from tests._parity import compare, sample_rows

pytestmark = pytest.mark.gpu

CASES = [
    # name,              B, H, H_kv, d,  S_Q, S_KV, E,   n
    ("gqa_ragged",        1, 4, 2,  128, 256, 1000, 512, 3),
    ("two_batches_simt",  2, 2, 2,  128, 130,  700, 256, 2),   # S_Q % 4 != 0: CUDA-core backward
    ("d64_empty_block",   1, 4, 4,   64, 200,    9, 256, 4),   # blocks 3, 3, 3, 0 keys
]


def _workload(B, H, H_kv, d, S_Q, S_KV, E, n):
    return inputs.WORKLOADS["C2"].scaled(B=B, H=H, H_kv=H_kv, d=d, S_Q=S_Q, S_KV=S_KV, d_embed=E,
                                         n_blocks=n)


def _gpu(w, host):
    dev = {t: x.cuda() for t, x in host.items()}
    fws, bws = lvx.recompute_workspaces(dev["q"], dev["y"], w.H_kv, w.n_blocks)
    out = torch.full_like(dev["q"], float("nan"))
    lse = torch.full((w.B, w.H, w.S_Q), float("nan"), dtype=torch.float32, device="cuda")
    lvx.lvx_attn_fwd_recompute(dev["q"], dev["y"], dev["w_k"], dev["w_v"], out, lse, w.H_kv,
                               w.n_blocks, workspace=fws)
    dq = torch.full_like(dev["q"], float("nan"))
    dy = torch.full_like(dev["y"], float("nan"))
    dwk = torch.full(dev["w_k"].shape, float("nan"), dtype=torch.float32, device="cuda")
    dwv = torch.full_like(dwk, float("nan"))
    lvx.lvx_attn_bwd_recompute(dev["q"], dev["y"], dev["w_k"], dev["w_v"], out, lse, dev["do"],
                               dq, dy, dwk, dwv, w.H_kv, w.n_blocks, workspace=bws)
    lvx.lvx_last_device_error()
    torch.cuda.synchronize()
    return dev, out, lse, dq, dy, dwk, dwv


def _materialised(w, dev):
    """The same step with K, V (and dK, dV) materialised whole."""
    k = torch.empty(w.B, w.S_KV, w.H_kv, w.d, dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    lvx.lvx_kv_recompute(dev["y"], dev["w_k"], dev["w_v"], k, v, w.H_kv, w.d)
    out, lse = lvx.attention_forward(dev["q"], k, v, w.n_blocks)
    dq, dk, dv = lvx.attention_backward(dev["q"], k, v, out, lse, dev["do"])
    dy, dwk, dwv = lvx.kv_recompute_backward(dev["y"], dev["w_k"], dev["w_v"], dk, dv)
    torch.cuda.synchronize()
    return out, lse, dq, dy, dwk, dwv


def _rms_compare(got, ref, what):
    s = float(np.sqrt(np.mean(ref * ref)))
    compare(got / s, ref / s, "bf16", what, mean_abs=4e-3, max_abs=4e-2)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_recompute_matches_oracle_and_materialised_path(case):
    name, *shape = case
    w = _workload(*shape)
    host = inputs.make(w, tensors=("q", "do", "y", "w_k", "w_v"))
    dev, out, lse, dq, dy, dwk, dwv = _gpu(w, host)
    m_out, m_lse, m_dq, m_dy, m_dwk, m_dwv = _materialised(w, dev)
    # the forward runs the same kernels on the same tiles as the materialising path
    assert torch.equal(out, m_out), f"{name}: out differs from the materialising path"
    assert torch.equal(lse, m_lse), f"{name}: lse differs from the materialising path"
    # the definition, in fp64 from the inputs
    y, wk, wv, q, do = (host[t].double().numpy() for t in ("y", "w_k", "w_v", "q", "do"))
    K, V = oracle.kv_recompute(y, wk, wv)
    K = K.reshape(w.B, w.S_KV, w.H_kv, w.d)
    V = V.reshape(w.B, w.S_KV, w.H_kv, w.d)
    o_r, l_r = oracle.attention_fwd(q, K, V)
    compare(out, o_r, "bf16", f"{name}: O")
    # K, V reach the attention as bf16 GEMM outputs (one rounding, ~1e-3 on a
    # logit here) where the attention tests feed exact inputs: the LSE's
    # relative bar is 1e-3 instead of 1e-4, the bf16 absolute bars unchanged
    compare(lse, l_r, "bf16", f"{name}: LSE", rel_rms=1e-3)
    dq_r, dk_r, dv_r = oracle.attention_bwd(q, K, V, do)
    dy_r, dwk_r, dwv_r = oracle.kv_recompute_bwd(y, wk, wv, dk_r.reshape(w.B, w.S_KV, -1),
                                                 dv_r.reshape(w.B, w.S_KV, -1))
    compare(dq, dq_r, "bf16", f"{name}: dQ")
    _rms_compare(dy.double().cpu().numpy(), dy_r, f"{name}: dy")
    _rms_compare(dwk.double().cpu().numpy(), dwk_r, f"{name}: dW_k")
    _rms_compare(dwv.double().cpu().numpy(), dwv_r, f"{name}: dW_v")
    # a second call overwrites the weight gradients (they start from zero every call)
    _, _, _, dq2, dy2, dwk2, dwv2 = _gpu(w, host)
    _rms_compare(dwk2.double().cpu().numpy(), dwk_r, f"{name}: dW_k, second call")
    _rms_compare(dwv2.double().cpu().numpy(), dwv_r, f"{name}: dW_v, second call")


def test_recompute_full_size_sampled():
    """The full Llama-3-V-like visual-feature workload: dQ on 256 sampled query
    rows of every head, dy on 256 sampled key rows (first, last and block-edge
    rows included), against the oracle on K, V = y W in fp64; dW_k, dW_v (every
    key's gradient summed) against the materialising path."""
    w = inputs.WORKLOADS["C2"]
    host = inputs.make(w, tensors=("q", "do", "y", "w_k", "w_v"))
    dev, out, lse, dq, dy, dwk, dwv = _gpu(w, host)
    for t in (dq, dy, dwk, dwv):
        assert torch.isfinite(t.float()).all()
    y = host["y"].double().numpy()
    wk, wv = host["w_k"].double().numpy(), host["w_v"].double().numpy()
    q, do = host["q"].double().numpy(), host["do"].double().numpy()
    K, V = oracle.kv_recompute(y, wk, wv)
    K = K.reshape(w.B, w.S_KV, w.H_kv, w.d)
    V = V.reshape(w.B, w.S_KV, w.H_kv, w.d)
    rows = sample_rows(w.S_Q, w.n_blocks, count=256)
    dq_r = oracle.attention_bwd_rows(q, K, V, do, rows)
    compare(dq[:, rows], dq_r, "bf16", "full size: dQ (sampled rows)")
    keys = sample_rows(w.S_KV, w.n_blocks, count=256, seed=2)
    dk_r, dv_r = oracle.attention_bwd_keys(q, K, V, do, keys, list(range(w.H_kv)), batches=[0])
    dy_r, _, _ = oracle.kv_recompute_bwd(y[0, keys], wk, wv, dk_r[0].reshape(len(keys), -1),
                                         dv_r[0].reshape(len(keys), -1))
    _rms_compare(dy[0, keys].double().cpu().numpy(), dy_r, "full size: dy (sampled key rows)")
    m_out, m_lse, m_dq, m_dy, m_dwk, m_dwv = _materialised(w, dev)
    assert torch.equal(out, m_out) and torch.equal(lse, m_lse)
    ref_k, ref_v = m_dwk.double().cpu().numpy(), m_dwv.double().cpu().numpy()
    _rms_compare(dwk.double().cpu().numpy(), ref_k, "full size: dW_k vs materialising path")
    _rms_compare(dwv.double().cpu().numpy(), ref_v, "full size: dW_v vs materialising path")
