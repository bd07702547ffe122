"""Forward parity on the Video-MME-average shape (S_Q = 5514 text tokens,
S_KV = 15,279,944 visual tokens, Llama-3-V heads, n = 8 blocks): neither length
is a multiple of the 128-row tiles, and no KV block boundary falls on one.

* Scaled down (same S_Q, S_KV = 100,003, one KV-head group): sampled rows,
  the ragged tail among them, against the unsplit oracle.
* Full size (K + V = 62.6 GB, drawn on the device): sampled rows of the
  first KV-head group.  The oracle evaluates the unsplit definition over
  key ranges of 2^20 and combines them with its own log-sum-exp merge (pinned
  against unsplit attention on the CPU), reading K and V back range by range.
"""

import numpy as np
import pytest
import torch

import oracle
from blockwise_long_context_b200 import inputs
from blockwise_long_context_b200 import binding as lvx
from tests._parity import compare, sample_rows

pytestmark = pytest.mark.gpu

W = inputs.WORKLOADS["VMME"]


def _rows(S_Q, n, count, seed):
    rows = set(sample_rows(S_Q, n, count=count, seed=seed).tolist())
    rows |= {S_Q - 1, S_Q - 2, S_Q - 10, S_Q - 11, (S_Q // 128) * 128, (S_Q // 128) * 128 - 1}
    return np.array(sorted(r for r in rows if 0 <= r < S_Q))


def test_vmme_scaled_ragged():
    w = W.scaled(S_KV=100003, H=4, H_kv=1)
    host = inputs.make(w, tensors=("q", "k", "v"))
    d = {k: t.cuda() for k, t in host.items()}
    out, lse = lvx.attention_forward(d["q"], d["k"], d["v"], w.n_blocks)
    torch.cuda.synchronize()
    lvx.lvx_last_device_error()
    rows = _rows(w.S_Q, w.n_blocks, 192, 3)
    o_ref, l_ref = oracle.attention_fwd(*(host[n].double().numpy() for n in ("q", "k", "v")),
                                        rows=rows)
    compare(out[:, rows], o_ref, "bf16", "O (VMME scaled, sampled rows)")
    compare(lse[:, :, rows], l_ref, "bf16", "LSE (VMME scaled, sampled rows)", rel_rms=1e-4)


def test_vmme_full_size_sampled_rows():
    torch.cuda.empty_cache()
    free, total = torch.cuda.mem_get_info()
    need = 2 * W.B * W.S_KV * W.H_kv * W.d * 2 + (8 << 30)
    if free < need:
        pytest.skip(f"needs {need / 2**30:.0f} GiB free on the device, has {free / 2**30:.0f}")
    try:
        _full_size_check()
    finally:
        torch.cuda.empty_cache()


def _full_size_check():
    d = inputs.make_device(W, tensors=("q", "k", "v"))
    out, lse = lvx.attention_forward(d["q"], d["k"], d["v"], W.n_blocks)
    torch.cuda.synchronize()
    lvx.lvx_last_device_error()
    grp = W.H // W.H_kv
    heads = list(range(grp))          # the query heads of KV head 0
    rows = _rows(W.S_Q, W.n_blocks, 12, 7)
    q64 = d["q"][:, :, :grp].double().cpu().numpy()
    O_parts, L_parts = [], []
    step = 1 << 20
    for k0 in range(0, W.S_KV, step):
        k1 = min(W.S_KV, k0 + step)
        kc = d["k"][:, k0:k1, :1].double().cpu().numpy()
        vc = d["v"][:, k0:k1, :1].double().cpu().numpy()
        o, l = oracle.attention_fwd(q64, kc, vc, scale=1.0 / np.sqrt(W.d), rows=rows, heads=heads)
        O_parts.append(o)
        L_parts.append(l)
    o_ref, l_ref = oracle.merge_partials(np.stack(O_parts), np.stack(L_parts))
    compare(out[:, rows][:, :, :grp], o_ref, "bf16", "O (VMME full size, sampled rows)")
    compare(lse[:, :grp][:, :, rows], l_ref, "bf16", "LSE (VMME full size, sampled rows)",
            rel_rms=1e-4)
    assert torch.isfinite(out.float()).all()
