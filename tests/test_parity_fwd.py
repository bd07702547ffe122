"""Forward parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small cases are compared element by element (outputs, log-sum-exp and every
block partial O_i, L_i read from the documented workspace layout); they span
several 128-row/128-key tiles, ragged tails, empty blocks and single-key
blocks.  The full-size workloads are compared on sampled query rows (all
heads), which the oracle evaluates row by row with the plain definition.
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
    # name,            B, H, H_kv, d,  S_Q,  S_KV, n, causal, dtype
    ("c0_full",          1, 1, 1,   64, 128,  1024, 4, False, "f32"),
    ("bf16_d128_ragged", 2, 4, 2,  128, 300,  1000, 3, False, "bf16"),
    ("bf16_d64_ragged",  1, 4, 1,   64, 257,   777, 5, False, "bf16"),
    ("bf16_n1",          1, 2, 2,  128, 130,   513, 1, False, "bf16"),
    ("bf16_gqa8",        1, 8, 1,  128, 384,  2048, 2, False, "bf16"),
    ("bf16_causal",      1, 2, 2,  128, 700,   700, 3, True,  "bf16"),
    ("bf16_causal_d64",  2, 2, 1,   64, 513,   513, 4, True,  "bf16"),
    ("bf16_causal_n1",   1, 2, 1,   64, 300,   300, 1, True,  "bf16"),
    ("bf16_keyblocks",   1, 2, 1,  128,  64,    37, 37, False, "bf16"),
    ("bf16_empty_block", 1, 1, 1,  128, 200,     5, 4, False, "bf16"),
    ("bf16_one_by_one",  1, 1, 1,  128,   1,     1, 1, False, "bf16"),
    ("bf16_d96_simt",    1, 2, 1,   96, 100,   300, 2, False, "bf16"),
    ("f32_ragged_d40",   1, 3, 1,   40,  50,    99, 4, False, "f32"),
    ("f32_causal",       1, 2, 2,   64, 100,   100, 3, True,  "f32"),
]


def _workload(B, H, H_kv, d, S_Q, S_KV, n, causal, dtype):
    base = inputs.WORKLOADS["C0" if dtype == "f32" else "C1"]
    return base.scaled(B=B, H=H, H_kv=H_kv, d=d, S_Q=S_Q, S_KV=S_KV, n_blocks=n, causal=causal,
                       dtype=dtype)


def _run(w, host):
    dev = {k: t.cuda() for k, t in host.items()}
    out = torch.empty_like(dev["q"])
    lse = torch.empty(w.B, w.H, w.S_Q, dtype=torch.float32, device="cuda")
    ws = lvx.fwd_workspace(dev["q"], dev["k"], w.n_blocks, w.causal)
    lvx.lvx_attn_fwd(dev["q"], dev["k"], dev["v"], out, lse, w.n_blocks, w.causal, 0.0, ws)
    lvx.lvx_last_device_error()
    torch.cuda.synchronize()
    return out, lse, ws


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_forward_small(case):
    name, *shape = case
    w = _workload(*shape)
    host = inputs.make(w)
    out, lse, ws = _run(w, host)
    q, k, v = (host[t].double().numpy() for t in ("q", "k", "v"))
    o_ref, l_ref = oracle.attention_fwd(q, k, v, causal=w.causal)
    compare(out, o_ref, w.dtype, f"{name}: O")
    compare(lse, l_ref, w.dtype, f"{name}: LSE", rel_rms=1e-4 if w.dtype == "bf16" else 1e-6)
    if w.n_blocks > 1:
        O_p, L_p = lvx.fwd_partials_view(ws, w.n_blocks, w.B, w.H, w.S_Q, w.d)
        O_r, L_r = oracle.block_partials(q, k, v, w.n_blocks, causal=w.causal)
        # oracle partials are [n, B, R, H, d]; the workspace holds [n, B, H, S_Q, d]
        O_r = np.transpose(O_r, (0, 1, 3, 2, 4))
        O_g, L_g = O_p.cpu().double().numpy(), L_p.cpu().double().numpy()
        if w.causal:
            bs = -(-w.S_KV // w.n_blocks)
            valid = np.array([[j <= r // bs for r in range(w.S_Q)] for j in range(w.n_blocks)])
            mask_o = np.broadcast_to(valid[:, None, None, :, None], O_g.shape)
            mask_l = np.broadcast_to(valid[:, None, None, :], L_g.shape)
            O_g = np.where(mask_o, O_g, 0.0); O_r = np.where(mask_o, O_r, 0.0)
            L_g = np.where(mask_l, L_g, 0.0); L_r = np.where(mask_l, L_r, 0.0)
        # partials are fp32: they carry no output rounding
        compare(O_g, O_r, w.dtype, f"{name}: O_i", rel_rms=5e-3 if w.dtype == "bf16" else None)
        compare(L_g, L_r, w.dtype, f"{name}: L_i", rel_rms=1e-4 if w.dtype == "bf16" else 1e-6)


def test_forward_rising_logits_rescale():
    """Logits that step up from tile to tile inside each key block, so that the
    running maximum of a row moves after its first tile.  Query head 0 steps by
    ~12 (log2 units) per 128-key tile: past the rescale threshold of 8, every
    later tile rescales O.  Head 1 steps by ~6: no exponential exceeds 2^8,
    but a tile's sum of exponentials does.  Key 262 adds a spike far above the
    rest (argument > 128 in log2 units for head 0); it sits at a position whose
    exponential the kernel computes with the FMA-pipe polynomial in the steady
    state.  All three must match plain attention."""
    rng = np.random.default_rng(11)
    B, H, H_kv, d, S_Q, S_KV, n = 1, 2, 1, 128, 130, 1000, 2
    q = rng.standard_normal((B, S_Q, H, d)) * 0.5
    k = rng.standard_normal((B, S_KV, H_kv, d)) * 0.5
    v = rng.standard_normal((B, S_KV, H_kv, d))
    q[:, :, 0, 0] = 16.0
    q[:, :, 1, 0] = 8.0
    block = -(-S_KV // n)
    k[0, :, 0, 0] = 6.0 * ((np.arange(S_KV) % block) // 128)
    k[0, 262, 0, 0] = 80.0
    host = {name: torch.from_numpy(t).to(torch.bfloat16) for name, t in (("q", q), ("k", k), ("v", v))}
    w = _workload(B, H, H_kv, d, S_Q, S_KV, n, False, "bf16")
    out, lse, ws = _run(w, host)
    q, k, v = (host[t].double().numpy() for t in ("q", "k", "v"))
    o_ref, l_ref = oracle.attention_fwd(q, k, v)
    compare(out, o_ref, "bf16", "rising logits: O")
    compare(lse, l_ref, "bf16", "rising logits: LSE", rel_rms=1e-4)
    O_p, L_p = lvx.fwd_partials_view(ws, n, B, H, S_Q, d)
    O_r, L_r = oracle.block_partials(q, k, v, n)
    compare(O_p, np.transpose(O_r, (0, 1, 3, 2, 4)), "bf16", "rising logits: O_i", rel_rms=5e-3)
    compare(L_p, L_r, "bf16", "rising logits: L_i", rel_rms=1e-4)


def test_merge_entry_point_matches_oracle():
    rng = np.random.default_rng(3)
    n, B, H, S_Q, d = 5, 2, 3, 77, 128
    O = rng.standard_normal((n, B, H, S_Q, d)).astype(np.float32)
    L = (rng.standard_normal((n, B, H, S_Q)) * 3).astype(np.float32)
    L[1, 0, 0, :10] = -np.inf            # empty partials are the identity
    L[:, 1, 2, 5] = -np.inf              # a row that saw nothing
    out = torch.empty(B, S_Q, H, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, H, S_Q, dtype=torch.float32, device="cuda")
    lvx.lvx_merge_partials(torch.from_numpy(O).cuda(), torch.from_numpy(L).cuda(), out, lse)
    O_r, L_r = oracle.merge_partials(np.transpose(O, (0, 1, 3, 2, 4)), L)
    compare(out, O_r, "bf16", "merge O", rel_rms=5e-3)
    compare(lse, L_r, "f32", "merge L", rel_rms=1e-6)
    assert float(out[1, 5, 2].abs().max()) == 0.0


@pytest.mark.parametrize("cfg", ["C1", "C4", "C3"])
def test_forward_full_size_sampled_rows(cfg):
    w = inputs.WORKLOADS[cfg]
    host = inputs.make(w)
    out, lse, _ = _run(w, host)
    rows = sample_rows(w.S_Q, w.n_blocks, count=256)
    q, k, v = (host[t].double().numpy() for t in ("q", "k", "v"))
    o_ref, l_ref = oracle.attention_fwd(q, k, v, causal=w.causal, rows=rows)
    compare(out[:, rows], o_ref, "bf16", f"{cfg}: O (sampled rows)")
    compare(lse[:, :, rows], l_ref, "bf16", f"{cfg}: LSE (sampled rows)", rel_rms=1e-4)
    # properties over all rows: finite, and |O| bounded by max |V| of the group
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    assert float(out.float().abs().max()) <= float(host["v"].float().abs().max()) + 1e-2
