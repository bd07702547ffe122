"""Guard bands around every buffer the library writes.

compute-sanitizer is not available for these kernels, so out-of-range writes
are looked for directly: each output, workspace and partials array is placed
inside a larger device allocation whose 4 KiB bands before and after it hold
a fixed byte pattern, every entry point runs on ragged shapes (sequence
lengths that are not multiples of the 128-row tiles, GQA, causal, both head
widths, the tensor-core and CUDA-core paths), and the bands must come back
unchanged.  The parity tests check the values inside; this checks that
nothing lands outside.
"""

import math

import pytest
import torch

from blockwise_long_context_b200 import binding as lvx
from blockwise_long_context_b200 import inputs

pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5


class Guarded:
    """A tensor view with pattern-filled bands on both sides."""

    def __init__(self, shape, dtype):
        nbytes = math.prod(shape) * torch.tensor([], dtype=dtype).element_size()
        body = (nbytes + 15) // 16 * 16
        self.buf = torch.full((2 * GUARD + body,), PATTERN, dtype=torch.uint8, device="cuda")
        self.lo, self.hi = GUARD, GUARD + nbytes
        self.t = self.buf[self.lo:self.hi].view(dtype).view(shape)

    def intact(self) -> bool:
        b = self.buf
        return bool((b[:self.lo] == PATTERN).all()) and bool((b[self.hi:] == PATTERN).all())


def _check(name, *gs):
    torch.cuda.synchronize()
    lvx.lvx_last_device_error()
    bad = [i for i, g in enumerate(gs) if not g.intact()]
    assert not bad, f"{name}: write outside buffer(s) {bad}"


FWD = [
    # name,              B, H, H_kv, d,  S_Q,  S_KV, n, causal, dtype
    ("bf16_d128_ragged",  2, 4, 2,  128, 300,  1000, 3, False, "bf16"),
    ("bf16_d64_ragged",   1, 4, 1,   64, 257,   777, 5, False, "bf16"),
    ("bf16_causal",       1, 2, 2,  128, 700,   700, 3, True,  "bf16"),
    ("bf16_d96_simt",     1, 2, 1,   96, 100,   300, 2, False, "bf16"),
    ("f32_ragged_d40",    1, 3, 1,   40,  50,    99, 4, False, "f32"),
]


def _host(B, H, H_kv, d, S_Q, S_KV, n, causal, dtype, backward=False):
    base = inputs.WORKLOADS["C0" if dtype == "f32" else "C2"]
    w = base.scaled(B=B, H=H, H_kv=H_kv, d=d, S_Q=S_Q, S_KV=S_KV, n_blocks=n, causal=causal,
                    dtype=dtype, backward=backward, d_embed=0)
    names = ("q", "k", "v", "do") if backward else ("q", "k", "v")
    return w, {t: x.cuda() for t, x in inputs.make(w, tensors=names).items()}


@pytest.mark.parametrize("case", FWD, ids=[c[0] for c in FWD])
def test_forward_and_merge_write_only_their_buffers(case):
    name, *shape = case
    w, d = _host(*shape)
    B, S_Q, H, hd = d["q"].shape
    dt = lvx._dt(d["q"])
    out = Guarded(d["q"].shape, d["q"].dtype)
    lse = Guarded((B, H, S_Q), torch.float32)
    nbytes = lvx.lvx_attn_fwd_workspace(B, H, w.H_kv, S_Q, w.S_KV, hd, w.n_blocks, w.causal, dt)
    ws = Guarded((max(nbytes, 16),), torch.uint8)
    lvx.lvx_attn_fwd(d["q"], d["k"], d["v"], out.t, lse.t, w.n_blocks, w.causal, 0.0,
                     ws.t if nbytes else None)
    _check(f"{name}: lvx_attn_fwd", out, lse, ws)
    out2 = Guarded(d["q"].shape, d["q"].dtype)
    lse2 = Guarded((B, H, S_Q), torch.float32)
    lvx.lvx_attn_fwd_noalloc(d["q"], d["k"], d["v"], out2.t, lse2.t, w.n_blocks, w.causal)
    _check(f"{name}: lvx_attn_fwd_noalloc", out2, lse2)
    if not w.causal:
        n = w.n_blocks
        O = Guarded((n, B, H, S_Q, hd), torch.float32)
        L = Guarded((n, B, H, S_Q), torch.float32)
        lvx.lvx_attn_fwd_partials(d["q"], d["k"], d["v"], O.t, L.t)
        _check(f"{name}: lvx_attn_fwd_partials", O, L)
        out3 = Guarded(d["q"].shape, d["q"].dtype)
        lse3 = Guarded((B, H, S_Q), torch.float32)
        lvx.lvx_merge_partials(O.t, L.t, out3.t, lse3.t)
        _check(f"{name}: lvx_merge_partials", out3, lse3)


BWD = [
    # name,              B, H, H_kv, d,  S_Q, S_KV, causal, dtype
    ("bf16_d128_gqa",     1, 4, 2,  128, 300, 1000, False, "bf16"),
    ("bf16_d64",          2, 2, 2,   64, 256,  777, False, "bf16"),
    ("bf16_causal",       1, 2, 2,  128, 700,  700, True,  "bf16"),
    ("bf16_rows_not_4k",  1, 2, 1,  128, 130,  513, False, "bf16"),
    ("f32_small",         1, 2, 1,   64, 128,  256, False, "f32"),
]


@pytest.mark.parametrize("case", BWD, ids=[c[0] for c in BWD])
def test_backward_writes_only_its_buffers(case):
    name, B, H, H_kv, hd, S_Q, S_KV, causal, dtype = case
    w, d = _host(B, H, H_kv, hd, S_Q, S_KV, 1, causal, dtype, backward=True)
    out, lse = lvx.attention_forward(d["q"], d["k"], d["v"], 1, causal)
    dt = lvx._dt(d["q"])
    nbytes = lvx.lvx_attn_bwd_workspace(B, H, H_kv, S_Q, S_KV, hd, causal, dt)
    for accumulate in (False, True):
        gdt = torch.float32 if accumulate else d["q"].dtype
        dq = Guarded(d["q"].shape, gdt)
        dk = Guarded(d["k"].shape, gdt)
        dv = Guarded(d["v"].shape, gdt)
        ws = Guarded((nbytes,), torch.uint8)
        if accumulate:
            for g in (dq, dk, dv):
                g.t.zero_()
            lvx.lvx_attn_bwd_accumulate(d["q"], d["k"], d["v"], out, lse, d["do"], dq.t, dk.t,
                                        dv.t, causal=causal, workspace=ws.t)
        else:
            lvx.lvx_attn_bwd(d["q"], d["k"], d["v"], out, lse, d["do"], dq.t, dk.t, dv.t,
                             causal, 0.0, ws.t)
        _check(f"{name}: backward (accumulate={accumulate})", dq, dk, dv, ws)


@pytest.mark.parametrize("S_KV,d_embed", [(1000, 256), (300, 128)])
def test_kv_recompute_and_its_gradients_write_only_their_buffers(S_KV, d_embed):
    w = inputs.WORKLOADS["C2"].scaled(S_KV=S_KV, d_embed=d_embed, H_kv=2)
    h = {t: x.cuda() for t, x in inputs.make(w, tensors=("y", "w_k", "w_v")).items()}
    shape = (w.B, S_KV, w.H_kv, w.d)
    k, v = Guarded(shape, torch.bfloat16), Guarded(shape, torch.bfloat16)
    lvx.lvx_kv_recompute(h["y"], h["w_k"], h["w_v"], k.t, v.t, w.H_kv, w.d)
    _check("lvx_kv_recompute", k, v)
    dy = Guarded(h["y"].shape, torch.bfloat16)
    dwk, dwv = Guarded(h["w_k"].shape, torch.bfloat16), Guarded(h["w_v"].shape, torch.bfloat16)
    lvx.lvx_kv_recompute_bwd(h["y"], h["w_k"], h["w_v"], k.t, v.t, dy.t, dwk.t, dwv.t)
    _check("lvx_kv_recompute_bwd", dy, dwk, dwv)
