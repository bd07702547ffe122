"""CPU-side checks of the C ABI: the library loads, exports every entry point
that include/lvx.h declares, and rejects invalid arguments synchronously
without launching anything (no GPU needed: every case returns before the
first CUDA call)."""

import os
import re
import subprocess

import pytest

from blockwise_long_context_b200 import binding as lvx

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lvx.h")
INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3


def _declared():
    with open(HEADER) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lvx_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert {"lvx_attn_fwd", "lvx_attn_bwd", "lvx_kv_recompute", "lvx_kv_recompute_bwd"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", lvx.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (lvx_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    L = lvx.lib()
    for n in names:
        assert hasattr(L, n)


def test_status_strings_and_version():
    assert lvx.lvx_status_string(0) == "LVX_OK"
    assert lvx.lvx_status_string(5) == "LVX_ERR_DEVICE_TIMEOUT"
    assert lvx.lib().lvx_version() >= 100


def test_workspace_sizes():
    # O parts [n,B,H,S_Q,d] fp32 + L parts [n,B,H,S_Q] fp32, each 256-byte aligned
    ws = lvx.lvx_attn_fwd_workspace(1, 32, 8, 2048, 65536, 128, 8, 0, lvx.LVX_BF16)
    assert ws == 8 * 32 * 2048 * 128 * 4 + 8 * 32 * 2048 * 4
    assert lvx.lvx_attn_fwd_workspace(1, 32, 8, 2048, 65536, 128, 1, 0, lvx.LVX_BF16) == 0
    assert lvx.lvx_attn_fwd_workspace(1, 3, 2, 10, 10, 64, 2, 0, lvx.LVX_BF16) == 0   # H % H_kv
    bw = lvx.lvx_attn_bwd_workspace(1, 2, 1, 100, 300, 64, 0, lvx.LVX_BF16)
    assert bw == 2 * 1024 + 100 * 2 * 64 * 4   # D and LSE*log2(e), 256-byte aligned, then dQ_acc


P16 = 16   # a non-null, 16-byte-aligned address; never dereferenced on these paths


def _fwd(**kw):
    a = dict(q=P16, k=P16, v=P16, out=P16, lse=P16, B=1, H=2, H_kv=1, S_Q=4, S_KV=4, d=64,
             n=1, causal=0, dt=lvx.LVX_BF16, scale=0.0, ws=None, ws_bytes=0)
    a.update(kw)
    return lvx.lib().lvx_attn_fwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["H"],
                                  a["H_kv"], a["S_Q"], a["S_KV"], a["d"], a["n"], a["causal"],
                                  a["dt"], a["scale"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), INVALID), (dict(lse=None), INVALID), (dict(k=24), INVALID),
    (dict(B=0), INVALID), (dict(S_KV=0), INVALID), (dict(H=3, H_kv=2), INVALID),
    (dict(n=5), INVALID), (dict(n=0), INVALID),
    (dict(d=136), UNSUPPORTED), (dict(d=60), UNSUPPORTED), (dict(dt=7), UNSUPPORTED),
    (dict(causal=1, S_Q=3), UNSUPPORTED),
    (dict(n=2), INVALID),                       # workspace needed but NULL
    (dict(n=2, ws=P16, ws_bytes=64), WORKSPACE),
    (dict(scale=float("nan")), INVALID),
])
def test_fwd_rejects_invalid_arguments(kw, code):
    assert _fwd(**kw) == code


def test_bwd_and_kv_reject_invalid_arguments():
    L = lvx.lib()
    args = [P16] * 9 + [1, 2, 1, 4, 4, 64, 0, lvx.LVX_BF16, 0.0, P16, 0, None]
    assert L.lvx_attn_bwd(*args) == WORKSPACE
    bad = list(args); bad[0] = None
    assert L.lvx_attn_bwd(*bad) == INVALID
    bad = list(args); bad[14] = 256
    assert L.lvx_attn_bwd(*bad) == UNSUPPORTED
    # the accumulating form validates the same way
    assert L.lvx_attn_bwd_accumulate(*args) == WORKSPACE
    bad = list(args); bad[6] = None                        # dq
    assert L.lvx_attn_bwd_accumulate(*bad) == INVALID
    bad = list(args); bad[8] = 24                          # dv misaligned
    assert L.lvx_attn_bwd_accumulate(*bad) == INVALID
    bad = list(args); bad[15] = 1; bad[12] = 8             # causal with S_Q != S_KV
    assert L.lvx_attn_bwd_accumulate(*bad) == UNSUPPORTED
    assert L.lvx_kv_recompute(P16, P16, None, P16, P16, 1, 4, 64, 1, 64, lvx.LVX_BF16, None) == INVALID
    assert L.lvx_kv_recompute(P16, P16, P16, P16, P16, 1, 0, 64, 1, 64, lvx.LVX_BF16, None) == INVALID
    assert L.lvx_kv_recompute(P16, P16, P16, P16, P16, 1, 4, 64, 1, 64, 9, None) == UNSUPPORTED
    kvb = [P16] * 8 + [1, 4, 256, 1, 256, lvx.LVX_BF16, None]
    for i in range(8):   # every pointer is checked
        bad = list(kvb); bad[i] = None
        assert L.lvx_kv_recompute_bwd(*bad) == INVALID
    bad = list(kvb); bad[5] = P16 + 8   # misaligned output
    assert L.lvx_kv_recompute_bwd(*bad) == INVALID
    for i in range(8, 13):
        bad = list(kvb); bad[i] = 0
        assert L.lvx_kv_recompute_bwd(*bad) == INVALID
    bad = list(kvb); bad[13] = 9
    assert L.lvx_kv_recompute_bwd(*bad) == UNSUPPORTED
    bad = list(kvb); bad[8] = 1 << 16; bad[9] = 1 << 16   # B*S_KV >= 2^31
    assert L.lvx_kv_recompute_bwd(*bad) == UNSUPPORTED
    assert L.lvx_merge_partials(P16, P16, P16, None, 2, 1, 1, 4, 64, lvx.LVX_BF16, None) == INVALID
    assert L.lvx_merge_partials(P16, P16, P16, P16, 2, 1, 1, 4, 12, lvx.LVX_BF16, None) == UNSUPPORTED


def _parts(**kw):
    a = dict(q=P16, k=P16, v=P16, O=P16, L=P16, B=1, H=2, H_kv=1, S_Q=4, S_KV=4, d=64, n=1,
             causal=0, dt=lvx.LVX_BF16, scale=0.0)
    a.update(kw)
    return lvx.lib().lvx_attn_fwd_partials(a["q"], a["k"], a["v"], a["O"], a["L"], a["B"], a["H"],
                                           a["H_kv"], a["S_Q"], a["S_KV"], a["d"], a["n"],
                                           a["causal"], a["dt"], a["scale"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(O=None), INVALID), (dict(L=None), INVALID), (dict(v=None), INVALID),
    (dict(O=24), INVALID), (dict(n=0), INVALID), (dict(n=5), INVALID),
    (dict(H=3, H_kv=2), INVALID), (dict(d=136), UNSUPPORTED), (dict(dt=7), UNSUPPORTED),
    (dict(scale=float("nan")), INVALID), (dict(causal=1, S_KV=8), UNSUPPORTED),
])
def test_fwd_partials_rejects_invalid_arguments(kw, code):
    assert _parts(**kw) == code


def test_recompute_entry_points_validate_before_launching():
    """The key-block-at-a-time recomputation: workspace sizes and argument
    checks, all on the host (no GPU needed)."""
    L = lvx.lib()
    bf16 = lvx.LVX_BF16
    # B, H, H_kv, S_Q, S_KV, d, d_embed, n
    shape = (1, 32, 8, 2048, 65536, 128, 4096, 8)
    block_kv = 8192 * 8 * 128 * 2
    fwd = L.lvx_attn_fwd_recompute_workspace(*shape, bf16)
    assert fwd == L.lvx_attn_fwd_workspace(1, 32, 8, 2048, 65536, 128, 8, 0, bf16) + 2 * block_kv
    bwd = L.lvx_attn_bwd_recompute_workspace(*shape, bf16)
    assert bwd == L.lvx_attn_bwd_workspace(1, 32, 8, 2048, 65536, 128, 0, bf16) + 4 * block_kv
    # unsupported: fp32, d_embed not a multiple of 256, H_kv*d not a multiple of 256
    assert L.lvx_attn_fwd_recompute_workspace(*shape, lvx.LVX_FP32) == 0
    assert L.lvx_attn_bwd_recompute_workspace(1, 32, 8, 2048, 65536, 128, 4000, 8, bf16) == 0
    assert L.lvx_attn_bwd_recompute_workspace(1, 4, 1, 64, 512, 128, 512, 2, bf16) == 0
    P = 16
    st = L.lvx_attn_fwd_recompute(P, P, P, P, P, P, *shape, bf16, 0.0, P, fwd - 1, None)
    assert st == 3   # LVX_ERR_WORKSPACE
    st = L.lvx_attn_fwd_recompute(None, P, P, P, P, P, *shape, bf16, 0.0, P, fwd, None)
    assert st == 1   # LVX_ERR_INVALID_ARG
    st = L.lvx_attn_bwd_recompute(P, P, P, P, P, P, P, P, P, P, P, *shape, lvx.LVX_FP32, 0.0, P,
                                  bwd, None)
    assert st == 2   # LVX_ERR_UNSUPPORTED
    st = L.lvx_attn_bwd_recompute(P, P, P, P, P, P, P, P, P, 8, P, *shape, bf16, 0.0, P, bwd, None)
    assert st == 1   # misaligned dw_k
