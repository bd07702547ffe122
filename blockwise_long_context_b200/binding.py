"""ctypes binding of liblvx.so (argument marshalling only).

Each ``lvx_*`` function here has the C entry point's name and meaning (see
``include/lvx.h``).  Sizes are read from tensor shapes, pointers from
``data_ptr()``, the stream from ``torch.cuda.current_stream()`` unless one is
given.  Every step of the computation runs in the library's kernels.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("LVX_LIBRARY", os.path.join(_HERE, "liblvx.so"))

LVX_FP32 = 0
LVX_BF16 = 1
STATUS = {0: "LVX_OK", 1: "LVX_ERR_INVALID_ARG", 2: "LVX_ERR_UNSUPPORTED",
          3: "LVX_ERR_WORKSPACE", 4: "LVX_ERR_CUDA", 5: "LVX_ERR_DEVICE_TIMEOUT"}


class LvxError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}")
        self.status = status


_lib = None

_c_int, _c_float, _c_size, _vp = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p

_SIGS = {
    "lvx_status_string": ([_c_int], ctypes.c_char_p),
    "lvx_version": ([], _c_int),
    "lvx_attn_fwd_workspace": ([_c_int] * 8 + [_c_int], _c_size),
    "lvx_attn_fwd": ([_vp] * 5 + [_c_int] * 8 + [_c_int, _c_float, _vp, _c_size, _vp], _c_int),
    "lvx_merge_partials": ([_vp] * 4 + [_c_int] * 5 + [_c_int, _vp], _c_int),
    "lvx_attn_fwd_partials": ([_vp] * 5 + [_c_int] * 8 + [_c_int, _c_float, _vp], _c_int),
    "lvx_attn_fwd_noalloc": ([_vp] * 5 + [_c_int] * 8 + [_c_int, _c_float, _vp], _c_int),
    "lvx_attn_bwd_workspace": ([_c_int] * 7 + [_c_int], _c_size),
    "lvx_attn_bwd": ([_vp] * 9 + [_c_int] * 7 + [_c_int, _c_float, _vp, _c_size, _vp], _c_int),
    "lvx_attn_bwd_accumulate": ([_vp] * 9 + [_c_int] * 7 + [_c_int, _c_float, _vp, _c_size, _vp],
                                _c_int),
    "lvx_kv_recompute": ([_vp] * 5 + [_c_int] * 5 + [_c_int, _vp], _c_int),
    "lvx_kv_recompute_bwd": ([_vp] * 8 + [_c_int] * 5 + [_c_int, _vp], _c_int),
    "lvx_attn_fwd_recompute_workspace": ([_c_int] * 8 + [_c_int], _c_size),
    "lvx_attn_fwd_recompute": ([_vp] * 6 + [_c_int] * 8 + [_c_int, _c_float, _vp, _c_size, _vp],
                               _c_int),
    "lvx_attn_bwd_recompute_workspace": ([_c_int] * 8 + [_c_int], _c_size),
    "lvx_attn_bwd_recompute": ([_vp] * 11 + [_c_int] * 8 + [_c_int, _c_float, _vp, _c_size, _vp],
                               _c_int),
    "lvx_last_device_error": ([_vp], _c_int),
    "lvx_selftest_wait_timeout": ([_vp], _c_int),
}


def lib() -> ctypes.CDLL:
    """Loads liblvx.so once; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m blockwise_long_context_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(status: int, where: str) -> None:
    if status != 0:
        raise LvxError(status, where)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return LVX_FP32
    if t.dtype == torch.bfloat16:
        return LVX_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors must be contiguous CUDA tensors")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def lvx_status_string(status: int) -> str:
    return lib().lvx_status_string(status).decode()


def lvx_attn_fwd_workspace(B, H, H_kv, S_Q, S_KV, d, n_blocks, causal, dtype: int) -> int:
    return lib().lvx_attn_fwd_workspace(B, H, H_kv, S_Q, S_KV, d, n_blocks, int(causal), dtype)


def lvx_attn_bwd_workspace(B, H, H_kv, S_Q, S_KV, d, causal, dtype: int) -> int:
    return lib().lvx_attn_bwd_workspace(B, H, H_kv, S_Q, S_KV, d, int(causal), dtype)


def lvx_attn_fwd(q, k, v, out, lse, n_blocks: int, causal: bool = False, scale: float = 0.0,
                 workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """q [B,S_Q,H,d], k/v [B,S_KV,H_kv,d], out like q, lse [B,H,S_Q] fp32."""
    B, S_Q, H, d = q.shape
    S_KV, H_kv = k.shape[1], k.shape[2]
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().lvx_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, H_kv, S_Q,
                              S_KV, d, n_blocks, int(causal), _dt(q), float(scale),
                              _ptr(workspace), ws, _stream(stream)), "lvx_attn_fwd")


def lvx_attn_fwd_noalloc(q, k, v, out, lse, n_blocks: int, causal: bool = False,
                         scale: float = 0.0, stream=None) -> None:
    """lvx_attn_fwd for callers that cannot allocate: the block partials live in
    the library's fixed 64 MiB device array instead of a caller workspace."""
    B, S_Q, H, d = q.shape
    S_KV, H_kv = k.shape[1], k.shape[2]
    _check(lib().lvx_attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, H_kv,
                                      S_Q, S_KV, d, n_blocks, int(causal), _dt(q), float(scale),
                                      _stream(stream)), "lvx_attn_fwd_noalloc")


def lvx_attn_fwd_partials(q, k, v, o_parts, l_parts, scale: float = 0.0, stream=None,
                          causal: bool = False) -> None:
    """q [B,S_Q,H,d], k/v [B,S_KV,H_kv,d] (a shard of the keys/values) ->
    o_parts [n,B,H,S_Q,d] fp32, l_parts [n,B,H,S_Q] fp32; n is o_parts.shape[0].
    causal: key j visible to row r iff j <= r (S_Q == S_KV)."""
    B, S_Q, H, d = q.shape
    S_KV, H_kv = k.shape[1], k.shape[2]
    n = o_parts.shape[0]
    _check(lib().lvx_attn_fwd_partials(_ptr(q), _ptr(k), _ptr(v), _ptr(o_parts), _ptr(l_parts), B, H,
                                       H_kv, S_Q, S_KV, d, n, int(bool(causal)), _dt(q), float(scale),
                                       _stream(stream)), "lvx_attn_fwd_partials")


def lvx_merge_partials(o_parts, l_parts, out, lse, stream=None) -> None:
    """o_parts [n,B,H,S_Q,d] fp32, l_parts [n,B,H,S_Q] fp32 -> out [B,S_Q,H,d], lse [B,H,S_Q]."""
    n, B, H, S_Q, d = o_parts.shape
    _check(lib().lvx_merge_partials(_ptr(o_parts), _ptr(l_parts), _ptr(out), _ptr(lse), n, B, H,
                                    S_Q, d, _dt(out), _stream(stream)), "lvx_merge_partials")


def lvx_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, causal: bool = False, scale: float = 0.0,
                 workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    B, S_Q, H, d = q.shape
    S_KV, H_kv = k.shape[1], k.shape[2]
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().lvx_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout),
                              _ptr(dq), _ptr(dk), _ptr(dv), B, H, H_kv, S_Q, S_KV, d,
                              int(causal), _dt(q), float(scale), _ptr(workspace), ws,
                              _stream(stream)), "lvx_attn_bwd")


def lvx_attn_bwd_accumulate(q, k, v, out, lse, dout, dq, dk, dv, causal: bool = False,
                            scale: float = 0.0, workspace: Optional[torch.Tensor] = None,
                            stream=None) -> None:
    """As lvx_attn_bwd, with dq, dk, dv float32 arrays the gradients are added to."""
    B, S_Q, H, d = q.shape
    S_KV, H_kv = k.shape[1], k.shape[2]
    for t in (dq, dk, dv):
        if t.dtype != torch.float32:
            raise TypeError("lvx_attn_bwd_accumulate adds into float32 gradients")
    if workspace is None:
        workspace = bwd_workspace(q, k, causal)
    ws = workspace.numel() * workspace.element_size()
    _check(lib().lvx_attn_bwd_accumulate(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                         _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), B, H, H_kv, S_Q,
                                         S_KV, d, int(causal), _dt(q), float(scale),
                                         _ptr(workspace), ws, _stream(stream)),
           "lvx_attn_bwd_accumulate")


def lvx_kv_recompute(y, w_k, w_v, k, v, H_kv: int, d: int, stream=None) -> None:
    """y [B,S_KV,d_embed], w [d_embed, H_kv*d] -> k, v [B,S_KV,H_kv,d]."""
    B, S_KV, d_embed = y.shape
    _check(lib().lvx_kv_recompute(_ptr(y), _ptr(w_k), _ptr(w_v), _ptr(k), _ptr(v), B, S_KV,
                                  d_embed, H_kv, d, _dt(y), _stream(stream)), "lvx_kv_recompute")


def lvx_kv_recompute_bwd(y, w_k, w_v, dk, dv, dy, dw_k, dw_v, stream=None) -> None:
    """y [B,S_KV,d_embed], w [d_embed,H_kv*d], dk/dv [B,S_KV,H_kv,d] ->
    dy like y, dw_k/dw_v like w (dW = y^T dK, dy = dK W_k^T + dV W_v^T)."""
    B, S_KV, d_embed = y.shape
    H_kv, d = dk.shape[2], dk.shape[3]
    _check(lib().lvx_kv_recompute_bwd(_ptr(y), _ptr(w_k), _ptr(w_v), _ptr(dk), _ptr(dv), _ptr(dy),
                                      _ptr(dw_k), _ptr(dw_v), B, S_KV, d_embed, H_kv, d, _dt(y),
                                      _stream(stream)), "lvx_kv_recompute_bwd")


def lvx_attn_fwd_recompute_workspace(B, H, H_kv, S_Q, S_KV, d, d_embed, n_blocks, dtype: int) -> int:
    return lib().lvx_attn_fwd_recompute_workspace(B, H, H_kv, S_Q, S_KV, d, d_embed, n_blocks, dtype)


def lvx_attn_bwd_recompute_workspace(B, H, H_kv, S_Q, S_KV, d, d_embed, n_blocks, dtype: int) -> int:
    return lib().lvx_attn_bwd_recompute_workspace(B, H, H_kv, S_Q, S_KV, d, d_embed, n_blocks, dtype)


def lvx_attn_fwd_recompute(q, y, w_k, w_v, out, lse, H_kv: int, n_blocks: int, scale: float = 0.0,
                           workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """q [B,S_Q,H,d], y [B,S_KV,d_embed], w [d_embed,H_kv*d] -> out like q,
    lse [B,H,S_Q] fp32, with K, V regenerated from y one key block at a time."""
    B, S_Q, H, d = q.shape
    S_KV, d_embed = y.shape[1], y.shape[2]
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().lvx_attn_fwd_recompute(_ptr(q), _ptr(y), _ptr(w_k), _ptr(w_v), _ptr(out), _ptr(lse),
                                        B, H, H_kv, S_Q, S_KV, d, d_embed, n_blocks, _dt(q),
                                        float(scale), _ptr(workspace), ws, _stream(stream)),
           "lvx_attn_fwd_recompute")


def lvx_attn_bwd_recompute(q, y, w_k, w_v, out, lse, dout, dq, dy, dw_k, dw_v, H_kv: int,
                           n_blocks: int, scale: float = 0.0,
                           workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Gradients of attention(q, y W_k, y W_v): dq like q, dy like y (bf16), dw_k,
    dw_v [d_embed, H_kv*d] float32, with K, V regenerated one key block at a time."""
    B, S_Q, H, d = q.shape
    S_KV, d_embed = y.shape[1], y.shape[2]
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().lvx_attn_bwd_recompute(_ptr(q), _ptr(y), _ptr(w_k), _ptr(w_v), _ptr(out), _ptr(lse),
                                        _ptr(dout), _ptr(dq), _ptr(dy), _ptr(dw_k), _ptr(dw_v), B, H,
                                        H_kv, S_Q, S_KV, d, d_embed, n_blocks, _dt(q), float(scale),
                                        _ptr(workspace), ws, _stream(stream)),
           "lvx_attn_bwd_recompute")


def lvx_last_device_error(stream=None) -> None:
    _check(lib().lvx_last_device_error(_stream(stream)), "lvx_last_device_error")


def lvx_selftest_wait_timeout(stream=None) -> None:
    _check(lib().lvx_selftest_wait_timeout(_stream(stream)), "lvx_selftest_wait_timeout")


# ------------------------------------------------------------------ conveniences

def fwd_workspace(q, k, n_blocks: int, causal: bool = False) -> Optional[torch.Tensor]:
    B, S_Q, H, d = q.shape
    S_KV, H_kv = k.shape[1], k.shape[2]
    nbytes = lvx_attn_fwd_workspace(B, H, H_kv, S_Q, S_KV, d, n_blocks, causal, _dt(q))
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=q.device)


def bwd_workspace(q, k, causal: bool = False) -> torch.Tensor:
    B, S_Q, H, d = q.shape
    S_KV, H_kv = k.shape[1], k.shape[2]
    nbytes = lvx_attn_bwd_workspace(B, H, H_kv, S_Q, S_KV, d, causal, _dt(q))
    return torch.empty(nbytes, dtype=torch.uint8, device=q.device)


def fwd_partials_view(workspace: torch.Tensor, n, B, H, S_Q, d):
    """(O_parts [n,B,H,S_Q,d], L_parts [n,B,H,S_Q]) views of a forward workspace."""
    o_bytes = (n * B * H * S_Q * d * 4 + 255) // 256 * 256
    O = workspace[: n * B * H * S_Q * d * 4].view(torch.float32).view(n, B, H, S_Q, d)
    L = workspace[o_bytes: o_bytes + n * B * H * S_Q * 4].view(torch.float32).view(n, B, H, S_Q)
    return O, L


def attention_forward(q, k, v, n_blocks: int, causal: bool = False, scale: float = 0.0):
    """Allocates outputs and workspace, runs lvx_attn_fwd, returns (out, lse)."""
    B, S_Q, H, d = q.shape
    out = torch.empty_like(q)
    lse = torch.empty(B, H, S_Q, dtype=torch.float32, device=q.device)
    ws = fwd_workspace(q, k, n_blocks, causal)
    lvx_attn_fwd(q, k, v, out, lse, n_blocks, causal, scale, ws)
    return out, lse


def kv_recompute_backward(y, w_k, w_v, dk, dv):
    """Allocates dy, dw_k, dw_v and runs lvx_kv_recompute_bwd; returns them."""
    dy = torch.empty_like(y); dw_k = torch.empty_like(w_k); dw_v = torch.empty_like(w_v)
    lvx_kv_recompute_bwd(y, w_k, w_v, dk, dv, dy, dw_k, dw_v)
    return dy, dw_k, dw_v


def recompute_workspaces(q, y, H_kv: int, n_blocks: int):
    """(forward, backward) workspaces of the recomputing entry points."""
    B, S_Q, H, d = q.shape
    S_KV, d_embed = y.shape[1], y.shape[2]
    f = lvx_attn_fwd_recompute_workspace(B, H, H_kv, S_Q, S_KV, d, d_embed, n_blocks, _dt(q))
    b = lvx_attn_bwd_recompute_workspace(B, H, H_kv, S_Q, S_KV, d, d_embed, n_blocks, _dt(q))
    if f == 0 or b == 0:
        raise LvxError(2, "recompute_workspaces: unsupported shape or dtype")
    return (torch.empty(f, dtype=torch.uint8, device=q.device),
            torch.empty(b, dtype=torch.uint8, device=q.device))


def attention_backward(q, k, v, out, lse, dout, causal: bool = False, scale: float = 0.0):
    dq = torch.empty_like(q); dk = torch.empty_like(k); dv = torch.empty_like(v)
    ws = bwd_workspace(q, k, causal)
    lvx_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, causal, scale, ws)
    return dq, dk, dv
