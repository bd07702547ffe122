"""B200-native blockwise attention with online-softmax merging.

The compute path is ``liblvx.so`` (C ABI, declared in ``include/lvx.h``):
hand-written sm_100a kernels for the block partials, their merge, the
backward pass and the K/V recomputation.  This package is a thin ctypes
binding with the same entry-point names; it only marshals arguments (shapes,
pointers, the current CUDA stream) and raises on error.  PyTorch supplies
device memory and streams.  There is no fallback: if the library is missing
every call raises.

``inputs`` (seeded synthetic workloads) imports without the library.
``distributed`` (LV-XAttn's exchange across ranks) and ``ring`` (Ring
Attention pass-KV) drive the same entry points over ``torch.distributed``.
"""

from __future__ import annotations

__all__ = [
    "LvxError", "lib", "lvx_attn_fwd", "lvx_attn_bwd", "lvx_attn_bwd_accumulate",
    "lvx_kv_recompute", "lvx_kv_recompute_bwd", "lvx_merge_partials", "lvx_attn_fwd_partials",
    "lvx_attn_fwd_noalloc", "lvx_attn_fwd_workspace", "lvx_attn_bwd_workspace",
    "lvx_attn_fwd_recompute", "lvx_attn_bwd_recompute", "lvx_attn_fwd_recompute_workspace",
    "lvx_attn_bwd_recompute_workspace",
    "lvx_last_device_error", "lvx_status_string", "LVX_FP32", "LVX_BF16",
]


def __getattr__(name):
    if name in __all__:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
