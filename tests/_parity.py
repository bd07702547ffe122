"""Shared helpers for GPU-vs-oracle parity tests.

Tolerances (from the stated bar for this path): bf16 inputs with fp32
accumulation must match the fp64 oracle within max-abs 2e-2 and mean-abs
2e-3; the fp32 configuration within max-abs 1e-4.  Because the outputs of
the long-KV workloads are small (|O| ~ 3e-3), an absolute bar alone would
pass an all-zero output, so every comparison also requires a relative RMS
error ||gpu - oracle||_2 / ||oracle||_2 below 1e-2 (bf16) or 1e-5 (fp32).
"""

from __future__ import annotations

import numpy as np
import torch

TOL = {
    "bf16": dict(max_abs=2e-2, mean_abs=2e-3, rel_rms=1e-2),
    "f32": dict(max_abs=1e-4, mean_abs=1e-5, rel_rms=1e-5),
}


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def compare(gpu, ref, dtype: str, what: str, rel_rms: float | None = None,
            mean_abs: float | None = None, max_abs: float | None = None) -> dict:
    g = to64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    fin = np.isfinite(r)
    # -inf (rows that saw no key) must match exactly
    assert np.array_equal(np.isneginf(g), np.isneginf(r)), f"{what}: -inf pattern differs"
    diff = np.abs(g[fin] - r[fin])
    stats = dict(max_abs=float(diff.max()) if diff.size else 0.0,
                 mean_abs=float(diff.mean()) if diff.size else 0.0)
    nrm = float(np.linalg.norm(r[fin]))
    stats["rel_rms"] = float(np.linalg.norm(g[fin] - r[fin]) / nrm) if nrm > 0 else 0.0
    tol = dict(TOL[dtype])
    if rel_rms is not None:
        tol["rel_rms"] = rel_rms
    if mean_abs is not None:
        tol["mean_abs"] = mean_abs
    if max_abs is not None:
        tol["max_abs"] = max_abs
    for key in ("max_abs", "mean_abs", "rel_rms"):
        assert stats[key] <= tol[key], f"{what}: {key}={stats[key]:.3e} > {tol[key]:.1e} ({stats})"
    return stats


def sample_rows(S: int, n_blocks: int, count: int = 256, seed: int = 0) -> np.ndarray:
    """First, last, block-boundary rows and a seeded random remainder."""
    bs = -(-S // n_blocks)
    must = {0, S - 1}
    for i in range(1, n_blocks):
        for r in (i * bs - 1, i * bs, i * bs + 1):
            if 0 <= r < S:
                must.add(r)
    for t in (127, 128, 255, 256):
        if t < S:
            must.add(t)
    rng = np.random.default_rng(seed)
    extra = rng.choice(S, size=min(S, max(0, count - len(must))), replace=False)
    return np.array(sorted(must | set(int(x) for x in extra)), dtype=np.int64)
