"""Plain fp64 definitions of what the blockwise attention path computes.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Slow and obviously
correct: every function is the textbook definition written out with numpy
fp64 arithmetic; the only library primitives used are matmul, exp, log, max
and sum.  There is no tiling, no online softmax, no fusion.

Layouts (all numpy arrays, converted to float64 on entry):
  q, o, dq, do : [B, S_Q,  H,    d]
  k, v, dk, dv : [B, S_KV, H_kv, d]
  lse          : [B, H, S_Q]   natural-log log-sum-exp of the scaled logits

Readings of the pages that this file fixes (where the pages are silent or ambiguous):
  * scale s = 1/sqrt(d), d the per-head width, unless given;
  * query head h reads key/value head floor(h / (H / H_kv)) (contiguous
    groups, the repeat-interleave convention for grouped-query attention);
  * causal masking is for self-attention only: key j is visible to query r
    iff j <= r;
  * key/value block i of n holds keys [i*ceil(S_KV/n), min((i+1)*ceil(S_KV/n), S_KV));
  * an empty (or fully masked) block has the partial (O_i, L_i) = (0, -inf),
    the identity of the merge; Algorithm 1's "O_i, L_i <- 0" is read as this
    empty result because L_i is a log-sum-exp;
  * L_i is stored in natural log; O_i is stored normalised (divided by its
    own softmax denominator).
"""

from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence

import numpy as np


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _default_scale(d: int, scale: Optional[float]) -> float:
    return 1.0 / math.sqrt(d) if scale is None or scale <= 0 else float(scale)


def _kv_head(h: int, H: int, H_kv: int) -> int:
    """Grouped-query head mapping: query head h reads KV head h // (H / H_kv)."""
    return h // (H // H_kv)


def kv_block_bounds(S_KV: int, n_blocks: int) -> list[tuple[int, int]]:
    """Partition of the key/value sequence into n stationary blocks.

    LV-XAttn review page, Figure 3 (the KV sequence is partitioned into one
    block K_i, V_i per worker) and "The reading".  The pages use sequence
    lengths that n divides; for the general case block i is
    [i*ceil(S_KV/n), min((i+1)*ceil(S_KV/n), S_KV)), possibly empty.
    """
    if n_blocks < 1:
        raise ValueError("n_blocks must be >= 1")
    bs = -(-S_KV // n_blocks) if S_KV > 0 else 0
    out = []
    for i in range(n_blocks):
        lo = min(i * bs, S_KV)
        hi = min((i + 1) * bs, S_KV)
        out.append((lo, hi))
    return out


def _logits(qh: np.ndarray, kg: np.ndarray, scale: float, causal: bool,
            rows: np.ndarray, key_offset: int) -> np.ndarray:
    """Scaled logits s[r, j] = scale * <q_r, k_j>, with -inf where masked."""
    s = scale * (qh @ kg.T)
    if causal:
        keys = key_offset + np.arange(kg.shape[0])
        s = np.where(keys[None, :] <= rows[:, None], s, -np.inf)
    return s


def attention_probs(q, k, scale: Optional[float] = None, causal: bool = False,
                    b: int = 0, h: int = 0,
                    rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Softmax attention matrix P[r, j] for one (batch, query head).

    P = softmax_j(scale * q_r . k_j) over the visible keys (Ring Attention
    page, abstract: exact attention; LV-XAttn review page, "Assumptions":
    blockwise evaluation reproduces exactly this result).
    """
    q = _f64(q); k = _f64(k)
    B, S_Q, H, d = q.shape
    H_kv = k.shape[2]
    sc = _default_scale(d, scale)
    rows = np.arange(S_Q) if rows is None else np.asarray(rows)
    s = _logits(q[b, rows, h, :], k[b, :, _kv_head(h, H, H_kv), :], sc, causal, rows, 0)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=1, keepdims=True)


def attention_fwd(q, k, v, scale: Optional[float] = None, causal: bool = False,
                  rows: Optional[Sequence[int]] = None,
                  heads: Optional[Iterable[int]] = None,
                  key_offset: int = 0):
    """Unsplit softmax attention O = softmax(s Q K^T) V and its log-sum-exp.

    The blockwise method reaches this result exactly (LV-XAttn review page,
    "If this is right": the output matches scaled-dot-product attention;
    "Assumptions": online-softmax rescaling is exact).  For each (b, h, r):
      s_j = scale * q_r . k_j   for the visible keys j
      m   = max_j s_j,  Z = sum_j exp(s_j - m)
      o   = sum_j exp(s_j - m) v_j / Z,   lse = m + ln Z
    A row that sees no key (empty key range, or fully masked) returns
    o = 0, lse = -inf.

    ``rows`` restricts the query rows (absolute indices, used for the causal
    mask), ``heads`` the query heads; ``key_offset`` is the absolute index of
    k[:, 0] for the causal mask when k, v are one block of a longer sequence.
    Returns o [B, R, H_sel, d] and lse [B, H_sel, R].
    """
    q = _f64(q); k = _f64(k); v = _f64(v)
    B, S_Q, H, d = q.shape
    S_KV, H_kv = k.shape[1], k.shape[2]
    sc = _default_scale(d, scale)
    rows = np.arange(S_Q) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = list(range(H)) if heads is None else list(heads)
    R = rows.shape[0]
    o = np.zeros((B, R, len(heads), d))
    lse = np.full((B, len(heads), R), -np.inf)
    if S_KV == 0 or R == 0:
        return o, lse
    for b in range(B):
        for hi, h in enumerate(heads):
            g = _kv_head(h, H, H_kv)
            s = _logits(q[b, rows, h, :], k[b, :, g, :], sc, causal, rows, key_offset)
            m = s.max(axis=1)
            seen = np.isfinite(m)
            m_safe = np.where(seen, m, 0.0)
            e = np.exp(s - m_safe[:, None])
            Z = e.sum(axis=1)
            Z_safe = np.where(seen, Z, 1.0)
            o[b, :, hi, :] = np.where(seen[:, None], (e @ v[b, :, g, :]) / Z_safe[:, None], 0.0)
            lse[b, hi, :] = np.where(seen, m_safe + np.log(Z_safe), -np.inf)
    return o, lse


def block_partials(q, k, v, n_blocks: int, scale: Optional[float] = None,
                   causal: bool = False, rows: Optional[Sequence[int]] = None,
                   heads: Optional[Iterable[int]] = None):
    """Per-block partial results (O_i, L_i), one per stationary KV block.

    LV-XAttn review page, Figure 3 / Algorithm 1 and "The reading": each
    worker keeps K_i, V_i and produces, for the queries it sees, the partial
    output O_i and softmax statistics L_i of attention over its own block.
    O_i is the block's normalised attention output, L_i its log-sum-exp.
    For causal self-attention the mask uses absolute key positions, so a
    block entirely above the diagonal gives (0, -inf).
    Returns O [n, B, R, H_sel, d] and L [n, B, H_sel, R].
    """
    k = _f64(k); v = _f64(v)
    Os, Ls = [], []
    for lo, hi in kv_block_bounds(k.shape[1], n_blocks):
        o_i, l_i = attention_fwd(q, k[:, lo:hi], v[:, lo:hi], scale=scale,
                                 causal=causal, rows=rows, heads=heads, key_offset=lo)
        Os.append(o_i); Ls.append(l_i)
    return np.stack(Os), np.stack(Ls)


def merge_partials(O_parts, L_parts):
    """Combine block partials by log-sum-exp rescaling.

    The pages say the partial outputs and statistics are "rescaled as in
    FlashAttention" (LV-XAttn review page, "What carries the argument";
    "Assumptions": the rescaling is exact).  Written out:
      M = max_i L_i,   L = M + ln sum_i exp(L_i - M),
      O = sum_i exp(L_i - L) O_i
    where O_i are normalised partial outputs.  If every L_i is -inf the row
    saw no key: O = 0, L = -inf.
    O_parts [n, B, R, H, d], L_parts [n, B, H, R] -> O [B, R, H, d], L [B, H, R].
    """
    O_parts = _f64(O_parts); L_parts = _f64(L_parts)
    M = L_parts.max(axis=0)                                   # [B, H, R]
    seen = np.isfinite(M)
    M_safe = np.where(seen, M, 0.0)
    w = np.exp(L_parts - M_safe[None])                        # [n, B, H, R]
    tot = w.sum(axis=0)
    L = np.where(seen, M_safe + np.log(np.where(seen, tot, 1.0)), -np.inf)
    coef = np.where(seen[None], np.exp(L_parts - np.where(seen, L, 0.0)[None]), 0.0)
    # coef [n, B, H, R] -> [n, B, R, H, 1]
    coef = np.transpose(coef, (0, 1, 3, 2))[..., None]
    O = (coef * O_parts).sum(axis=0)
    return O, L


def attention_bwd(q, k, v, do, scale: Optional[float] = None, causal: bool = False):
    """Exact gradient of O = softmax(s Q K^T) V with respect to Q, K, V.

    The pages leave the backward pass unspecified (LV-XAttn review page,
    referee report, major comment 1, which asks for a check against the
    exact formula's gradient).  This is that textbook gradient, from the
    oracle's own probabilities P:
      dV = P^T dO,   dP = dO V^T,   D_r = sum_j P_rj dP_rj,
      dS = P o (dP - D),   dQ = s dS K,   dK = s dS^T Q.
    With grouped-query heads, dK and dV sum over the query heads of a group.
    """
    q = _f64(q); k = _f64(k); v = _f64(v); do = _f64(do)
    B, S_Q, H, d = q.shape
    H_kv = k.shape[2]
    sc = _default_scale(d, scale)
    dq = np.zeros_like(q); dk = np.zeros_like(k); dv = np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            g = _kv_head(h, H, H_kv)
            P = attention_probs(q, k, scale=sc, causal=causal, b=b, h=h)
            dO = do[b, :, h, :]
            dv[b, :, g, :] += P.T @ dO
            dP = dO @ v[b, :, g, :].T
            D = (P * dP).sum(axis=1, keepdims=True)
            dS = P * (dP - D)
            dq[b, :, h, :] = sc * (dS @ k[b, :, g, :])
            dk[b, :, g, :] += sc * (dS.T @ q[b, :, h, :])
    return dq, dk, dv


def attention_bwd_rows(q, k, v, do, rows: Sequence[int], scale: Optional[float] = None,
                       causal: bool = False, batches: Optional[Iterable[int]] = None):
    """dQ of ``attention_bwd`` for some query rows (all query heads).

    dQ_r depends only on row r's own softmax: dQ_r = s sum_j P_rj (dP_rj - D_r) k_j.
    Returns dq of shape [B_sel, len(rows), H, d].
    """
    q = _f64(q); k = _f64(k); v = _f64(v); do = _f64(do)
    B, S_Q, H, d = q.shape
    H_kv = k.shape[2]
    sc = _default_scale(d, scale)
    rows = np.asarray(rows, dtype=np.int64)
    batches = list(range(B)) if batches is None else list(batches)
    dq = np.zeros((len(batches), len(rows), H, d))
    for bi, b in enumerate(batches):
        for h in range(H):
            g = _kv_head(h, H, H_kv)
            P = attention_probs(q, k, scale=sc, causal=causal, b=b, h=h, rows=rows)
            dP = do[b, rows, h, :] @ v[b, :, g, :].T
            D = (P * dP).sum(axis=1, keepdims=True)
            dq[bi, :, h, :] = sc * ((P * (dP - D)) @ k[b, :, g, :])
    return dq


def attention_bwd_keys(q, k, v, do, keys: Sequence[int], kv_heads: Iterable[int],
                       scale: Optional[float] = None, causal: bool = False,
                       batches: Optional[Iterable[int]] = None,
                       row_chunk: int = 256, rows: Optional[Sequence[int]] = None):
    """dK and dV of ``attention_bwd`` restricted to some keys and KV heads.

    Same definition as ``attention_bwd``; each query row's P and D need that
    row's full set of logits, so rows are evaluated independently (in chunks
    of ``row_chunk`` rows to bound memory) and only the requested key columns
    of dK, dV are kept.  ``rows`` limits the query rows summed over; it is
    only exact when the other rows give the keys no gradient (causal masking
    with keys j > every omitted row).  Returns dk, dv of shape
    [B_sel, len(keys), len(kv_heads), d].
    """
    q = _f64(q); k = _f64(k); v = _f64(v); do = _f64(do)
    B, S_Q, H, d = q.shape
    H_kv = k.shape[2]
    sc = _default_scale(d, scale)
    keys = np.asarray(keys, dtype=np.int64)
    kv_heads = list(kv_heads)
    batches = list(range(B)) if batches is None else list(batches)
    grp = H // H_kv
    all_rows = np.arange(S_Q) if rows is None else np.asarray(rows, dtype=np.int64)
    dk = np.zeros((len(batches), len(keys), len(kv_heads), d))
    dv = np.zeros_like(dk)
    for bi, b in enumerate(batches):
        for gi, g in enumerate(kv_heads):
            for h in range(g * grp, (g + 1) * grp):
                for r0 in range(0, len(all_rows), row_chunk):
                    rows_c = all_rows[r0:r0 + row_chunk]
                    P = attention_probs(q, k, scale=sc, causal=causal, b=b, h=h, rows=rows_c)
                    dO = do[b, rows_c, h, :]
                    dP = dO @ v[b, :, g, :].T
                    D = (P * dP).sum(axis=1, keepdims=True)
                    Pj = P[:, keys]
                    dSj = Pj * (dP[:, keys] - D)
                    dv[bi, :, gi, :] += Pj.T @ dO
                    dk[bi, :, gi, :] += sc * (dSj.T @ q[b, rows_c, h, :])
    return dk, dv


def kv_recompute(y, w_k, w_v, rows: Optional[Sequence[int]] = None):
    """Keys and values regenerated from the shared visual features.

    LV-XAttn review page, "What carries the argument" and Figure 6: one copy
    of the visual features y is kept for all cross-attention layers and K, V
    are recomputed from it in the backward pass.  K = y W_k, V = y W_v, with
    y [B, S_KV, d_embed] (or [S_KV, d_embed]) and W [d_embed, H_kv*d]
    row-major, no bias.  Returns K, V of shape [..., S_sel, H_kv*d] in fp64.
    """
    y = _f64(y); w_k = _f64(w_k); w_v = _f64(w_v)
    if rows is not None:
        y = y[..., np.asarray(rows), :]
    return y @ w_k, y @ w_v


def kv_recompute_bwd(y, w_k, w_v, dk, dv, rows: Optional[Sequence[int]] = None):
    """Gradients of the K/V recomputation K = y W_k, V = y W_v.

    LV-XAttn review page, "What carries the argument" and Figure 6: keys and
    values are regenerated from the one shared copy of the visual features
    y, so training needs the gradients of that linear map (the pages do not
    write them out; this is the textbook gradient of a matrix product):
      dW_k = y^T dK,   dW_v = y^T dV,   dy = dK W_k^T + dV W_v^T.
    y [S, d_embed] (or [B, S, d_embed], batches summed into dW); dk, dv
    [..., S, H_kv*d]; ``rows`` restricts dy to some rows (dW always uses all).
    Returns dy, dw_k, dw_v in fp64.
    """
    y = _f64(y); w_k = _f64(w_k); w_v = _f64(w_v); dk = _f64(dk); dv = _f64(dv)
    y2 = y.reshape(-1, y.shape[-1])
    dk2 = dk.reshape(-1, dk.shape[-1])
    dv2 = dv.reshape(-1, dv.shape[-1])
    dw_k = y2.T @ dk2
    dw_v = y2.T @ dv2
    if rows is not None:
        rows = np.asarray(rows)
        dy = dk[..., rows, :] @ w_k.T + dv[..., rows, :] @ w_v.T
    else:
        dy = dk @ w_k.T + dv @ w_v.T
    return dy, dw_k, dw_v
