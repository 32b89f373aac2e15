"""Masked softmax attention, fp64 (test infrastructure).

Sparse-vDiT blog, "核心公式 / 全注意力机制": per head,
Attention(Q_h, K_h, V_h) = softmax(Q_h K_hᵀ / √d) V_h.  Block-sparse attention
(BLADE digest, abstract: "focus computation" on the kept blocks) applies the
same formula to each query token t of q-block i over only the key tokens of the
blocks listed in its CSR row that lie below N:

  O_t   = Σ_u softmax_u(q_t·k_u·scale) v_u
  LSE_t = ln Σ_u exp(q_t·k_u·scale)        (natural log, scaled-score units)

A row that lists nothing (the skip head M1 of the Sparse-vDiT blog's
"四种注意力模式" table: output set to zero) gives O_t = 0 and LSE_t = -inf.
"""
from __future__ import annotations

import math

import numpy as np


def _row_keys(cols, blk: int, n: int) -> np.ndarray:
    if len(cols) == 0:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(j * blk, min(n, (j + 1) * blk)) for j in cols])


def attention_rows(q, k, v, blk: int, row_ptr, col_idx, rows, scale: float | None = None):
    """O and LSE of the listed mask rows.

    q, k, v: float64 [B, H, N, d].  rows: iterable of CSR row ids r = (b·H + h)·nb + i.
    Returns {r: (O [tokens, d], LSE [tokens])} for the valid tokens of q-block i.
    """
    B, H, n, d = q.shape
    nb = -(-n // blk)
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    out = {}
    for r in rows:
        r = int(r)
        i = r % nb
        bh = r // nb
        b, h = bh // H, bh % H
        t0, t1 = i * blk, min(n, (i + 1) * blk)
        keys = _row_keys(col_idx[row_ptr[r]:row_ptr[r + 1]], blk, n)
        if keys.size == 0:
            out[r] = (np.zeros((t1 - t0, d)), np.full(t1 - t0, -np.inf))
            continue
        s = (q[b, h, t0:t1] @ k[b, h, keys].T) * scale
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)
        o = (e @ v[b, h, keys]) / l
        out[r] = (o, (m + np.log(l))[:, 0])
    return out


def masked_attention(q, k, v, blk: int, row_ptr, col_idx, scale: float | None = None):
    """O [B, H, N, d] and LSE [B, H, N] over every mask row."""
    B, H, n, d = q.shape
    nb = -(-n // blk)
    o = np.zeros((B, H, n, d))
    lse = np.full((B, H, n), -np.inf)
    res = attention_rows(q, k, v, blk, row_ptr, col_idx, range(B * H * nb), scale)
    for r, (orow, lrow) in res.items():
        i = r % nb
        bh = r // nb
        b, h = bh // H, bh % H
        t0, t1 = i * blk, min(n, (i + 1) * blk)
        o[b, h, t0:t1] = orow
        lse[b, h, t0:t1] = lrow
    return o, lse


def attention_probs(q, k, blk: int, row_ptr, col_idx, scale: float | None = None):
    """The attention weights P [B, H, N, N] of every query token over every key
    token: softmax_u(q_t·k_u·scale) over the keys its row lists (u < N), and 0
    for keys it does not list.  A row that lists nothing is all zeros.

    Dense over N x N: for small sequences only (the per-element rounding bounds
    of the gradient tests use it).
    """
    B, H, n, d = q.shape
    nb = -(-n // blk)
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    p = np.zeros((B, H, n, n))
    for r in range(B * H * nb):
        i = r % nb
        bh = r // nb
        b, h = bh // H, bh % H
        t0, t1 = i * blk, min(n, (i + 1) * blk)
        keys = _row_keys(col_idx[row_ptr[r]:row_ptr[r + 1]], blk, n)
        if keys.size == 0:
            continue
        s = (q[b, h, t0:t1] @ k[b, h, keys].T) * scale
        e = np.exp(s - s.max(axis=1, keepdims=True))
        p[b, h, t0:t1][:, keys] = e / e.sum(axis=1, keepdims=True)
    return p
