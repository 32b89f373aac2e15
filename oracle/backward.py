"""Gradients of masked softmax attention, fp64 (test infrastructure).

BLADE digest, "技术框架" and the abstract: ASA is trained jointly with the
sparsity-aware step distillation, so the network differentiates through the
attention over the kept blocks.  The pages print no backward formulas; the
plain reading used here:

* the block mask is a constant of the step (its selection is piecewise constant
  in Q and K and carries no gradient);
* the gradient is that of the forward definition (``attention.py``: softmax of
  scale * q_t . k_u over the key tokens u < N of the listed blocks) with respect
  to q, k and v, given dO = d(loss)/dO;
* the LSE output receives no gradient.

For a query token t with key set K_t and an incoming dO_t:

  P_tu  = exp(scale q_t.k_u - LSE_t)           u in K_t
  dV_u += P_tu dO_t
  dP_tu = dO_t . v_u
  D_t   = sum_u P_tu dP_tu                      (equals dO_t . O_t)
  dS_tu = P_tu (dP_tu - D_t)
  dQ_t  = scale sum_u dS_tu k_u
  dK_u += scale dS_tu q_t

A token whose row lists nothing (skip head) contributes nothing and gets
dQ_t = 0.

``mask_transpose`` lists, for every kv-block j of a (b, h), the q-blocks whose
rows keep j: the view a key-side gradient pass walks.  It is the plain
transpose of the CSR block mask.
"""
from __future__ import annotations

import math

import numpy as np

from .attention import _row_keys


def attention_backward(q, k, v, do, blk: int, row_ptr, col_idx, scale: float | None = None):
    """dQ, dK, dV [B, H, N, d] float64 of sum(dO * O) over every mask row.

    q, k, v, do: float64 [B, H, N, d]; the CSR mask is the forward's.
    """
    q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
    B, H, n, d = q.shape
    nb = -(-n // blk)
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for r in range(B * H * nb):
        i = r % nb
        bh = r // nb
        b, h = bh // H, bh % H
        t0, t1 = i * blk, min(n, (i + 1) * blk)
        keys = _row_keys(col_idx[row_ptr[r]:row_ptr[r + 1]], blk, n)
        if keys.size == 0:
            continue
        qt, kt, vt, dot = q[b, h, t0:t1], k[b, h, keys], v[b, h, keys], do[b, h, t0:t1]
        s = (qt @ kt.T) * scale
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        p = e / e.sum(axis=1, keepdims=True)
        dv[b, h, keys] += p.T @ dot
        dp = dot @ vt.T
        dd = (p * dp).sum(axis=1, keepdims=True)
        ds = p * (dp - dd)
        dq[b, h, t0:t1] += scale * (ds @ kt)
        dk[b, h, keys] += scale * (ds.T @ qt)
    return dq, dk, dv


def mask_transpose(row_ptr, col_idx, B: int, H: int, nb: int):
    """CSC view of a CSR block mask.

    Input rows r = (b*H + h)*nb + i list kv-blocks j.  Output column
    c = (b*H + h)*nb + j lists, ascending, every q-block i whose row keeps j.
    Returns (col_ptr [B*H*nb + 1] int64, row_idx [nnz] int32).
    """
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    col_idx = np.asarray(col_idx, dtype=np.int64)
    cols = [[] for _ in range(B * H * nb)]
    for r in range(B * H * nb):
        bh, i = divmod(r, nb)
        for j in col_idx[row_ptr[r]:row_ptr[r + 1]]:
            cols[bh * nb + int(j)].append(i)
    col_ptr = np.zeros(B * H * nb + 1, dtype=np.int64)
    col_ptr[1:] = np.cumsum([len(c) for c in cols])
    row_idx = np.asarray([i for c in cols for i in sorted(c)], dtype=np.int32)
    return col_ptr, row_idx


def attention_backward_sampled(q, k, v, do, blk: int, row_ptr, col_idx, q_rows, kv_cols,
                               scale: float | None = None):
    """The same gradients, for a sample only.

    q_rows: CSR row ids r = (b*H + h)*nb + i -> {r: dQ [tokens of q-block i, d]}.
    kv_cols: ids c = (b*H + h)*nb + j -> {c: (dK, dV) [tokens of kv-block j, d]},
    summed over every row of that (b, h) that lists j.
    """
    q, k, v, do = (np.asarray(x) for x in (q, k, v, do))
    B, H, n, d = q.shape
    nb = -(-n // blk)
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    col_idx = np.asarray(col_idx, dtype=np.int64)

    def row_terms(r):
        i = r % nb
        bh = r // nb
        b, h = bh // H, bh % H
        t0, t1 = i * blk, min(n, (i + 1) * blk)
        cols = col_idx[row_ptr[r]:row_ptr[r + 1]]
        keys = _row_keys(cols, blk, n)
        qt = q[b, h, t0:t1].astype(np.float64)
        dot = do[b, h, t0:t1].astype(np.float64)
        kt = k[b, h, keys].astype(np.float64)
        vt = v[b, h, keys].astype(np.float64)
        s = (qt @ kt.T) * scale
        e = np.exp(s - s.max(axis=1, keepdims=True))
        p = e / e.sum(axis=1, keepdims=True)
        dp = dot @ vt.T
        ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
        return keys, qt, dot, kt, p, ds

    dq = {}
    for r in q_rows:
        r = int(r)
        i = r % nb
        rows_here = min(n, (i + 1) * blk) - i * blk
        if row_ptr[r + 1] == row_ptr[r]:
            dq[r] = np.zeros((rows_here, d))
            continue
        keys, qt, dot, kt, p, ds = row_terms(r)
        dq[r] = scale * (ds @ kt)
    dkv = {}
    for c in kv_cols:
        c = int(c)
        j = c % nb
        bh = c // nb
        u0, u1 = j * blk, min(n, (j + 1) * blk)
        gk = np.zeros((u1 - u0, d))
        gv = np.zeros((u1 - u0, d))
        for i in range(nb):
            r = bh * nb + i
            cols = col_idx[row_ptr[r]:row_ptr[r + 1]]
            if j not in cols:
                continue
            keys, qt, dot, kt, p, ds = row_terms(r)
            sel = (keys >= u0) & (keys < u1)
            gv += p[:, sel].T @ dot
            gk += scale * (ds[:, sel].T @ qt)
        dkv[c] = (gk, gv)
    return dq, dkv
