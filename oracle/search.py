"""Offline pattern-search quantities of Sparse-vDiT (test infrastructure).

Sparse-vDiT blog, "核心公式 / 离线搜索损失函数" and "注意力模式选择", with the
steps of "Algorithm 1: Offline Sparse Diffusion Search":

  L_i = MSE(O_i - O_0) + lambda * (1 - S_i)

  O_0     output of full attention (M0)
  O_i     output of the head under sparse pattern i
  S_i     sparsity of pattern i
  lambda  quality / efficiency trade-off

and the head keeps full attention when L_i > eps for every candidate i,
otherwise takes the pattern of the smallest L_i.

Readings where the page is silent (the same in the CUDA path):
  * MSE is the mean over every element the head outputs: batch, query tokens
    and the head dimension, i.e. B * N * d terms per head.
  * S_i is the fraction of (query token, key token) pairs of the head that the
    mask does not compute: 1 - (kept pairs) / (B * N * N), the kept pairs of a
    kept block pair (i, j) being n_q(i) * n_k(j) over valid tokens.  M0 gives
    0 and M1 (skip) gives 1, as the page's pattern table states.
  * ties of L_i go to the candidate listed first.
"""
from __future__ import annotations

import numpy as np


def head_mse(o_ref: np.ndarray, o: np.ndarray) -> np.ndarray:
    """MSE(O - O_ref) per head; o_ref, o [B, H, N, d] -> [H] float64."""
    a = np.asarray(o_ref, dtype=np.float64)
    b = np.asarray(o, dtype=np.float64)
    diff = b - a
    return np.mean(diff * diff, axis=(0, 2, 3))


def head_sparsity(row_ptr: np.ndarray, col_idx: np.ndarray, B: int, H: int, N: int,
                  blk: int) -> np.ndarray:
    """S per head from a CSR block mask over B*H*nb rows -> [H] float64."""
    nb = -(-N // blk)
    sizes = np.full(nb, blk, dtype=np.int64)
    sizes[-1] = N - (nb - 1) * blk
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    col_idx = np.asarray(col_idx, dtype=np.int64)
    kept = np.zeros(H, dtype=np.int64)
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                r = (b * H + h) * nb + i
                cols = col_idx[row_ptr[r]:row_ptr[r + 1]]
                kept[h] += int(sizes[i]) * int(sizes[cols].sum())
    return 1.0 - kept / float(B * N * N)


def search_loss(mse: np.ndarray, sparsity: np.ndarray, lam: float) -> np.ndarray:
    """L_i = MSE_i + lambda * (1 - S_i); arrays [P, H] -> [P, H]."""
    return np.asarray(mse, dtype=np.float64) + lam * (1.0 - np.asarray(sparsity, dtype=np.float64))


def select_pattern(loss: np.ndarray, candidates, eps: float, full_id: int = 0) -> np.ndarray:
    """Per head: full_id if every candidate's L > eps, else the candidate of the
    smallest L (first listed on ties).  loss [P, H], candidates [P] -> [H] int."""
    loss = np.asarray(loss, dtype=np.float64)
    P, H = loss.shape
    out = np.empty(H, dtype=np.int64)
    for h in range(H):
        if all(loss[i, h] > eps for i in range(P)):
            out[h] = full_id
            continue
        best = 0
        for i in range(1, P):
            if loss[i, h] < loss[best, h]:
                best = i
        out[h] = candidates[best]
    return out
