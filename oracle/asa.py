"""ASA block mask, fp64 (test infrastructure; see the package docstring).

BLADE digest, abstract: ASA "dynamically generates content-aware sparsity masks"
so that attention is computed where the spatio-temporal features are salient;
"方法详解 / 关键设计" reads this as scoring the relevance between blocks and
keeping a block according to that relevance.  The pages stop there.  The steps
below are the plainest reading that fits, in the order they are applied:

1. pool   -- mean of each token block's *valid* rows (the last block may be
             partial): q̄_i = (1/|I_i|) Σ_{t∈I_i} q_t, I_i = [i·blk, min((i+1)·blk, N)).
2. score  -- s_ij = q̄_i · k̄_j · scale with scale = 1/√d (the attention scale of
             the Sparse-vDiT blog, "核心公式"); p_i = softmax_j(s_i) over all nb
             blocks of the (b, h).
3. order  -- blocks sorted by (p descending, block index ascending).
4. keep   -- top-k: the first k; mass: the shortest prefix whose sum reaches τ.
5. cap    -- truncate to max(1, floor(ρ·nb)) when ρ > 0.
6. force  -- union with the diagonal block (i) and the first n_sink blocks.
7. CSR    -- row r = (b·H + h)·nb + i lists its blocks ascending.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

MODE_TOPK = 0
MODE_MASS = 1


def pool(x: np.ndarray, blk: int) -> np.ndarray:
    """Block means over valid tokens.  x [..., N, d] float64 -> [..., nb, d]."""
    n = x.shape[-2]
    nb = -(-n // blk)
    out = np.empty(x.shape[:-2] + (nb, x.shape[-1]), dtype=np.float64)
    for i in range(nb):
        lo, hi = i * blk, min(n, (i + 1) * blk)
        out[..., i, :] = x[..., lo:hi, :].sum(axis=-2) / float(hi - lo)
    return out


def pooled_probs(q: np.ndarray, k: np.ndarray, blk: int, scale: float | None = None) -> np.ndarray:
    """p[b, h, i, j] = softmax_j(q̄_i · k̄_j · scale).  q, k [B, H, N, d] float64."""
    d = q.shape[-1]
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    qb = pool(q, blk)
    kb = pool(k, blk)
    s = np.matmul(qb, np.swapaxes(kb, -1, -2)) * scale
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=-1, keepdims=True)


def keep_cap(nb: int, max_keep_ratio: float) -> int:
    """Largest number of selected (non-forced) blocks; nb when there is no cap."""
    if max_keep_ratio <= 0:
        return nb
    return max(1, int(math.floor(max_keep_ratio * nb)))


@dataclass
class RowSelection:
    cols: list            # kept blocks, ascending (forced ones included)
    p_thr: float          # p of the last block kept by the rule (after the cap)
    mass_at_cut: float    # cumulative p of the kept prefix (before the cap)
    n_selected: int       # blocks kept by the rule (before forcing)
    mass_before_cut: float = 0.0  # cumulative p of the prefix one shorter
    n_prefix: int = 0     # length of the rule's prefix before the cap


def select_row(p_row: np.ndarray, i: int, mode: int, topk: int = 0, mass_tau: float = 0.0,
               max_keep_ratio: float = 0.0, keep_diag: int = 0, n_sink_blocks: int = 0) -> RowSelection:
    """Steps 3-6 for one q-block row."""
    nb = p_row.shape[0]
    # (p desc, index asc): lexsort's last key is the primary one.
    order = np.lexsort((np.arange(nb), -p_row))
    if mode == MODE_TOPK:
        m = min(max(topk, 0), nb)
        mass = math.fsum(p_row[order[:m]].tolist())
        before = math.fsum(p_row[order[:max(m - 1, 0)]].tolist())
    elif mode == MODE_MASS:
        ps = p_row[order]
        csum = np.cumsum(ps)
        hit = np.nonzero(csum >= mass_tau)[0]
        m = int(hit[0]) + 1 if hit.size else nb
        # settle the cut on exactly rounded prefix sums, not on the running sum's rounding
        prefix = lambda n: math.fsum(ps[:n].tolist())
        while m > 1 and prefix(m - 1) >= mass_tau:
            m -= 1
        while m < nb and prefix(m) < mass_tau:
            m += 1
        mass = prefix(m)
        before = prefix(m - 1)
    else:
        raise ValueError(f"unknown mode {mode}")
    m_prefix = m
    m = min(m, keep_cap(nb, max_keep_ratio))
    chosen = set(int(j) for j in order[:m])
    p_thr = float(p_row[order[m - 1]]) if m > 0 else float("inf")
    if keep_diag:
        chosen.add(int(i))
    chosen.update(range(min(max(n_sink_blocks, 0), nb)))
    return RowSelection(sorted(chosen), p_thr, mass, m, before, m_prefix)


@dataclass
class MaskInfo:
    row_ptr: np.ndarray   # int64 [rows + 1]
    col_idx: np.ndarray   # int32 [nnz]
    p_thr: np.ndarray     # float64 [rows]
    mass_at_cut: np.ndarray  # float64 [rows]
    probs: np.ndarray     # float64 [B, H, nb, nb]
    mass_before_cut: np.ndarray = None  # float64 [rows]
    n_prefix: np.ndarray = None  # int64 [rows]: the rule's prefix length before the cap


def asa_mask(q: np.ndarray, k: np.ndarray, blk: int, mode: int, topk: int = 0,
             mass_tau: float = 0.0, max_keep_ratio: float = 0.0, keep_diag: int = 0,
             n_sink_blocks: int = 0, scale: float | None = None) -> MaskInfo:
    """Steps 1-7 for every (b, h, i).  q, k [B, H, N, d] float64."""
    B, H, N, _ = q.shape
    nb = -(-N // blk)
    p = pooled_probs(q, k, blk, scale)
    rows = B * H * nb
    row_ptr = np.zeros(rows + 1, dtype=np.int64)
    cols = []
    p_thr = np.empty(rows)
    mass = np.empty(rows)
    before = np.empty(rows)
    n_prefix = np.empty(rows, dtype=np.int64)
    r = 0
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                sel = select_row(p[b, h, i], i, mode, topk, mass_tau, max_keep_ratio, keep_diag,
                                 n_sink_blocks)
                cols.extend(sel.cols)
                row_ptr[r + 1] = row_ptr[r] + len(sel.cols)
                p_thr[r] = sel.p_thr
                mass[r] = sel.mass_at_cut
                before[r] = sel.mass_before_cut
                n_prefix[r] = sel.n_prefix
                r += 1
    return MaskInfo(row_ptr, np.asarray(cols, dtype=np.int32), p_thr, mass, p, before, n_prefix)
