"""Fixed block masks, exact token-level closed forms (test infrastructure).

Sparse-vDiT blog, "四种注意力模式" table and "解决方案概述":
  M0 full            every block (sparsity 0);
  M1 skip            the head is skipped and its output is zero (sparsity 1);
  M2 diagonal        large values on the main diagonal (intra-frame interaction);
  M3 multi-diagonal  several evenly spaced diagonals (cross-frame consistency);
  M4 vertical stripe global tokens that every query attends to.
Efficient-vDiT blog, "3.1 注意力图块化": the 3D attention map repeats block-wise,
giving a pruned pattern of linear complexity that keeps inter-frame consistency.

The pages give no widths, strides or counts.  The readings used (parameters are
inputs): a block pair (i, j) is kept when some token pair (t, u), t in q-block i
and u in kv-block j (both clipped to N), satisfies

  diag        |i - j| <= w                                   (matrix bandwidth w)
  multidiag   exists f in [f_lo, f_hi]: |u - t - f*S| <= w*blk  (S = frame tokens)
  stripe      u in [f*S, f*S + stripe_blocks*blk) for some frame f
  tile3d      frame(u) == frame(t) or frame(u) < g              (g global frames)

For f = 0 the multidiag rule is exactly the diagonal band.  Token indices are
positions in the sequence as given (no text offset).
"""
from __future__ import annotations

import numpy as np

FULL, SKIP, DIAG, MULTIDIAG, STRIPE, TILE3D = 0, 1, 2, 3, 4, 5


def _span(j: int, blk: int, n: int):
    return j * blk, min(n, (j + 1) * blk) - 1


def keep_token_pair(pattern: int, t: int, u: int, blk: int, frame_tokens: int, band_w: int,
                    f_lo: int, f_hi: int, stripe_blocks: int, tile_global_frames: int) -> bool:
    """The token-level definition each block rule is derived from (diag is block-level)."""
    S = frame_tokens
    if pattern == FULL:
        return True
    if pattern == SKIP:
        return False
    if pattern == MULTIDIAG:
        return any(abs(u - t - f * S) <= band_w * blk for f in range(f_lo, f_hi + 1))
    if pattern == STRIPE:
        return (u % S) < stripe_blocks * blk
    if pattern == TILE3D:
        return (u // S) == (t // S) or (u // S) < tile_global_frames
    raise ValueError(pattern)


def pattern_row(pattern: int, i: int, nb: int, n: int, blk: int, band_w: int, frame_tokens: int,
                f_lo: int, f_hi: int, stripe_blocks: int, tile_global_frames: int) -> list:
    """Kept kv-blocks of q-block i, ascending (the rule evaluated for all j at once)."""
    S = frame_tokens
    if pattern == FULL:
        return list(range(nb))
    if pattern == SKIP:
        return []
    if pattern == DIAG:
        return list(range(max(0, i - band_w), min(nb, i + band_w + 1)))
    ti_lo, ti_hi = _span(i, blk, n)
    j = np.arange(nb, dtype=np.int64)
    uj_lo = j * blk
    uj_hi = np.minimum(n, (j + 1) * blk) - 1
    if pattern == MULTIDIAG:
        # offsets u - t over the two blocks form the integer interval [lo, hi]
        lo, hi = uj_lo - ti_hi, uj_hi - ti_lo
        keep = np.zeros(nb, dtype=bool)
        for f in range(f_lo, f_hi + 1):
            keep |= (lo <= f * S + band_w * blk) & (hi >= f * S - band_w * blk)
    elif pattern == STRIPE:
        # the first stripe token at or after uj_lo lies in the block (there is
        # none when a frame has no stripe tokens)
        f = uj_lo // S
        keep = ((uj_lo - f * S) < stripe_blocks * blk) | ((f + 1) * S <= uj_hi)
        if stripe_blocks <= 0:
            keep = np.zeros(nb, dtype=bool)
    elif pattern == TILE3D:
        fi_lo, fi_hi = ti_lo // S, ti_hi // S
        fj_lo, fj_hi = uj_lo // S, uj_hi // S
        keep = ((fj_lo <= fi_hi) & (fj_hi >= fi_lo)) | (fj_lo < tile_global_frames)
    else:
        raise ValueError(pattern)
    return np.nonzero(keep)[0].tolist()


def pattern_mask(head_pattern, B: int, H: int, n: int, blk: int, band_w: int, frame_tokens: int,
                 f_lo: int, f_hi: int, stripe_blocks: int, tile_global_frames: int):
    """CSR (row_ptr int64 [B*H*nb+1], col_idx int32) for per-head patterns, rows replicated over b."""
    nb = -(-n // blk)
    per_head = []
    for h in range(H):
        per_head.append([pattern_row(int(head_pattern[h]), i, nb, n, blk, band_w, frame_tokens,
                                     f_lo, f_hi, stripe_blocks, tile_global_frames)
                         for i in range(nb)])
    row_ptr = [0]
    cols = []
    for _b in range(B):
        for h in range(H):
            for i in range(nb):
                cols.extend(per_head[h][i])
                row_ptr.append(len(cols))
    return np.asarray(row_ptr, dtype=np.int64), np.asarray(cols, dtype=np.int32)
