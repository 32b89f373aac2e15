"""Pins of the fixed-pattern oracle: every block rule against enumeration of all
token pairs (t, u) of the two blocks under the token-level definition, plus the
special cases that reduce to textbook masks."""
import itertools

import numpy as np
import pytest

import oracle
from oracle.patterns import DIAG, FULL, MULTIDIAG, SKIP, STRIPE, TILE3D

CASES = [
    # n, blk, frame_tokens, band_w, f_lo, f_hi, stripe_blocks, global_frames
    (96, 8, 20, 1, -2, 2, 1, 1),
    (101, 8, 24, 2, -1, 1, 2, 0),
    (70, 16, 30, 0, -2, 2, 1, 2),
    (64, 4, 16, 2, 0, 0, 3, 1),
    (50, 7, 13, 1, -3, 3, 1, 1),
    (90, 8, 21, 1, -1, 1, 0, 0),      # no stripe tokens: frame starts inside blocks
]


def _brute_row(pattern, i, n, blk, S, w, f_lo, f_hi, sb, g):
    nb = -(-n // blk)
    ti = range(i * blk, min(n, (i + 1) * blk))
    out = []
    for j in range(nb):
        uj = range(j * blk, min(n, (j + 1) * blk))
        if any(oracle.keep_token_pair(pattern, t, u, blk, S, w, f_lo, f_hi, sb, g)
               for t, u in itertools.product(ti, uj)):
            out.append(j)
    return out


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("pattern", [FULL, SKIP, MULTIDIAG, STRIPE, TILE3D])
def test_block_rule_equals_token_enumeration(case, pattern):
    n, blk, S, w, f_lo, f_hi, sb, g = case
    nb = -(-n // blk)
    for i in range(nb):
        got = oracle.pattern_row(pattern, i, nb, n, blk, w, S, f_lo, f_hi, sb, g)
        assert got == _brute_row(pattern, i, n, blk, S, w, f_lo, f_hi, sb, g), (pattern, i)


@pytest.mark.parametrize("case", CASES)
def test_diag_is_multidiag_at_frame_offset_zero(case):
    n, blk, S, w, _, _, sb, g = case
    nb = -(-n // blk)
    for i in range(nb):
        d = oracle.pattern_row(DIAG, i, nb, n, blk, w, S, 0, 0, sb, g)
        m = oracle.pattern_row(MULTIDIAG, i, nb, n, blk, w, S, 0, 0, sb, g)
        assert d == m
        assert d == [j for j in range(nb) if abs(i - j) <= w]   # matrix bandwidth w


def test_tile3d_frame_aligned_is_block_diagonal():
    # frames of 32 tokens, blocks of 8: frame f = blocks 4f..4f+3; no global frame
    n, blk, S = 128, 8, 32
    nb = n // blk
    for i in range(nb):
        got = oracle.pattern_row(TILE3D, i, nb, n, blk, 0, S, 0, 0, 0, 0)
        f = i // 4
        assert got == list(range(4 * f, 4 * f + 4))


def test_pattern_mask_replicates_over_batch_and_skip_rows_empty():
    hp = [FULL, SKIP, DIAG, MULTIDIAG, STRIPE, TILE3D]
    rp, ci = oracle.pattern_mask(hp, 2, 6, 100, 8, 1, 24, -1, 1, 1, 1)
    nb = 13
    per_b = 6 * nb
    row = lambda r: ci[rp[r]:rp[r + 1]].tolist()
    for r in range(per_b):
        assert row(r) == row(r + per_b)
    for i in range(nb):
        assert row(1 * nb + i) == []
        assert row(0 * nb + i) == list(range(nb))
    assert rp[0] == 0 and np.all(np.diff(rp) >= 0)


def test_tile3d_hand_example_not_frame_aligned():
    # tests/golden/tile3d_example.json: rows derived by hand from the token-level
    # reading, for frames (6 tokens) that straddle the blocks (4 tokens) and a
    # partial last frame and block
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "tile3d_example.json")) as f:
        g = json.load(f)
    n, S, blk = g["N"], g["frame_tokens"], g["blk"]
    nb = -(-n // blk)
    for gf, rows in g["rows"].items():
        got = [oracle.pattern_row(TILE3D, i, nb, n, blk, 0, S, 0, 0, 0, int(gf)) for i in range(nb)]
        assert got == rows, (gf, got)
        rp, ci = oracle.pattern_mask([TILE3D], 1, 1, n, blk, 0, S, 0, 0, 0, int(gf))
        assert [ci[rp[i]:rp[i + 1]].tolist() for i in range(nb)] == rows
