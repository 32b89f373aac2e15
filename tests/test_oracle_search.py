"""Pins of the oracle's Sparse-vDiT search quantities (CPU).

* MSE vs an element-by-element Python loop;
* sparsity vs token-pair enumeration of the mask, and the page's fixed values
  (M0 full: 0, M1 skip: 1);
* the loss and the eps rule on hand-made cases (all above eps -> full; argmin
  otherwise; ties -> first listed);
* a pattern that keeps every block reproduces full attention (MSE 0), and the
  skip pattern's MSE is the mean square of the full output.
"""
import itertools

import numpy as np

import oracle
from oracle import search


def test_head_mse_brute_force():
    rng = np.random.default_rng(5)
    a = rng.standard_normal((2, 3, 7, 4))
    b = rng.standard_normal((2, 3, 7, 4))
    got = search.head_mse(a, b)
    for h in range(3):
        s, n = 0.0, 0
        for bb, t, e in itertools.product(range(2), range(7), range(4)):
            s += (b[bb, h, t, e] - a[bb, h, t, e]) ** 2
            n += 1
        assert abs(got[h] - s / n) < 1e-12


def _pairs_brute(rp, ci, B, H, N, blk):
    nb = -(-N // blk)
    kept = np.zeros(H)
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                r = (b * H + h) * nb + i
                cols = set(ci[rp[r]:rp[r + 1]].tolist())
                for t in range(i * blk, min(N, (i + 1) * blk)):
                    for u in range(N):
                        if u // blk in cols:
                            kept[h] += 1
    return 1.0 - kept / (B * N * N)


def test_head_sparsity_token_pairs_and_fixed_values():
    B, N, blk = 2, 70, 16           # ragged last block (6 tokens)
    hp = [0, 1, 2, 3, 4, 5]
    rp, ci = oracle.pattern_mask(hp, B, len(hp), N, blk, 1, 32, -1, 1, 1, 1)
    got = search.head_sparsity(rp, ci, B, len(hp), N, blk)
    np.testing.assert_allclose(got, _pairs_brute(rp, ci, B, len(hp), N, blk), atol=1e-15)
    assert got[0] == 0.0 and got[1] == 1.0          # M0 full, M1 skip
    # diagonal band w = 0 keeps the diagonal blocks: sum of n_i^2 over N^2
    rp0, ci0 = oracle.pattern_mask([2], 1, 1, N, blk, 0, 32, 0, 0, 1, 0)
    sizes = [16, 16, 16, 16, 6]
    want = 1.0 - sum(s * s for s in sizes) / N ** 2
    assert abs(search.head_sparsity(rp0, ci0, 1, 1, N, blk)[0] - want) < 1e-15


def test_loss_and_selection_rule():
    mse = np.array([[0.50, 0.01, 0.02],     # candidate 1 (skip)
                    [0.03, 0.20, 0.02],     # candidate 2 (diag)
                    [0.04, 0.20, 0.30]])    # candidate 3 (multidiag)
    spars = np.array([[1.0, 1.0, 1.0],
                      [0.9, 0.9, 0.9],
                      [0.5, 0.5, 0.8]])
    lam = 0.1
    L = search.search_loss(mse, spars, lam)
    np.testing.assert_allclose(L[:, 0], [0.50, 0.03 + 0.01, 0.04 + 0.05])
    # head 0: diag (0.04) is best; head 1: skip (0.01); head 2: skip (0.02) beats diag (0.03)
    got = search.select_pattern(L, [1, 2, 3], eps=0.1)
    assert got.tolist() == [2, 1, 1]
    # every loss above eps -> full attention
    assert search.select_pattern(L, [1, 2, 3], eps=0.005).tolist() == [0, 0, 0]
    # exact tie -> the candidate listed first
    tie = np.array([[0.02], [0.02]])
    assert search.select_pattern(tie, [4, 2], eps=1.0).tolist() == [4]


def test_all_block_pattern_equals_full_and_skip_mse():
    rng = np.random.default_rng(9)
    B, H, N, d, blk = 1, 2, 48, 8, 16
    q, k, v = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    rp0, ci0 = oracle.pattern_mask([0, 0], B, H, N, blk, 0, 16, 0, 0, 1, 0)
    o0, _ = oracle.masked_attention(q, k, v, blk, rp0, ci0)
    # a diagonal band as wide as the head keeps every block
    rpw, ciw = oracle.pattern_mask([2, 2], B, H, N, blk, 10, 16, 0, 0, 1, 0)
    ow, _ = oracle.masked_attention(q, k, v, blk, rpw, ciw)
    assert np.all(search.head_mse(o0, ow) == 0.0)
    assert np.all(search.head_sparsity(rpw, ciw, B, H, N, blk) == 0.0)
    rps, cis = oracle.pattern_mask([1, 1], B, H, N, blk, 0, 16, 0, 0, 1, 0)
    os_, _ = oracle.masked_attention(q, k, v, blk, rps, cis)
    assert np.all(os_ == 0.0)
    np.testing.assert_allclose(search.head_mse(o0, os_), np.mean(o0 ** 2, axis=(0, 2, 3)),
                               rtol=1e-15)
