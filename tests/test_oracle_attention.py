"""Pins of the fp64 masked-attention oracle.

* keep-all == dense attention: torch's float64 scaled_dot_product_attention and
  torch.logsumexp (library routines), with ragged N and d in {64, 128}
* a block mask == dense attention with an additive -inf token mask (SDPA attn_mask)
* invariants: each output row is a convex combination of the kept V rows, the
  LSE bounds, skip rows are exactly zero / -inf, permuting tokens inside a kept
  block changes nothing, one block of identical keys averages its V rows
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _qkv(B, H, N, d, seed):
    rng = np.random.default_rng(seed)
    return tuple(rng.standard_normal((B, H, N, d)) for _ in range(3))


def _full_csr(B, H, nb):
    rows = B * H * nb
    return np.arange(rows + 1, dtype=np.int64) * nb, np.tile(np.arange(nb, dtype=np.int32), rows)


@pytest.mark.parametrize("N,d,blk", [(128, 64, 16), (100, 64, 16), (200, 128, 64), (37, 64, 128)])
def test_keep_all_equals_sdpa(N, d, blk):
    q, k, v = _qkv(2, 2, N, d, N + d)
    nb = -(-N // blk)
    rp, ci = _full_csr(2, 2, nb)
    o, lse = oracle.masked_attention(q, k, v, blk, rp, ci)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    ref_lse = torch.logsumexp(tq @ tk.transpose(-1, -2) / math.sqrt(d), dim=-1).numpy()
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_block_mask_equals_sdpa_token_mask():
    B, H, N, d, blk = 1, 3, 90, 64, 16
    nb = -(-N // blk)
    q, k, v = _qkv(B, H, N, d, 5)
    rng = np.random.default_rng(9)
    rows = []
    for r in range(B * H * nb):
        cols = sorted(rng.choice(nb, size=int(rng.integers(1, nb + 1)), replace=False).tolist())
        rows.append(cols)
    rp = np.zeros(len(rows) + 1, dtype=np.int64)
    rp[1:] = np.cumsum([len(c) for c in rows])
    ci = np.asarray([c for cols in rows for c in cols], dtype=np.int32)
    o, lse = oracle.masked_attention(q, k, v, blk, rp, ci)
    mask = np.full((B, H, N, N), -np.inf)
    for r, cols in enumerate(rows):
        h, i = r // nb, r % nb
        for j in cols:
            mask[0, h, i * blk:(i + 1) * blk, j * blk:(j + 1) * blk] = 0.0
    tq, tk, tv, tm = (torch.from_numpy(x) for x in (q, k, v, mask))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=tm).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    ref_lse = torch.logsumexp(tq @ tk.transpose(-1, -2) / math.sqrt(d) + tm, dim=-1).numpy()
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def _random_csr(rows, nb, seed, p_empty=0.2):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(rows):
        if rng.random() < p_empty:
            out.append([])
        else:
            out.append(sorted(rng.choice(nb, size=int(rng.integers(1, nb + 1)), replace=False).tolist()))
    rp = np.zeros(rows + 1, dtype=np.int64)
    rp[1:] = np.cumsum([len(c) for c in out])
    return rp, np.asarray([c for cols in out for c in cols], dtype=np.int32), out


def test_invariants_convex_combination_and_lse_bounds():
    B, H, N, d, blk = 1, 2, 75, 64, 16
    nb = -(-N // blk)
    q, k, v = _qkv(B, H, N, d, 21)
    rp, ci, rows = _random_csr(B * H * nb, nb, 3)
    o, lse = oracle.masked_attention(q, k, v, blk, rp, ci)
    scale = 1 / math.sqrt(d)
    for r, cols in enumerate(rows):
        h, i = r // nb, r % nb
        toks = slice(i * blk, min(N, (i + 1) * blk))
        if not cols:
            assert np.all(o[0, h, toks] == 0.0) and np.all(np.isneginf(lse[0, h, toks]))
            continue
        keys = np.concatenate([np.arange(j * blk, min(N, (j + 1) * blk)) for j in cols])
        vk = v[0, h, keys]
        assert np.all(o[0, h, toks] >= vk.min(0) - 1e-12) and np.all(o[0, h, toks] <= vk.max(0) + 1e-12)
        s = q[0, h, toks] @ k[0, h, keys].T * scale
        # weights recovered from the LSE sum to one
        w = np.exp(s - lse[0, h, toks][:, None])
        np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-12)
        np.testing.assert_allclose(w @ vk, o[0, h, toks], atol=1e-12)
        assert np.all(lse[0, h, toks] >= s.max(1) - 1e-12)
        assert np.all(lse[0, h, toks] <= s.max(1) + math.log(len(keys)) + 1e-12)


def test_permutation_inside_kept_block_is_invariant():
    B, H, N, d, blk = 1, 1, 64, 64, 16
    q, k, v = _qkv(B, H, N, d, 8)
    rp = np.array([0, 2, 3, 5, 6])
    ci = np.array([0, 2, 1, 0, 3, 2], dtype=np.int32)
    o1, l1 = oracle.masked_attention(q, k, v, blk, rp, ci)
    perm = np.arange(N)
    perm[32:48] = perm[32:48][np.random.default_rng(0).permutation(16)]
    o2, l2 = oracle.masked_attention(q, k[:, :, perm], v[:, :, perm], blk, rp, ci)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


def test_identical_keys_average_values():
    B, H, N, d, blk = 1, 1, 32, 64, 16
    q, k, v = _qkv(B, H, N, d, 4)
    k[0, 0, 16:32] = k[0, 0, 16]
    rp = np.array([0, 1, 2])
    ci = np.array([1, 1], dtype=np.int32)
    o, lse = oracle.masked_attention(q, k, v, blk, rp, ci)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(v[0, 0, 16:32].mean(0), (32, d)), atol=1e-13)
    s = q[0, 0] @ k[0, 0, 16] / math.sqrt(d)
    np.testing.assert_allclose(lse[0, 0], s + math.log(16), atol=1e-12)


def test_skip_row_is_zero_and_neg_inf():
    q, k, v = _qkv(1, 1, 40, 64, 2)
    rp = np.array([0, 0, 1, 1])
    ci = np.array([0], dtype=np.int32)
    o, lse = oracle.masked_attention(q, k, v, 16, rp, ci)
    assert np.all(o[0, 0, :16] == 0.0) and np.all(np.isneginf(lse[0, 0, :16]))
    assert np.all(o[0, 0, 32:] == 0.0) and np.all(np.isneginf(lse[0, 0, 32:]))
    assert np.all(np.isfinite(lse[0, 0, 16:32]))


def test_attention_probs_pins():
    # P @ V is the oracle's O, kept rows sum to 1 and empty rows to 0; with every
    # block kept P is torch's softmax of the scaled scores
    rng = np.random.default_rng(12)
    B, H, N, d, blk = 1, 2, 37, 16, 8
    q, k, v = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    nb = -(-N // blk)
    rows = [[] if r % 3 == 0 else sorted(rng.choice(nb, size=2, replace=False).tolist())
            for r in range(B * H * nb)]
    rp = np.zeros(B * H * nb + 1, dtype=np.int64)
    rp[1:] = np.cumsum([len(c) for c in rows])
    ci = np.asarray([c for cols in rows for c in cols], dtype=np.int32)
    p = oracle.attention_probs(q, k, blk, rp, ci)
    o, lse = oracle.masked_attention(q, k, v, blk, rp, ci)
    np.testing.assert_allclose(p @ v, o, rtol=0, atol=1e-12)
    sums = p.sum(axis=-1)
    np.testing.assert_allclose(sums[np.isfinite(lse)], 1.0, rtol=0, atol=1e-12)
    assert np.all(sums[~np.isfinite(lse)] == 0)
    rp_all = np.arange(B * H * nb + 1, dtype=np.int64) * nb
    ci_all = np.tile(np.arange(nb, dtype=np.int32), B * H * nb)
    p_all = oracle.attention_probs(q, k, blk, rp_all, ci_all)
    want = torch.softmax(torch.from_numpy(q) @ torch.from_numpy(k).transpose(-1, -2) / np.sqrt(d), -1)
    np.testing.assert_allclose(p_all, want.numpy(), rtol=0, atol=1e-12)
