"""Pins of the fp64 attention-gradient oracle and the block-mask transpose (CPU).

* keep-all == torch float64 autograd through scaled_dot_product_attention, with
  ragged N and d in {64, 128};
* a block mask with no empty row == autograd through SDPA with an additive
  -inf token mask;
* central finite differences of the forward oracle on tiny inputs, empty
  rows and a ragged tail included (every element of dQ, dK, dV);
* identities of the softmax that hold for any mask: shifting every key by one
  vector changes nothing; sum_u dK_u = 0; sum_u dV_u = sum of dO over the
  tokens whose row is not empty; sum_t dQ_t . q_t = sum_u dK_u . k_u; scaling
  V by a scales dQ and dK by a and leaves dV;
* special cases: skip rows get dQ = 0 and feed nothing; one block of identical
  keys gives dQ = 0 and dV = the mean of dO over its queries; a permutation
  inside a kept block permutes dK and dV and leaves dQ;
* the transpose vs a dense boolean block matrix, and transposing twice;
* the GPU tests' gradient bounds accept the oracle's own result and reject
  planted mistakes (a dropped scale, swapped gradients, another scale, another
  mask).
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _qkv(B, H, N, d, seed, n=4):
    rng = np.random.default_rng(seed)
    return tuple(rng.standard_normal((B, H, N, d)) for _ in range(n))


def _full_csr(B, H, nb):
    rows = B * H * nb
    return np.arange(rows + 1, dtype=np.int64) * nb, np.tile(np.arange(nb, dtype=np.int32), rows)


def _random_csr(rows, nb, seed, p_empty=0.0):
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


def _autograd(q, k, v, do, mask=None):
    tq, tk, tv = (torch.from_numpy(x.copy()).requires_grad_(True) for x in (q, k, v))
    am = None if mask is None else torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=am)
    o.backward(torch.from_numpy(do))
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("N,d,blk", [(96, 64, 16), (100, 64, 16), (130, 128, 64), (37, 64, 128)])
def test_keep_all_equals_sdpa_autograd(N, d, blk):
    q, k, v, do = _qkv(2, 2, N, d, 7 * N + d)
    rp, ci = _full_csr(2, 2, -(-N // blk))
    got = oracle.attention_backward(q, k, v, do, blk, rp, ci)
    want = _autograd(q, k, v, do)
    for g, w in zip(got, want):
        np.testing.assert_allclose(g, w, rtol=0, atol=1e-12)


def test_block_mask_equals_sdpa_autograd_with_token_mask():
    B, H, N, d, blk = 1, 3, 90, 64, 16
    nb = -(-N // blk)
    q, k, v, do = _qkv(B, H, N, d, 5)
    rp, ci, rows = _random_csr(B * H * nb, nb, 9)
    mask = np.full((B, H, N, N), -np.inf)
    for r, cols in enumerate(rows):
        h, i = r // nb, r % nb
        for j in cols:
            mask[0, h, i * blk:(i + 1) * blk, j * blk:(j + 1) * blk] = 0.0
    got = oracle.attention_backward(q, k, v, do, blk, rp, ci)
    want = _autograd(q, k, v, do, mask)
    for g, w in zip(got, want):
        np.testing.assert_allclose(g, w, rtol=0, atol=1e-12)


def _loss(q, k, v, do, blk, rp, ci, scale=None):
    o, _ = oracle.masked_attention(q, k, v, blk, rp, ci, scale)
    return float(np.sum(o * do))


@pytest.mark.parametrize("scale", [None, 0.7])
def test_central_finite_differences(scale):
    # N = 10 at blk 4: blocks of 4, 4, 2; one empty row per head
    B, H, N, d, blk = 1, 2, 10, 3, 4
    nb = 3
    q, k, v, do = _qkv(B, H, N, d, 13)
    rp = np.array([0, 2, 2, 5, 6, 7, 7], dtype=np.int64)
    ci = np.array([0, 2, 0, 1, 2, 1, 2], dtype=np.int32)
    assert len(rp) == B * H * nb + 1
    grads = oracle.attention_backward(q, k, v, do, blk, rp, ci, scale)
    eps = 1e-6
    for which, g in enumerate(grads):
        for idx in np.ndindex(*q.shape):
            args = [q.copy(), k.copy(), v.copy()]
            args[which][idx] += eps
            up = _loss(*args, do, blk, rp, ci, scale)
            args[which][idx] -= 2 * eps
            dn = _loss(*args, do, blk, rp, ci, scale)
            fd = (up - dn) / (2 * eps)
            assert abs(fd - g[idx]) < 1e-8, (which, idx, fd, g[idx])


def _masked_case(seed, p_empty=0.25):
    B, H, N, d, blk = 2, 2, 75, 64, 16
    nb = -(-N // blk)
    q, k, v, do = _qkv(B, H, N, d, seed)
    rp, ci, rows = _random_csr(B * H * nb, nb, seed + 1, p_empty)
    assert any(not c for c in rows) and any(c for c in rows)
    return q, k, v, do, blk, rp, ci, rows, nb


def test_softmax_identities_any_mask():
    q, k, v, do, blk, rp, ci, rows, nb = _masked_case(31)
    B, H, N, d = q.shape
    dq, dk, dv = oracle.attention_backward(q, k, v, do, blk, rp, ci)
    # a common shift of every key moves each row's scores by a constant
    c = np.random.default_rng(2).standard_normal(d)
    for g, w in zip(oracle.attention_backward(q, k + c, v, do, blk, rp, ci), (dq, dk, dv)):
        np.testing.assert_allclose(g, w, rtol=0, atol=1e-11)
    # each row's dS sums to zero over its keys
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-11)
    live = np.zeros((B, H, N), dtype=bool)
    for r, cols in enumerate(rows):
        bh, i = divmod(r, nb)
        live[bh // H, bh % H, i * blk:min(N, (i + 1) * blk)] = bool(cols)
    np.testing.assert_allclose(dv.sum(axis=2), (do * live[..., None]).sum(axis=2), atol=1e-11)
    np.testing.assert_allclose(np.einsum("bhtd,bhtd->bh", dq, q), np.einsum("bhud,bhud->bh", dk, k),
                               rtol=1e-10, atol=1e-10)
    a = 2.5
    g2 = oracle.attention_backward(q, k, a * v, do, blk, rp, ci)
    np.testing.assert_allclose(g2[0], a * dq, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g2[1], a * dk, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g2[2], dv, rtol=1e-12, atol=1e-12)


def test_skip_rows_get_and_give_nothing():
    q, k, v, do, blk, rp, ci, rows, nb = _masked_case(41)
    B, H, N, d = q.shape
    dq, dk, dv = oracle.attention_backward(q, k, v, do, blk, rp, ci)
    # dO on skip rows changes nothing anywhere
    do2 = do.copy()
    for r, cols in enumerate(rows):
        bh, i = divmod(r, nb)
        toks = slice(i * blk, min(N, (i + 1) * blk))
        if not cols:
            assert np.all(dq[bh // H, bh % H, toks] == 0.0)
            do2[bh // H, bh % H, toks] = 1e3
    for g, w in zip(oracle.attention_backward(q, k, v, do2, blk, rp, ci), (dq, dk, dv)):
        np.testing.assert_array_equal(g, w)
    # kv-blocks that no row lists get zero gradient
    listed = np.zeros((B * H, nb), dtype=bool)
    for r, cols in enumerate(rows):
        listed[r // nb, cols] = True
    for bh in range(B * H):
        for j in np.flatnonzero(~listed[bh]):
            toks = slice(j * blk, min(N, (j + 1) * blk))
            assert np.all(dk[bh // H, bh % H, toks] == 0.0) and np.all(dv[bh // H, bh % H, toks] == 0.0)


def test_identical_keys_block():
    B, H, N, d, blk = 1, 1, 32, 64, 16
    q, k, v, do = _qkv(B, H, N, d, 4)
    k[0, 0, 16:32] = k[0, 0, 16]
    rp = np.array([0, 1, 2])
    ci = np.array([1, 1], dtype=np.int32)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, blk, rp, ci)
    np.testing.assert_allclose(dq, 0.0, atol=1e-13)
    np.testing.assert_allclose(dv[0, 0, 16:32], np.broadcast_to(do[0, 0].sum(0) / 16, (16, d)), atol=1e-13)
    assert np.all(dv[0, 0, :16] == 0.0) and np.all(dk[0, 0, :16] == 0.0)


def test_permutation_inside_kept_block():
    B, H, N, d, blk = 1, 1, 64, 64, 16
    q, k, v, do = _qkv(B, H, N, d, 8)
    rp = np.array([0, 2, 3, 5, 6])
    ci = np.array([0, 2, 1, 0, 3, 2], dtype=np.int32)
    g1 = oracle.attention_backward(q, k, v, do, blk, rp, ci)
    perm = np.arange(N)
    perm[32:48] = perm[32:48][np.random.default_rng(0).permutation(16)]
    g2 = oracle.attention_backward(q, k[:, :, perm], v[:, :, perm], do, blk, rp, ci)
    np.testing.assert_allclose(g2[0], g1[0], atol=1e-13)
    np.testing.assert_allclose(g2[1], g1[1][:, :, perm], atol=1e-13)
    np.testing.assert_allclose(g2[2], g1[2][:, :, perm], atol=1e-13)


def test_default_scale_is_inverse_sqrt_d():
    q, k, v, do = _qkv(1, 1, 20, 64, 3)
    rp, ci = _full_csr(1, 1, 2)
    a = oracle.attention_backward(q, k, v, do, 16, rp, ci)
    b = oracle.attention_backward(q, k, v, do, 16, rp, ci, 1 / math.sqrt(64))
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_mask_transpose_vs_dense(seed):
    B, H, nb = 2, 3, 7
    rp, ci, rows = _random_csr(B * H * nb, nb, seed, p_empty=0.3)
    cp, ri = oracle.mask_transpose(rp, ci, B, H, nb)
    dense = np.zeros((B * H, nb, nb), dtype=bool)
    for r, cols in enumerate(rows):
        dense[r // nb, r % nb, cols] = True
    assert cp[-1] == len(ci) == len(ri)
    for c in range(B * H * nb):
        bh, j = divmod(c, nb)
        assert ri[cp[c]:cp[c + 1]].tolist() == np.flatnonzero(dense[bh, :, j]).tolist()
    # the transpose of the transpose is the mask
    rp2, ci2 = oracle.mask_transpose(cp, ri, B, H, nb)
    assert np.array_equal(rp2, rp) and np.array_equal(ci2, ci)


def test_gradient_comparator_rejects_planted_mistakes():
    # the GPU tests' bounds (tests/_compare.py) accept the oracle and reject
    # a dropped scale, swapped gradients, another softmax scale and another mask
    from tests._compare import compare_gradients, d_term
    B, H, N, d, blk = 1, 2, 96, 64, 16
    nb = N // blk
    q, k, v, do = _qkv(B, H, N, d, 17)
    rp, ci, _ = _random_csr(B * H * nb, nb, 5, p_empty=0.2)
    ref = oracle.attention_backward(q, k, v, do, blk, rp, ci)
    o, lse = oracle.masked_attention(q, k, v, blk, rp, ci)
    kbar, _ = oracle.masked_attention(q, k, k, blk, rp, ci)
    term = d_term(do, o, kbar, 1 / math.sqrt(d))
    compare_gradients(ref, ref, term)
    bad = [
        (ref[0] * math.sqrt(d), ref[1], ref[2]),                       # dQ without the scale
        (ref[0], ref[2], ref[1]),                                      # dK and dV swapped
        oracle.attention_backward(q, k, v, do, blk, rp, ci, 0.2),      # another scale
    ]
    rp2, ci2, _ = _random_csr(B * H * nb, nb, 6, p_empty=0.2)
    bad.append(oracle.attention_backward(q, k, v, do, blk, rp2, ci2))  # another mask
    for g in bad:
        with pytest.raises(AssertionError):
            compare_gradients(g, ref, term)


def test_sampled_gradients_equal_the_full_ones():
    # the per-row / per-kv-block restatement used at full layer sizes
    B, H, N, d, blk = 2, 2, 90, 64, 16
    nb = -(-N // blk)
    q, k, v, do = _qkv(B, H, N, d, 23)
    rp, ci, _ = _random_csr(B * H * nb, nb, 4, p_empty=0.2)
    full = oracle.attention_backward(q, k, v, do, blk, rp, ci)
    rows = range(B * H * nb)
    dq, dkv = oracle.attention_backward_sampled(q, k, v, do, blk, rp, ci, rows, rows)
    for r in rows:
        bh, i = divmod(r, nb)
        b, h = divmod(bh, H)
        t = slice(i * blk, min(N, (i + 1) * blk))
        np.testing.assert_allclose(dq[r], full[0][b, h, t], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dkv[r][0], full[1][b, h, t], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dkv[r][1], full[2][b, h, t], rtol=0, atol=1e-12)


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def test_zero_gradient_bound_single_key():
    # one token per head: the exact dQ and dK are zero.  A kernel forming dP and
    # D as fp32 sums in different orders (sequential vs reversed) and D from an
    # Ô that is one bf16 ulp off in one element stays within the rounding bound
    # of tests/_compare.py; a dropped D term or a planted 1e-3 does not.
    from tests._compare import compare_gradients, zero_gradient_bounds
    B, H, N, d, blk = 2, 2, 1, 64, 16
    q, k, v, do = (_bf16(x) for x in _qkv(B, H, N, d, 31))
    rp, ci = _full_csr(B, H, 1)
    scale = 1 / math.sqrt(d)
    ref = oracle.attention_backward(q, k, v, do, blk, rp, ci)
    assert np.all(ref[0] == 0) and np.all(ref[1] == 0)
    o_ref, _ = oracle.masked_attention(q, k, v, blk, rp, ci)
    o_hat = o_ref.copy()
    o_hat[0, 0, 0, 3] = _bf16(o_hat[0, 0, 0, 3] * (1 + 2.0 ** -7))[()]
    prod_v = (do * v).astype(np.float32)
    prod_o = (do * o_hat).astype(np.float32)
    dp32 = np.cumsum(prod_v, axis=-1, dtype=np.float32)[..., -1]
    d32 = np.cumsum(prod_o[..., ::-1], axis=-1, dtype=np.float32)[..., -1]
    ds = _bf16(dp32 - d32)[..., None]
    got = (_bf16(scale * ds * k), _bf16(scale * ds * q), _bf16(ref[2]))
    probs = oracle.attention_probs(q, k, blk, rp, ci)
    zb = zero_gradient_bounds(q, k, v, do, o_hat, o_ref, probs, scale)
    assert np.max(np.abs(got[0])) > 0     # the emulated rounding is not zero
    compare_gradients(got, ref, None, zb)
    with pytest.raises(AssertionError):   # without the bound: exact zero demanded
        compare_gradients(got, ref, None, None)
    dropped_d = _bf16(scale * dp32[..., None] * k)
    for g in ((dropped_d, got[1], got[2]), (got[0] + 1e-3, got[1], got[2]),
              (got[0], got[1] - 1e-3, got[2])):
        with pytest.raises(AssertionError):
            compare_gradients(g, ref, None, zb)
