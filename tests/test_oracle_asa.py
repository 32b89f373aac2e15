"""Pins of the fp64 ASA mask oracle against things other than itself.

* pooling  vs torch's avg_pool1d (ceil_mode: the last window averages its valid tokens)
* softmax  vs torch.softmax (library routine) on the pooled scores
* top-k / mass selection vs brute-force enumeration of every subset (nb = 8)
* the hand-computable worked example (tests/golden/worked_example.json)
* degenerate cases: tau = 1 and k >= nb keep every block, a head of one
  block keeps it, a single-token layer gives O = v and LSE = q.k * scale
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle.asa import MODE_MASS, MODE_TOPK, keep_cap

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("n,blk", [(128, 16), (100, 16), (7, 16), (33, 8), (64, 64)])
def test_pool_matches_avg_pool1d(n, blk):
    x = _rand((2, 3, n, 5), 11)
    got = oracle.pool(x, blk)
    t = torch.from_numpy(x).reshape(-1, n, 5).transpose(1, 2)  # [BH, d, N]
    ref = torch.nn.functional.avg_pool1d(t, blk, blk, ceil_mode=True)
    ref = ref.transpose(1, 2).reshape(2, 3, -1, 5).numpy()
    assert got.shape == ref.shape
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-13)


def test_pooled_probs_vs_library_softmax():
    q = _rand((1, 2, 50, 8), 1)
    k = _rand((1, 2, 50, 8), 2)
    p = oracle.pooled_probs(q, k, 16)
    qb = torch.nn.functional.avg_pool1d(torch.from_numpy(q)[0].transpose(1, 2), 16, 16, ceil_mode=True)
    kb = torch.nn.functional.avg_pool1d(torch.from_numpy(k)[0].transpose(1, 2), 16, 16, ceil_mode=True)
    s = torch.einsum("hdi,hdj->hij", qb, kb) / math.sqrt(8)
    ref = torch.softmax(s, dim=-1).numpy()[None]
    np.testing.assert_allclose(p, ref, rtol=0, atol=1e-14)
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-14)


def _best_subset(p, size):
    """Among all subsets of `size`, the one of largest exact sum; ties -> lexicographically smallest."""
    best, best_key = None, None
    for sub in itertools.combinations(range(len(p)), size):
        key = (-math.fsum(p[j] for j in sub), sub)
        if best_key is None or key < best_key:
            best, best_key = sub, key
    return set(best)


def _brute_mass(p, tau):
    nb = len(p)
    for size in range(1, nb + 1):
        if any(math.fsum(p[j] for j in sub) >= tau for sub in itertools.combinations(range(nb), size)):
            return size
    return nb


def _probe_rows(seed):
    rng = np.random.default_rng(seed)
    rows = [rng.dirichlet(np.ones(8)) for _ in range(12)]
    # ties: equal probabilities everywhere, and pairs of equal values at the boundary
    rows.append(np.full(8, 1 / 8))
    r = rng.dirichlet(np.ones(8))
    r[[1, 5]] = r[3]
    rows.append(r / r.sum())
    rows.append(np.array([0.3, 0.1, 0.1, 0.1, 0.1, 0.1, 0.1, 0.1]))
    return rows


@pytest.mark.parametrize("k", [1, 2, 3, 5, 8])
def test_topk_equals_brute_force(k):
    for p in _probe_rows(k):
        sel = oracle.select_row(p, 0, MODE_TOPK, topk=k)
        assert set(sel.cols) == _best_subset(p, k)


@pytest.mark.parametrize("tau", [0.1, 0.5, 0.9, 0.99])
def test_mass_equals_brute_force(tau):
    for p in _probe_rows(int(tau * 100)):
        sel = oracle.select_row(p, 0, MODE_MASS, mass_tau=tau)
        m = _brute_mass(p, tau)
        assert len(sel.cols) == m
        assert set(sel.cols) == _best_subset(p, m)
        assert math.fsum(p[j] for j in sel.cols) >= tau - 1e-12


def test_cap_and_forced_blocks():
    p = np.array([0.05, 0.4, 0.3, 0.1, 0.05, 0.05, 0.025, 0.025])
    # mass 0.9 would take 1,2,3,0 (ties 0<4<5) ... cap floor(0.25*8)=2 keeps {1,2}
    sel = oracle.select_row(p, 6, MODE_MASS, mass_tau=0.9, max_keep_ratio=0.25)
    assert sel.n_selected == 2 and sel.cols == [1, 2]
    sel = oracle.select_row(p, 6, MODE_MASS, mass_tau=0.9, max_keep_ratio=0.25, keep_diag=1, n_sink_blocks=2)
    assert sel.cols == [0, 1, 2, 6]
    assert keep_cap(512, 0.1) == 51 and keep_cap(8, 0.01) == 1 and keep_cap(9, 0.0) == 9


def _worked():
    with open(GOLDEN) as f:
        return json.load(f)


def _worked_qkv(g):
    q = np.array(g["q"], dtype=np.float64).reshape(1, 1, g["N"], 1)
    k = np.array(g["k"], dtype=np.float64).reshape(1, 1, g["N"], 1)
    v = np.array(g["v"], dtype=np.float64).reshape(1, 1, g["N"], 1)
    return q, k, v


def test_worked_example_mask():
    g = _worked()
    q, k, v = _worked_qkv(g)
    np.testing.assert_allclose(oracle.pool(q, 2)[0, 0, :, 0], g["pooled_q"], atol=0)
    np.testing.assert_allclose(oracle.pool(k, 2)[0, 0, :, 0], g["pooled_k"], atol=0)
    p = oracle.pooled_probs(q, k, 2, scale=1.0)[0, 0]
    for row, vals in g["p_rows"].items():
        np.testing.assert_allclose(p[int(row)], vals, atol=g["tol"])
    m = oracle.asa_mask(q, k, 2, MODE_TOPK, topk=2, keep_diag=1, scale=1.0)
    assert m.row_ptr.tolist() == g["top2_diag"]["row_ptr"]
    assert m.col_idx.tolist() == g["top2_diag"]["col_idx"]
    m = oracle.asa_mask(q, k, 2, MODE_MASS, mass_tau=0.9, scale=1.0)
    rows = [m.col_idx[m.row_ptr[i]:m.row_ptr[i + 1]].tolist() for i in range(4)]
    assert rows == g["mass_0.9"]["rows"]


def test_worked_example_attention():
    g = _worked()
    q, k, v = _worked_qkv(g)
    m = oracle.asa_mask(q, k, 2, MODE_TOPK, topk=2, keep_diag=1, scale=1.0)
    o, lse = oracle.masked_attention(q, k, v, 2, m.row_ptr, m.col_idx, scale=1.0)
    # the two tokens of a q-block are identical, so both rows carry the block's value
    np.testing.assert_allclose(o[0, 0, :, 0].reshape(4, 2), np.repeat(np.array(g["top2_diag"]["O_per_block"])[:, None], 2, 1), atol=g["tol"])
    np.testing.assert_allclose(lse[0, 0].reshape(4, 2), np.repeat(np.array(g["top2_diag"]["LSE_per_block"])[:, None], 2, 1), atol=g["tol"])
    # row 1 is closed-form: mean of v over kept blocks {0,1} and ln(4)
    assert o[0, 0, 2, 0] == pytest.approx(2.5, abs=1e-15)
    assert lse[0, 0, 2] == pytest.approx(math.log(4), abs=1e-15)
    full_ptr = np.arange(0, 17, 4)
    full_cols = np.tile(np.arange(4), 4).astype(np.int32)
    o, lse = oracle.masked_attention(q, k, v, 2, full_ptr, full_cols, scale=1.0)
    np.testing.assert_allclose(o[0, 0, ::2, 0], g["full"]["O_per_block"], atol=g["tol"])
    assert lse[0, 0, 2] == pytest.approx(g["full"]["LSE_row1"], abs=g["tol"])
    assert lse[0, 0, 2] == pytest.approx(math.log(8), abs=1e-15)


def test_degenerate_selections():
    rng = np.random.default_rng(4)
    for _ in range(20):
        p = rng.dirichlet(np.ones(8))
        # tau = 1 needs every block, also when the probabilities sum to just under 1
        assert oracle.select_row(p, 0, MODE_MASS, mass_tau=1.0).cols == list(range(8))
        # k at or above nb keeps every block
        for k in (8, 9, 100):
            assert oracle.select_row(p, 3, MODE_TOPK, topk=k).cols == list(range(8))
    # a single block per head (N <= blk): the only block, whatever the rule
    q, k = _rand((1, 2, 5, 4), 1), _rand((1, 2, 5, 4), 2)
    for mode, kw in ((MODE_TOPK, dict(topk=3)), (MODE_MASS, dict(mass_tau=0.5))):
        m = oracle.asa_mask(q, k, 16, mode, **kw)
        assert m.row_ptr.tolist() == [0, 1, 2] and m.col_idx.tolist() == [0, 0]


def test_single_token_layer():
    # N = 1: the pooled block is the token, the mask keeps it, O = v and
    # LSE = q.k * scale (one key: softmax weight 1)
    q, k, v = _rand((1, 1, 1, 4), 5), _rand((1, 1, 1, 4), 6), _rand((1, 1, 1, 4), 7)
    np.testing.assert_array_equal(oracle.pool(q, 16), q)
    m = oracle.asa_mask(q, k, 16, MODE_TOPK, topk=1)
    o, lse = oracle.masked_attention(q, k, v, 16, m.row_ptr, m.col_idx)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-15)
    assert abs(lse[0, 0, 0] - float((q * k).sum()) / 2.0) < 1e-15


def test_mask_comparator_exempt_rows():
    # a mass-mode row whose cut lies at tau is exempt from equality, but must
    # still be the forced blocks plus a prefix of the (p desc, j asc) order one
    # block either side of the oracle's: a row with the right count and a wrong
    # block fails tests/_compare.py
    from tests._compare import compare_masks, csr_rows
    rng = np.random.default_rng(8)
    B, H, N, d, blk = 1, 1, 128, 16, 16
    nb = N // blk
    q, k = (rng.standard_normal((B, H, N, d)) for _ in range(2))
    p = oracle.pooled_probs(q, k, blk)[0, 0, 0]
    order = np.lexsort((np.arange(nb), -p))
    tau = math.fsum(p[order[:3]].tolist())       # row 0's cut lands exactly on tau
    info = oracle.asa_mask(q, k, blk, oracle.asa.MODE_MASS, mass_tau=tau, keep_diag=1)
    assert info.n_prefix[0] == 3
    rows = csr_rows(info.row_ptr, info.col_idx)
    forced = lambda r: [r % nb]

    def check(row0):
        rs = [sorted(row0)] + rows[1:]
        rp = np.zeros(len(rs) + 1, dtype=np.int64)
        rp[1:] = np.cumsum([len(x) for x in rs])
        ci = np.asarray([c for x in rs for c in x], dtype=np.int32)
        return compare_masks(rp, ci, info, nb, 1, tau, None, forced)

    for L in (2, 3, 4):
        got = check(set(int(j) for j in order[:L]) | {0})
        assert got[3] == (0 if L == 3 else 1)
    wrong = set(int(j) for j in order[:3]) | {0}
    wrong = (wrong - {int(order[1])}) | {int(order[-1])}   # same count, wrong block
    if 0 in (int(order[1]), int(order[-1])):
        pytest.skip("seed puts the diagonal at the swapped position")
    with pytest.raises(AssertionError):
        check(wrong)
    with pytest.raises(AssertionError):
        check(set(int(j) for j in order[:6]) | {0})       # two blocks past the cut
