"""bsa_backward (tcgen05) vs the fp64 gradient oracle, through the C ABI.

O and LSE come from the GPU forward on the same inputs and mask; dO is seeded
bf16.  The oracle differentiates the forward definition in fp64 on the same
bf16-valued q, k, v, dO.  Bounds (tests/_compare.py, compare_gradients): per
gradient rel-RMS <= 1e-2 and max|err| <= 2e-2 * max|ref|, plus, for dQ, the
error that the bf16 rounding of O allows through D = dO . O.  An emulation of
the kernel's arithmetic (P and dS rounded to bf16 before their products, D
from the bf16 O, fp32 sums, bf16 outputs) lands at about 2.4e-3 rel-RMS and
5e-3 max on these cases.  Tokens whose row lists nothing get dQ exactly 0; key
tokens no row reaches get dK and dV exactly 0.  Two runs give identical bits
(no atomics).  The autograd node of the binding (block_sparse_attention)
returns exactly the kernels' O and gradients.  On the bench's Wan and Cog
layers (GPU mask -> forward -> backward) sampled q-blocks and kv-blocks are
checked against the oracle's per-block restatement with the same bounds.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_asa_b200 import workloads as W
from tests._compare import compare_gradients, d_term

pytestmark = pytest.mark.gpu


def _csr(rows, nb, seed, p_empty=0.15, p_full=0.1):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(rows):
        u = rng.random()
        if u < p_empty:
            out.append([])
        elif u < p_empty + p_full:
            out.append(list(range(nb)))
        else:
            out.append(sorted(rng.choice(nb, size=int(rng.integers(1, nb + 1)), replace=False).tolist()))
    rp = np.zeros(rows + 1, dtype=np.int32)
    rp[1:] = np.cumsum([len(c) for c in out])
    ci = np.asarray([c for cols in out for c in cols] or [0], dtype=np.int32)
    return rp, ci, out


def _run(cuda_lib, B, H, N, d, blk, rp, ci, seed, scale=0.0):
    g = torch.Generator().manual_seed(seed)
    q, k, v, do = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(4))
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    rpd = torch.as_tensor(rp).cuda()
    cid = torch.as_tensor(ci).cuda()
    o, lse = cuda_lib.bsa_forward(qd, kd, vd, blk, rpd, cid, softmax_scale=scale)
    grads = cuda_lib.bsa_backward(qd, kd, vd, o, dod, lse, blk, rpd, cid, softmax_scale=scale)
    assert cuda_lib.check_device_status() == 0
    got = [x.float().cpu().numpy().astype(np.float64) for x in grads]
    qf, kf, vf, dof = W.as_f64(q), W.as_f64(k), W.as_f64(v), W.as_f64(do)
    rp64 = np.asarray(rp, dtype=np.int64)
    sc = None if scale <= 0 else scale
    ref = oracle.attention_backward(qf, kf, vf, dof, blk, rp64, ci, sc)
    kbar, _ = oracle.masked_attention(qf, kf, kf, blk, rp64, ci, sc)
    term = d_term(dof, W.as_f64(o.cpu()), kbar, sc if sc else 1.0 / np.sqrt(d))
    return got, ref, term, (qd, kd, vd, o, dod, lse, rpd, cid)


def _compare(got, ref, term):
    compare_gradients(got, ref, term)


def _exact_zeros(got, rows, B, H, N, blk):
    nb = -(-N // blk)
    dq, dk, dv = got
    reached = np.zeros((B * H, nb), dtype=bool)
    for r, cols in enumerate(rows):
        bh, i = divmod(r, nb)
        reached[bh, cols] = True
        if not cols:
            assert np.all(dq[bh // H, bh % H, i * blk:min(N, (i + 1) * blk)] == 0.0)
    for bh in range(B * H):
        for j in np.flatnonzero(~reached[bh]):
            toks = slice(j * blk, min(N, (j + 1) * blk))
            assert np.all(dk[bh // H, bh % H, toks] == 0.0) and np.all(dv[bh // H, bh % H, toks] == 0.0)


@pytest.mark.parametrize("B,H,N,d,blk,seed", [
    (1, 2, 200, 64, 16, 0),      # ragged tail, 8 blocks per tile
    (2, 2, 333, 128, 64, 1),     # two q-blocks per tile, B = 2
    (1, 2, 300, 128, 128, 2),    # one block per tile
    (1, 3, 260, 64, 32, 3),
    (1, 2, 1000, 128, 64, 4),    # several steps per item
])
def test_backward_matches_oracle(cuda_lib, B, H, N, d, blk, seed):
    nb = -(-N // blk)
    rp, ci, rows = _csr(B * H * nb, nb, seed + 7)
    got, ref, term, _ = _run(cuda_lib, B, H, N, d, blk, rp, ci, seed)
    _compare(got, ref, term)
    _exact_zeros(got, rows, B, H, N, blk)


def test_backward_custom_scale_and_keep_all(cuda_lib):
    B, H, N, d, blk = 1, 2, 256, 128, 64
    nb = N // blk
    rows = B * H * nb
    rp = (np.arange(rows + 1) * nb).astype(np.int32)
    ci = np.tile(np.arange(nb, dtype=np.int32), rows)
    got, ref, term, _ = _run(cuda_lib, B, H, N, d, blk, rp, ci, 5, scale=0.05)
    _compare(got, ref, term)


def test_backward_empty_mask_gives_zeros(cuda_lib):
    B, H, N, d, blk = 1, 2, 130, 64, 64
    nb = -(-N // blk)
    rp = np.zeros(B * H * nb + 1, dtype=np.int32)
    ci = np.zeros(1, dtype=np.int32)
    got, ref, _, _ = _run(cuda_lib, B, H, N, d, blk, rp, ci, 6)
    for g in got:
        assert np.all(g == 0.0)


def test_backward_is_deterministic(cuda_lib):
    B, H, N, d, blk = 1, 2, 700, 64, 64
    nb = -(-N // blk)
    rp, ci, _ = _csr(B * H * nb, nb, 31)
    _, _, _, (qd, kd, vd, o, dod, lse, rpd, cid) = _run(cuda_lib, B, H, N, d, blk, rp, ci, 8)
    a = cuda_lib.bsa_backward(qd, kd, vd, o, dod, lse, blk, rpd, cid)
    b = cuda_lib.bsa_backward(qd, kd, vd, o, dod, lse, blk, rpd, cid)
    assert cuda_lib.check_device_status() == 0
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_autograd_node_returns_the_kernels_gradients(cuda_lib):
    B, H, N, d, blk = 1, 2, 300, 64, 64
    nb = -(-N // blk)
    rp, ci, _ = _csr(B * H * nb, nb, 41)
    g = torch.Generator().manual_seed(9)
    q, k, v, do = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16).cuda() for _ in range(4))
    rpd, cid = torch.as_tensor(rp).cuda(), torch.as_tensor(ci).cuda()
    qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
    o = cuda_lib.block_sparse_attention(qa, ka, va, blk, rpd, cid)
    o.backward(do)
    o2, lse = cuda_lib.bsa_forward(q, k, v, blk, rpd, cid)
    dq, dk, dv = cuda_lib.bsa_backward(q, k, v, o2, do, lse, blk, rpd, cid)
    assert cuda_lib.check_device_status() == 0
    assert torch.equal(o.detach(), o2)
    for got, want in ((qa.grad, dq), (ka.grad, dk), (va.grad, dv)):
        assert got.dtype == torch.bfloat16 and torch.equal(got, want)


@pytest.mark.parametrize("w", [W.WAN, W.COG], ids=lambda w: w.name)
def test_backward_full_config_sampled(cuda_lib, w):
    # the bench's layers end to end (GPU mask -> forward -> backward), checked
    # on 16+ sampled q-blocks (dQ) and 16+ sampled kv-blocks (dK, dV)
    q, k, v = W.make_qkv(w)
    g = torch.Generator().manual_seed(77)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    rp, ci = cuda_lib.asa_build_mask(qd, kd, w.blk, w.mode, w.topk, w.mass_tau, w.max_keep_ratio,
                                     w.keep_diag, w.n_sink_blocks)
    o, lse = cuda_lib.bsa_forward(qd, kd, vd, w.blk, rp, ci)
    dq, dk, dv = cuda_lib.bsa_backward(qd, kd, vd, o, dod, lse, w.blk, rp, ci)
    assert cuda_lib.check_device_status() == 0
    B, H, N, d = q.shape
    nb, blk = w.nb, w.blk
    rp_h, ci_h = rp.cpu().numpy().astype(np.int64), ci.cpu().numpy()
    rng = np.random.default_rng(19)
    rows = sorted(set(rng.choice(B * H * nb, size=16, replace=False).tolist() + [nb - 1]))
    cols = sorted(set(rng.choice(B * H * nb, size=16, replace=False).tolist() + [0, nb - 1]))
    qf, kf, vf, dof = W.as_f64(q), W.as_f64(k), W.as_f64(v), W.as_f64(do)
    ref_dq, ref_dkv = oracle.attention_backward_sampled(qf, kf, vf, dof, blk, rp_h, ci_h, rows,
                                                        cols)
    kbar = oracle.attention_rows(qf, kf, kf, blk, rp_h, ci_h, rows)
    dqh, dkh, dvh = (x.float().cpu().numpy() for x in (dq, dk, dv))
    oh = o.float().cpu().numpy()
    got, ref, term = ([], [], []), ([], [], []), []
    for r in rows:
        bh, i = divmod(r, nb)
        b, h = divmod(bh, H)
        t = slice(i * blk, min(N, (i + 1) * blk))
        got[0].append(dqh[b, h, t])
        ref[0].append(ref_dq[r])
        term.append(d_term(dof[b, h, t], oh[b, h, t], kbar[r][0], 1.0 / np.sqrt(d)))
    for c in cols:
        bh, j = divmod(c, nb)
        b, h = divmod(bh, H)
        t = slice(j * blk, min(N, (j + 1) * blk))
        got[1].append(dkh[b, h, t])
        got[2].append(dvh[b, h, t])
        ref[1].append(ref_dkv[c][0])
        ref[2].append(ref_dkv[c][1])
    compare_gradients([np.concatenate(x) for x in got], [np.concatenate(x) for x in ref],
                      np.concatenate(term))
