"""The training path end to end, through the C ABI: the binding's autograd node
and the backward on the bench's full layers.

* block_sparse_attention (one autograd node over bsa_forward / bsa_backward)
  returns exactly the kernels' O and gradients (the residual path);
* with the forward's rounding residual, D comes from the fp32 O and dQ meets
  the plain gradient bounds, with no term for O's bf16 rounding, on the
  PE-structured tiny layer where that term dominated; the residual is at most
  half an ulp of o;
* on the Wan and Cog layers (GPU mask -> forward -> backward), 16 random
  q-blocks plus the last (dQ) and 16 random kv-blocks plus the first and last
  (dK, dV) match the oracle's per-block restatement
  (oracle.attention_backward_sampled) within the gradient bounds of
  tests/_compare.py, the dQ term for the rounding of O included;
* sequences of 1 to 17 tokens (one partial block per head) through mask,
  forward and backward.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_asa_b200 import workloads as W
from tests._compare import compare_gradients, d_term, zero_gradient_bounds
from tests.test_gpu_backward import _csr

pytestmark = pytest.mark.gpu


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
    o2, lse, res = cuda_lib.bsa_forward(q, k, v, blk, rpd, cid, residual=True)
    dq, dk, dv = cuda_lib.bsa_backward(q, k, v, o2, do, lse, blk, rpd, cid, o_residual=res)
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


@pytest.mark.parametrize("N,d,blk", [(1, 64, 16), (1, 128, 64), (3, 128, 128), (17, 64, 16)])
def test_tiny_sequences_end_to_end(cuda_lib, N, d, blk):
    # one or a few tokens: a single (partial) block per head, the 128-row
    # tiles mostly past N; mask -> forward -> backward against the oracle
    B, H = 2, 2
    g = torch.Generator().manual_seed(N * 1000 + d + blk)
    q, k, v, do = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(4))
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    rp, ci = cuda_lib.asa_build_mask(qd, kd, blk, cuda_lib.MODE_TOPK, topk=2, keep_diag=1)
    o, lse = cuda_lib.bsa_forward(qd, kd, vd, blk, rp, ci)
    dq, dk, dv = cuda_lib.bsa_backward(qd, kd, vd, o, dod, lse, blk, rp, ci)
    assert cuda_lib.check_device_status() == 0
    rp_h, ci_h = rp.cpu().numpy().astype(np.int64), ci.cpu().numpy()
    nb = -(-N // blk)
    assert rp_h.tolist() == [min(2, nb) * r for r in range(B * H * nb + 1)]
    qf, kf, vf, dof = W.as_f64(q), W.as_f64(k), W.as_f64(v), W.as_f64(do)
    o_ref, l_ref = oracle.masked_attention(qf, kf, vf, blk, rp_h, ci_h)
    from tests._compare import compare_attention
    compare_attention(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)
    ref = oracle.attention_backward(qf, kf, vf, dof, blk, rp_h, ci_h)
    kbar, _ = oracle.masked_attention(qf, kf, kf, blk, rp_h, ci_h)
    oh = W.as_f64(o.cpu())
    term = d_term(dof, oh, kbar, 1.0 / np.sqrt(d))
    # with one token every row has a single live key and the exact dQ and dK are
    # zero; the kernels' values there are bounded by the rounding of dP - D
    probs = oracle.attention_probs(qf, kf, blk, rp_h, ci_h)
    zb = zero_gradient_bounds(qf, kf, vf, dof, oh, o_ref, probs, 1.0 / np.sqrt(d))
    compare_gradients([x.float().cpu().numpy() for x in (dq, dk, dv)], ref, term, zb)


@pytest.mark.parametrize("w", [W.TINY, W.COG], ids=lambda w: w.name)
def test_residual_backward_meets_plain_bounds(cuda_lib, w):
    # bsa_forward_residual / bsa_backward_residual: dQ within rel-RMS 1e-2 and
    # max 2e-2 of max|ref| with no allowance for O's rounding (R20); on the
    # Cog layer a few sampled heads keep the oracle fast
    q, k, v = W.make_qkv(w)
    if w is W.COG:
        q, k, v = (t[:1, :2].contiguous() for t in (q, k, v))
    B, H, N, d = q.shape
    g = torch.Generator().manual_seed(1234)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    rp, ci = cuda_lib.asa_build_mask(qd, kd, w.blk, w.mode, w.topk, w.mass_tau, w.max_keep_ratio,
                                     w.keep_diag, w.n_sink_blocks)
    o, lse, res = cuda_lib.bsa_forward(qd, kd, vd, w.blk, rp, ci, residual=True)
    dq, dk, dv = cuda_lib.bsa_backward(qd, kd, vd, o, dod, lse, w.blk, rp, ci, o_residual=res)
    assert cuda_lib.check_device_status() == 0
    # the residual is at most half an ulp of o (2^-8 |o|), up to its own bf16
    # rounding
    assert torch.all(res.float().abs() <= o.float().abs() * (2.0 ** -8) * (1 + 2.0 ** -7))
    rp_h, ci_h = rp.cpu().numpy().astype(np.int64), ci.cpu().numpy()
    qf, kf, vf, dof = W.as_f64(q), W.as_f64(k), W.as_f64(v), W.as_f64(do)
    ref = oracle.attention_backward(qf, kf, vf, dof, w.blk, rp_h, ci_h)
    rel = compare_gradients([x.float().cpu().numpy() for x in (dq, dk, dv)], ref, None)
    assert rel[0][0] <= 1e-2
