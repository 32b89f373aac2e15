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
(no atomics).  The autograd node and the full-layer checks are in
test_gpu_train_path.py.
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

