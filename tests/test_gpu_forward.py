"""bsa_forward (tcgen05) vs the fp64 oracle, through the C ABI.

The oracle is fed the CSR the GPU used (its own mask builder's output for the
layer configs), which keeps forward parity independent of mask-band ties.
Tolerances (tests/_compare.py): O max-abs 2e-2 and rel-RMS 1e-2, LSE 1e-3."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_asa_b200 import workloads as W
from tests._compare import compare_attention

pytestmark = pytest.mark.gpu


def _random_csr(rows, nb, seed, p_empty=0.15, p_full=0.1, max_keep=None):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(rows):
        u = rng.random()
        if u < p_empty:
            out.append([])
        elif u < p_empty + p_full:
            out.append(list(range(nb)))
        else:
            hi = nb if max_keep is None else min(nb, max_keep)
            out.append(sorted(rng.choice(nb, size=int(rng.integers(1, hi + 1)), replace=False).tolist()))
    rp = np.zeros(rows + 1, dtype=np.int32)
    rp[1:] = np.cumsum([len(c) for c in out])
    ci = np.asarray([c for cols in out for c in cols] or [0], dtype=np.int32)
    return rp, ci


def _run_and_compare(cuda_lib, q, k, v, blk, rp, ci, rows=None, scale=0.0):
    B, H, N, d = q.shape
    nb = -(-N // blk)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    rpd = torch.as_tensor(np.asarray(rp, dtype=np.int32)).cuda()
    cid = torch.as_tensor(np.asarray(ci, dtype=np.int32)).cuda()
    o, lse = cuda_lib.bsa_forward(qd, kd, vd, blk, rpd, cid, softmax_scale=scale)
    assert cuda_lib.check_device_status() == 0
    og = o.float().cpu().numpy()
    lg = lse.cpu().numpy()
    qf, kf, vf = W.as_f64(q), W.as_f64(k), W.as_f64(v)
    rp64 = np.asarray(rp, dtype=np.int64)
    sc = None if scale <= 0 else scale
    if rows is None:
        o_ref, l_ref = oracle.masked_attention(qf, kf, vf, blk, rp64, ci, sc)
        return compare_attention(og, lg, o_ref, l_ref)
    res = oracle.attention_rows(qf, kf, vf, blk, rp64, ci, rows, sc)
    got_o, got_l, ref_o, ref_l = [], [], [], []
    for r, (orow, lrow) in res.items():
        i, bh = r % nb, r // nb
        b, h = bh // H, bh % H
        t0, t1 = i * blk, min(N, (i + 1) * blk)
        got_o.append(og[b, h, t0:t1])
        got_l.append(lg[b, h, t0:t1])
        ref_o.append(orow)
        ref_l.append(lrow)
    return compare_attention(np.concatenate(got_o), np.concatenate(got_l), np.concatenate(ref_o),
                             np.concatenate(ref_l))


FWD_CASES = [
    # B, H, N, d, blk
    (1, 2, 128, 64, 16),
    (1, 2, 1000, 128, 64),     # ragged tail, partial q-tile
    (2, 3, 700, 64, 32),
    (1, 2, 2049, 128, 128),
    (1, 1, 77, 128, 16),       # N below one q-tile
    (2, 2, 1536, 64, 64),
    (1, 3, 3000, 128, 16),     # many slots per step, long unions
]


@pytest.mark.parametrize("case", FWD_CASES)
def test_forward_random_csr(cuda_lib, case):
    B, H, N, d, blk = case
    g = torch.Generator().manual_seed(N * d + blk)
    q, k, v = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
    nb = -(-N // blk)
    rp, ci = _random_csr(B * H * nb, nb, seed=N + blk)
    _run_and_compare(cuda_lib, q, k, v, blk, rp, ci)


def test_forward_all_empty_rows(cuda_lib):
    q = torch.randn(1, 2, 300, 64).to(torch.bfloat16)
    nb = -(-300 // 64)
    rp = np.zeros(2 * nb + 1, dtype=np.int32)
    o, lse = cuda_lib.bsa_forward(q.cuda(), q.cuda(), q.cuda(), 64, torch.as_tensor(rp).cuda(),
                                  torch.zeros(1, dtype=torch.int32, device="cuda"))
    assert cuda_lib.check_device_status() == 0
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_forward_large_logits_and_scale(cuda_lib):
    # scores spanning a wide range exercise the running-max rescale path
    g = torch.Generator().manual_seed(7)
    q = (torch.randn(1, 2, 1024, 128, generator=g) * 4).to(torch.bfloat16)
    k = (torch.randn(1, 2, 1024, 128, generator=g) * 4).to(torch.bfloat16)
    v = torch.randn(1, 2, 1024, 128, generator=g).to(torch.bfloat16)
    nb = 16
    rp, ci = _random_csr(2 * nb, nb, seed=3, p_empty=0.0, p_full=0.5)
    _run_and_compare(cuda_lib, q, k, v, 64, rp, ci, scale=0.05)


def test_forward_bad_csr_index_flagged(cuda_lib):
    q = torch.randn(1, 1, 256, 64).to(torch.bfloat16).cuda()
    rp = torch.tensor([0, 2, 2, 2, 2], dtype=torch.int32, device="cuda")
    ci = torch.tensor([0, 99], dtype=torch.int32, device="cuda")
    cuda_lib.bsa_forward(q, q, q, 64, rp, ci)
    assert cuda_lib.check_device_status() == cuda_lib.ERR_CSR
    assert cuda_lib.check_device_status() == 0


def test_forward_tiny_config_end_to_end(cuda_lib):
    w = W.TINY
    q, k, v = W.make_qkv(w)
    rp, ci = cuda_lib.asa_build_mask(q.cuda(), k.cuda(), w.blk, w.mode, w.topk, w.mass_tau,
                                     w.max_keep_ratio, w.keep_diag, w.n_sink_blocks)
    _run_and_compare(cuda_lib, q, k, v, w.blk, rp.cpu().numpy(), ci.cpu().numpy())


@pytest.mark.parametrize("w", [W.WAN, W.COG], ids=lambda w: w.name)
def test_forward_full_config(cuda_lib, w):
    q, k, v = W.make_qkv(w)
    rp, ci = cuda_lib.asa_build_mask(q.cuda(), k.cuda(), w.blk, w.mode, w.topk, w.mass_tau,
                                     w.max_keep_ratio, w.keep_diag, w.n_sink_blocks)
    _run_and_compare(cuda_lib, q, k, v, w.blk, rp.cpu().numpy(), ci.cpu().numpy())


def test_forward_hunyuan_patterns_sampled(cuda_lib):
    w = W.HUNYUAN
    q, k, v = W.make_qkv(w)
    rp, ci = cuda_lib.pattern_mask(w.head_pattern, w.B, w.H, w.N, w.blk, w.band_w, w.frame_tokens,
                                   w.f_lo, w.f_hi, w.stripe_blocks, w.tile_global_frames)
    rng = np.random.default_rng(11)
    rows = []
    for h, pid in enumerate(w.head_pattern):
        n = 12 if pid == W.PATTERN_FULL else 48
        picks = rng.choice(w.nb, size=n, replace=False).tolist() + [0, w.nb - 1]
        rows += [h * w.nb + i for i in sorted(set(picks))]
    _run_and_compare(cuda_lib, q, k, v, w.blk, rp.cpu().numpy(), ci.cpu().numpy(), rows=rows)


def test_forward_wan_tile3d_sampled(cuda_lib):
    # the 3D-tile layer: every head keeps its own frames' blocks and frame 0's
    w = W.WAN_TILE3D
    q, k, v = W.make_qkv(w)
    rp, ci = cuda_lib.pattern_mask(w.head_pattern, w.B, w.H, w.N, w.blk, w.band_w, w.frame_tokens,
                                   w.f_lo, w.f_hi, w.stripe_blocks, w.tile_global_frames)
    rng = np.random.default_rng(13)
    rows = sorted(set(rng.choice(w.H * w.nb, size=96, replace=False).tolist() + [0, w.nb - 1]))
    _run_and_compare(cuda_lib, q, k, v, w.blk, rp.cpu().numpy(), ci.cpu().numpy(), rows=rows)


@pytest.mark.parametrize("keep", [1.0, 0.1])
@pytest.mark.parametrize("blk", W.SWEEP_BLKS)
def test_forward_sweep_sampled(cuda_lib, keep, blk):
    w = W.sweep(keep, blk)
    q, k, v = W.make_qkv(w)
    rp, ci = cuda_lib.asa_build_mask(q.cuda(), k.cuda(), blk, w.mode, w.topk)
    rng = np.random.default_rng(5)
    rows = sorted(set(rng.choice(w.H * w.nb, size=96, replace=False).tolist() + [w.nb - 1]))
    _run_and_compare(cuda_lib, q, k, v, blk, rp.cpu().numpy(), ci.cpu().numpy(), rows=rows)


def test_exp2_polynomial_against_cuda_exp2(cuda_lib):
    # the softmax's FMA-pipe exponential vs CUDA's exp2f (torch.exp2 on the GPU)
    x = torch.cat([torch.linspace(-125.0, 126.0, 2_000_001), torch.linspace(-1, 1, 100_001),
                   torch.tensor([0.0, -0.5, 0.5, 8.0, -125.0])]).cuda()
    y = cuda_lib.debug_exp2_poly(x)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel < 1e-4, rel
    # below the clamp the result is tiny and non-negative (not exactly zero)
    z = cuda_lib.debug_exp2_poly(torch.tensor([-125.5, -126.0, -200.0, -1000.0], device="cuda"))
    assert torch.all(z >= 0) and torch.all(z < 2.0 ** -124)


@pytest.mark.parametrize("blk,d", [(128, 128), (64, 128), (16, 64)])
def test_forward_repeatable_under_load(cuda_lib, blk, d):
    # many empty rows (items without work), single-slot tails, back-to-back
    # launches: every launch must finish cleanly and give bit-identical output
    g = torch.Generator().manual_seed(blk + d)
    N = 5000
    q, k, v = (torch.randn(2, 3, N, d, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    nb = -(-N // blk)
    rp, ci = _random_csr(2 * 3 * nb, nb, seed=blk * 7 + d, p_empty=0.4, p_full=0.05)
    rpd, cid = torch.as_tensor(rp).cuda(), torch.as_tensor(ci).cuda()
    o0, l0 = cuda_lib.bsa_forward(q, k, v, blk, rpd, cid)
    assert cuda_lib.check_device_status() == 0
    for _ in range(20):
        o1, l1 = cuda_lib.bsa_forward(q, k, v, blk, rpd, cid)
        assert cuda_lib.check_device_status() == 0
        assert torch.equal(o0, o1) and torch.equal(l0, l1)


@pytest.mark.parametrize("blk", [64, 16])
def test_forward_dense_rows_longer_than_a_list_segment(cuda_lib, blk):
    # every row lists every block: the union of a tile runs over several of the
    # kernel's list segments (512 blocks each), including an exactly full one
    N = 64 * 1100 if blk == 64 else 16 * 1024
    g = torch.Generator().manual_seed(blk)
    q, k, v = (torch.randn(1, 1, N, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    nb = -(-N // blk)
    rp = (np.arange(nb + 1) * nb).astype(np.int32)
    ci = np.tile(np.arange(nb, dtype=np.int32), nb)
    rows = [0, 1, nb // 2, nb - 2, nb - 1]
    _run_and_compare(cuda_lib, q, k, v, blk, rp, ci, rows=rows)


def test_forward_item_order_does_not_change_results(cuda_lib):
    # with a workspace the CTAs take items from a counter (dynamic order);
    # without one the items are dealt round-robin: outputs must be identical
    g = torch.Generator().manual_seed(77)
    N, d, blk = 9000, 128, 64
    q, k, v = (torch.randn(1, 4, N, d, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    nb = -(-N // blk)
    rp, ci = _random_csr(4 * nb, nb, seed=78, p_empty=0.1, p_full=0.05)
    rpd, cid = torch.as_tensor(rp).cuda(), torch.as_tensor(ci).cuda()
    o_dyn, l_dyn = cuda_lib.bsa_forward(q, k, v, blk, rpd, cid)
    o_st, l_st = torch.empty_like(o_dyn), torch.empty_like(l_dyn)
    cuda_lib.bsa_forward_into(q, k, v, blk, rpd, cid, o_st, l_st, workspace=None)
    assert cuda_lib.check_device_status() == 0
    assert torch.equal(o_dyn, o_st) and torch.equal(l_dyn, l_st)


def test_forward_back_to_back_layers_finish_cleanly(cuda_lib):
    # The CogVideoX-shaped layer (d 64: 4-deep K/V rings) run as the bench runs
    # it, mask then forward, many times: every launch must finish with no
    # device-side wait giving up (a producer that blocked on a Q buffer while
    # its own V front owed the data that frees it once timed out here).
    w = W.COG
    q, k, v = (t.cuda() for t in W.make_qkv(w))
    B, H, N, d = q.shape
    cap = cuda_lib.asa_max_nnz(B, H, N, w.blk, w.mode, w.topk, w.max_keep_ratio, w.keep_diag,
                               w.n_sink_blocks)
    rp = torch.empty(B * H * w.nb + 1, dtype=torch.int32, device="cuda")
    ci = torch.empty(cap, dtype=torch.int32, device="cuda")
    ws = torch.empty(cuda_lib.asa_workspace_size(B, H, N, d, w.blk), dtype=torch.uint8,
                     device="cuda")
    fws = torch.empty(cuda_lib.forward_workspace_size(B, H, N, d, w.blk), dtype=torch.uint8,
                      device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    ref = None
    for it in range(60):
        cuda_lib.asa_build_mask_into(q, k, w.blk, w.mode, w.topk, w.mass_tau, w.max_keep_ratio,
                                     w.keep_diag, w.n_sink_blocks, 0.0, rp, ci, ws)
        cuda_lib.bsa_forward_into(q, k, v, w.blk, rp, ci, o, lse, workspace=fws)
        assert cuda_lib.check_device_status() == 0, f"iteration {it}"
        if ref is None:
            ref = o.clone()
        elif it % 10 == 0:
            assert torch.equal(o, ref)
