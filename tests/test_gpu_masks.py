"""GPU mask builders vs the fp64 oracle, through the C ABI.

pattern_mask: bit-exact CSR.  asa_build_mask: CSR equal apart from blocks inside
the 1e-5 band around each row's threshold p (see tests/_compare.py)."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_asa_b200 import workloads as W
from tests._compare import compare_masks

pytestmark = pytest.mark.gpu

# --------------------------------------------------------------------------- patterns
PATTERN_CASES = [
    # B, H, N, blk, band_w, S, f_lo, f_hi, stripe_blocks, global_frames
    (2, 6, 1000, 16, 2, 100, -2, 2, 1, 1),
    (1, 6, 777, 64, 1, 200, -1, 3, 2, 0),
    (3, 6, 130, 128, 0, 64, 0, 0, 1, 2),
    (1, 6, 4096, 32, 2, 512, -3, 3, 4, 1),
    (1, 6, 17, 16, 2, 5, -2, 2, 1, 1),           # N barely above one block
    (2, 6, 16, 16, 1, 8, -1, 1, 1, 0),           # a single block
]


@pytest.mark.parametrize("case", PATTERN_CASES)
def test_pattern_mask_bit_exact_small(cuda_lib, case):
    B, H, N, blk, w, S, f_lo, f_hi, sb, g = case
    hp = [0, 1, 2, 3, 4, 5][:H]
    rp, ci = cuda_lib.pattern_mask(hp, B, H, N, blk, w, S, f_lo, f_hi, sb, g)
    assert cuda_lib.check_device_status() == 0
    orp, oci = oracle.pattern_mask(hp, B, H, N, blk, w, S, f_lo, f_hi, sb, g)
    assert np.array_equal(rp.cpu().numpy().astype(np.int64), orp)
    assert np.array_equal(ci.cpu().numpy(), oci)


def test_pattern_mask_hunyuan_bit_exact(cuda_lib):
    w = W.HUNYUAN
    rp, ci = cuda_lib.pattern_mask(w.head_pattern, w.B, w.H, w.N, w.blk, w.band_w, w.frame_tokens,
                                   w.f_lo, w.f_hi, w.stripe_blocks, w.tile_global_frames)
    assert cuda_lib.check_device_status() == 0
    orp, oci = oracle.pattern_mask(w.head_pattern, w.B, w.H, w.N, w.blk, w.band_w, w.frame_tokens,
                                   w.f_lo, w.f_hi, w.stripe_blocks, w.tile_global_frames)
    assert np.array_equal(rp.cpu().numpy().astype(np.int64), orp)
    assert np.array_equal(ci.cpu().numpy(), oci)


def test_pattern_mask_tile3d_hand_example(cuda_lib):
    # the hand-derived 3D-tile rows of tests/golden/tile3d_example.json (frames
    # that straddle blocks), for 0, 1 and 2 global frames
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "tile3d_example.json")) as f:
        g = json.load(f)
    n, S, blk = g["N"], g["frame_tokens"], g["blk"]
    nb = -(-n // blk)
    for gf, rows in g["rows"].items():
        rp, ci = cuda_lib.pattern_mask([W.PATTERN_TILE3D], 1, 1, n, blk, 0, S, 0, 0, 0, int(gf))
        assert cuda_lib.check_device_status() == 0
        rp, ci = rp.cpu().numpy(), ci.cpu().numpy()
        assert [ci[rp[i]:rp[i + 1]].tolist() for i in range(nb)] == rows


def test_pattern_mask_wan_tile3d_bit_exact(cuda_lib):
    w = W.WAN_TILE3D
    rp, ci = cuda_lib.pattern_mask(w.head_pattern, w.B, w.H, w.N, w.blk, w.band_w, w.frame_tokens,
                                   w.f_lo, w.f_hi, w.stripe_blocks, w.tile_global_frames)
    assert cuda_lib.check_device_status() == 0
    orp, oci = oracle.pattern_mask(w.head_pattern, w.B, w.H, w.N, w.blk, w.band_w, w.frame_tokens,
                                   w.f_lo, w.f_hi, w.stripe_blocks, w.tile_global_frames)
    assert np.array_equal(rp.cpu().numpy().astype(np.int64), orp)
    assert np.array_equal(ci.cpu().numpy(), oci)


def test_pattern_mask_capacity_reported(cuda_lib):
    import ctypes
    lib = cuda_lib.load()
    hp = (ctypes.c_int32 * 2)(0, 2)
    rp = torch.empty(2 * 8 + 1, dtype=torch.int32, device="cuda")
    ci = torch.empty(4, dtype=torch.int32, device="cuda")
    nnz = ctypes.c_int64(0)
    rc = lib.pattern_mask(hp, 1, 2, 128, 16, 1, 64, 0, 0, 0, 0, ctypes.c_void_p(rp.data_ptr()),
                          ctypes.c_void_p(ci.data_ptr()), 4, ctypes.byref(nnz),
                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == cuda_lib.ERR_CAPACITY and nnz.value == 64 + 22
    # asynchronous form: the overflow shows up in the device status, nothing past capacity written
    guard = torch.full((64,), -7, dtype=torch.int32, device="cuda")
    ci2 = guard[:4]
    cuda_lib.pattern_mask_into([0, 2], 1, 2, 128, 16, 1, 64, 0, 0, 0, 0, rp, ci2)
    assert cuda_lib.check_device_status() == cuda_lib.ERR_CAPACITY
    assert torch.all(guard[4:] == -7)
    assert cuda_lib.check_device_status() == 0


# --------------------------------------------------------------------------- ASA
def _asa_case(q, k, blk, mode, topk=0, tau=0.0, ratio=0.0, diag=0, sink=0, cuda_lib=None):
    d = q.shape[-1]
    nb = -(-q.shape[2] // blk)
    rp, ci = cuda_lib.asa_build_mask(q.cuda(), k.cuda(), blk, mode, topk, tau, ratio, diag, sink)
    assert cuda_lib.check_device_status() == 0
    info = oracle.asa_mask(W.as_f64(q), W.as_f64(k), blk, mode, topk, tau, ratio, diag, sink)
    cap = oracle.asa.keep_cap(nb, ratio)
    H, B = q.shape[1], q.shape[0]

    def forced(r):
        i = r % nb
        f = list(range(min(sink, nb)))
        return f + ([i] if diag else [])

    stats = compare_masks(rp.cpu().numpy(), ci.cpu().numpy(), info, nb, mode, tau, cap, forced)
    return rp, ci, info, stats


def _rand_qk(B, H, N, d, seed, const=False):
    g = torch.Generator().manual_seed(seed)
    if const:
        q = torch.ones(B, H, N, d).to(torch.bfloat16)
        return q, q.clone()
    q = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    return q, k


ASA_SMALL = [
    # B, H, N, d, blk, mode, topk, tau, ratio, diag, sink
    (1, 2, 128, 64, 16, 0, 3, 0.0, 0.0, 1, 0),
    (2, 3, 1000, 128, 64, 1, 0, 0.5, 0.0, 0, 0),      # uncapped mass: several 64-rank chunks
    (1, 2, 5000, 64, 32, 1, 0, 0.9, 0.25, 1, 2),
    (1, 1, 300, 128, 128, 0, 9, 0.0, 0.0, 0, 0),      # topk > nb
    (2, 2, 70, 64, 16, 0, 2, 0.0, 0.0, 0, 7),         # sinks cover every block
    (1, 2, 9000, 128, 16, 1, 0, 0.3, 0.05, 0, 1),     # nb 563, ragged
    (1, 1, 20, 64, 64, 0, 1, 0.0, 0.0, 1, 0),         # N < blk
    (1, 2, 20000, 64, 16, 0, 40, 0.0, 0.0, 1, 1),     # nb 1250: shared-memory select path
    (1, 1, 20000, 128, 16, 1, 0, 0.6, 0.3, 0, 0),     # nb 1250, mass mode
    (1, 2, 16384, 64, 16, 1, 0, 0.8, 0.0, 1, 0),      # nb 1024 exactly, uncapped mass
]


@pytest.mark.parametrize("case", ASA_SMALL)
def test_asa_mask_small(cuda_lib, case):
    B, H, N, d, blk, mode, topk, tau, ratio, diag, sink = case
    q, k = _rand_qk(B, H, N, d, seed=N + d + blk)
    _asa_case(q, k, blk, mode, topk, tau, ratio, diag, sink, cuda_lib=cuda_lib)


def test_asa_mask_all_ties_lowest_index(cuda_lib):
    # constant inputs: every pooled score is equal, so ties go to the lowest indices
    q, k = _rand_qk(1, 2, 640, 64, 0, const=True)
    rp, ci, info, _ = _asa_case(q, k, 64, 0, topk=3, cuda_lib=cuda_lib)
    rows = np.split(ci.cpu().numpy(), rp.cpu().numpy()[1:-1])
    assert all(r.tolist() == [0, 1, 2] for r in rows)


def test_asa_mask_deterministic(cuda_lib):
    q, k = _rand_qk(1, 4, 4000, 128, 3)
    q, k = q.cuda(), k.cuda()
    a = cuda_lib.asa_build_mask(q, k, 64, 1, 0, 0.9, 0.1)
    b = cuda_lib.asa_build_mask(q, k, 64, 1, 0, 0.9, 0.1)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_asa_tiny_config(cuda_lib):
    w = W.TINY
    q, k, _ = W.make_qkv(w)
    _, _, _, (rows, ident, band, exempt) = _asa_case(q, k, w.blk, w.mode, w.topk, w.mass_tau,
                                                     w.max_keep_ratio, w.keep_diag,
                                                     w.n_sink_blocks, cuda_lib=cuda_lib)
    assert rows == 16


@pytest.mark.parametrize("w", [W.WAN, W.COG], ids=lambda w: w.name)
def test_asa_full_config(cuda_lib, w):
    q, k, _ = W.make_qkv(w)
    _, _, _, (rows, ident, band, exempt) = _asa_case(q, k, w.blk, w.mode, w.topk, w.mass_tau,
                                                     w.max_keep_ratio, w.keep_diag,
                                                     w.n_sink_blocks, cuda_lib=cuda_lib)
    assert ident + band + exempt == rows
    assert ident >= 0.99 * rows


@pytest.fixture(scope="module")
def wan_qk():
    q, k, _ = W.make_qkv(W.sweep(1.0, 64))
    return q, k


@pytest.mark.parametrize("keep", W.SWEEP_KEEPS)
@pytest.mark.parametrize("blk", W.SWEEP_BLKS)
def test_asa_sweep_masks(cuda_lib, wan_qk, keep, blk):
    w = W.sweep(keep, blk)
    q, k = wan_qk
    _, _, _, (rows, ident, band, exempt) = _asa_case(q, k, blk, w.mode, w.topk, cuda_lib=cuda_lib)
    assert ident + band == rows


def test_asa_capacity_overflow_reported(cuda_lib):
    q, k = _rand_qk(1, 2, 1024, 64, 5)
    q, k = q.cuda(), k.cuda()
    nb = 16
    rp = torch.empty(2 * nb + 1, dtype=torch.int32, device="cuda")
    guard = torch.full((256,), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(cuda_lib.asa_workspace_size(1, 2, 1024, 64, 64), dtype=torch.uint8,
                     device="cuda")
    cuda_lib.asa_build_mask_into(q, k, 64, 0, 4, 0.0, 0.0, 0, 0, 0.0, rp, guard[:10], ws)
    assert cuda_lib.check_device_status() == cuda_lib.ERR_CAPACITY
    assert torch.all(guard[10:] == -7)
    assert np.all(np.diff(rp.cpu().numpy()) == 4) and int(rp[0]) == 0
