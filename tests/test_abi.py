"""The C-ABI library builds, loads and exports every symbol include/bsa.h
declares; host-side validation rejects bad calls before any launch (these
paths touch no GPU, so they run on CPU)."""
import ctypes

import pytest

from block_sparse_attention_asa_b200 import build, bsa


@pytest.fixture(scope="module")
def lib():
    build.build()
    return bsa.load()


def test_exports_every_header_symbol(lib):
    names = bsa.header_functions()
    assert {"asa_build_mask", "pattern_mask", "bsa_forward", "bsa_check_device_status",
            "bsa_status_string", "asa_build_mask_workspace_size", "bsa_forward_workspace_size",
            "asa_build_mask_max_nnz", "bsa_version"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code in range(-7, 1):
        assert bsa.status_string(code)
    assert bsa.status_string(12345) == "unknown status"


def test_workspace_and_capacity_sizes(lib):
    # Wan2.1-shaped layer: q̄,k̄ fp32 (2*6144*128*4) + bitmaps (6144*16*4) + the
    # select kernels' look-back state (a 256-byte ticket area, one 8-byte flag
    # per row)
    assert bsa.asa_workspace_size(1, 12, 32760, 128, 64) == (2 * 6144 * 128 * 4 + 6144 * 16 * 4 +
                                                             256 + 6144 * 8)
    assert bsa.asa_max_nnz(1, 12, 32760, 64, bsa.MODE_MASS, 0, 0.1, 0, 0) == 6144 * 51
    assert bsa.asa_max_nnz(2, 48, 17776, 64, bsa.MODE_TOPK, 33, 0.0, 0, 4) == 2 * 48 * 278 * 37
    assert bsa.asa_max_nnz(1, 2, 128, 16, bsa.MODE_TOPK, 3, 0.0, 1, 0) == 16 * 4
    assert lib.asa_build_mask_workspace_size(1, 1, 100, 96, 16) == 0  # unsupported d
    assert bsa.forward_workspace_size(1, 12, 32760, 128, 64) == 256     # the item counter
    assert lib.bsa_forward_workspace_size(1, 1, 100, 96, 16) == 0


def _asa(lib, **kw):
    a = dict(q=256, k=256, B=1, H=1, N=128, d=64, blk=16, mode=0, topk=1, tau=0.0, ratio=0.0, diag=0,
             sink=0, scale=0.0, rp=256, ci=256, cap=16, ws=256, wsb=1 << 20)
    a.update(kw)
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.asa_build_mask(vp(a["q"]), vp(a["k"]), a["B"], a["H"], a["N"], a["d"], a["blk"],
                              a["mode"], a["topk"], a["tau"], a["ratio"], a["diag"], a["sink"],
                              a["scale"], vp(a["rp"]), vp(a["ci"]), a["cap"], vp(a["ws"]), a["wsb"],
                              None)


def test_asa_validation_rejects_before_launch(lib):
    assert _asa(lib, q=None) == bsa.ERR_INVALID_ARG
    assert _asa(lib, B=0) == bsa.ERR_INVALID_ARG
    assert _asa(lib, d=96) == bsa.ERR_UNSUPPORTED
    assert _asa(lib, blk=48) == bsa.ERR_UNSUPPORTED
    assert _asa(lib, q=3) == bsa.ERR_UNSUPPORTED          # misaligned
    assert _asa(lib, mode=7) == bsa.ERR_INVALID_ARG
    assert _asa(lib, topk=0) == bsa.ERR_INVALID_ARG
    assert _asa(lib, mode=1, tau=1.5) == bsa.ERR_INVALID_ARG
    assert _asa(lib, sink=-1) == bsa.ERR_INVALID_ARG
    assert _asa(lib, ws=None) == bsa.ERR_WORKSPACE
    assert _asa(lib, wsb=16) == bsa.ERR_WORKSPACE
    assert _asa(lib, ws=272) == bsa.ERR_WORKSPACE         # not 256-aligned


def test_forward_and_pattern_validation(lib):
    vp = ctypes.c_void_p
    args = [vp(16), vp(16), vp(16), 1, 1, 128, 64, 16, vp(16), vp(16), 0.0, vp(16), None, None, 0,
            None]
    bad = list(args)
    bad[0] = None
    assert lib.bsa_forward(*bad) == bsa.ERR_INVALID_ARG
    bad = list(args)
    bad[6] = 80
    assert lib.bsa_forward(*bad) == bsa.ERR_UNSUPPORTED
    bad = list(args)
    bad[7] = 24
    assert lib.bsa_forward(*bad) == bsa.ERR_UNSUPPORTED
    bad = list(args)
    bad[1] = vp(18)
    assert lib.bsa_forward(*bad) == bsa.ERR_UNSUPPORTED
    # a workspace, when given, must hold the 4-byte item counter, 4-byte aligned
    bad = list(args)
    bad[13], bad[14] = vp(256), 2
    assert lib.bsa_forward(*bad) == bsa.ERR_WORKSPACE
    bad[13], bad[14] = vp(258), 256
    assert lib.bsa_forward(*bad) == bsa.ERR_WORKSPACE
    hp = (ctypes.c_int32 * 2)(0, 9)
    assert lib.pattern_mask(hp, 1, 2, 128, 16, 2, 64, -1, 1, 1, 0, vp(16), vp(16), 8, None,
                            None) == bsa.ERR_INVALID_ARG
    hp = (ctypes.c_int32 * 2)(0, 1)
    assert lib.pattern_mask(hp, 1, 2, 128, 16, 2, 0, -1, 1, 1, 0, vp(16), vp(16), 8, None,
                            None) == bsa.ERR_INVALID_ARG
    assert lib.pattern_mask(hp, 1, 2, 128, 16, 2, 64, 2, 1, 1, 0, vp(16), vp(16), 8, None,
                            None) == bsa.ERR_INVALID_ARG
    assert lib.pattern_mask(None, 1, 2, 128, 16, 2, 64, -1, 1, 1, 0, vp(16), vp(16), 8, None,
                            None) == bsa.ERR_INVALID_ARG


def test_search_entry_points_validate_and_select_on_host(lib):
    import numpy as np
    from oracle import search
    vp = ctypes.c_void_p
    dv = ctypes.c_double
    # host validation (nothing launched)
    assert lib.attention_head_mse(None, vp(256), 1, 1, 64, 64, vp(256), vp(256), 1024,
                                  None) == bsa.ERR_INVALID_ARG
    assert lib.attention_head_mse(vp(256), vp(256), 1, 1, 64, 96, vp(256), vp(256), 1024,
                                  None) == bsa.ERR_UNSUPPORTED
    assert lib.attention_head_mse(vp(256), vp(256), 1, 1, 64, 64, vp(256), vp(256), 8,
                                  None) == bsa.ERR_WORKSPACE
    assert lib.csr_head_sparsity(vp(256), vp(256), 1, 2, 64, 24, vp(256), vp(256), 256,
                                 None) == bsa.ERR_UNSUPPORTED
    assert lib.csr_head_sparsity(vp(256), vp(256), 1, 2, 64, 16, vp(256), None, 0,
                                 None) == bsa.ERR_WORKSPACE
    assert lib.attention_head_mse_workspace_size(1, 12, 32760, 128) == 12 * 512 * 8
    # the selection itself is host code: parity with the oracle's rule
    rng = np.random.default_rng(3)
    for trial in range(20):
        P, H = 4, 9
        mse = rng.uniform(0, 0.2, (P, H))
        sp = rng.uniform(0, 1, (P, H))
        sp[0] = 1.0
        if trial % 5 == 0:
            mse[1] = mse[2]           # exact ties
            sp[1] = sp[2]
        cand = [1, 2, 3, 4]
        lam, eps = 0.01 * (trial % 3 + 1), 0.02 * (trial % 4 + 1)
        choice, loss = bsa.search_select(mse, sp, cand, lam, eps)
        ref_l = search.search_loss(mse, sp, lam)
        np.testing.assert_allclose(loss, ref_l, rtol=0, atol=0)
        assert choice.tolist() == search.select_pattern(ref_l, cand, eps).tolist()


def test_backward_validation_and_workspace(lib):
    vp = ctypes.c_void_p
    # D (fp32 per token), rounded up to 256 bytes
    assert bsa.backward_workspace_size(1, 12, 32760, 128, 64) == -(-12 * 32760 * 4 // 256) * 256
    assert bsa.backward_workspace_size(1, 1, 10, 64, 16) == 256
    assert lib.bsa_backward_workspace_size(1, 1, 100, 96, 16) == 0
    args = [vp(256)] * 6 + [1, 1, 128, 64, 16, vp(256), vp(256), 0.0, vp(256), vp(256), vp(256),
                            vp(256), 1 << 20, None]
    for i in range(6):                       # q, k, v, o, dout, lse
        bad = list(args)
        bad[i] = None
        assert lib.bsa_backward(*bad) == bsa.ERR_INVALID_ARG, i
    for i in (11, 12, 14, 15, 16):           # row_ptr, col_idx, dq, dk, dv
        bad = list(args)
        bad[i] = None
        assert lib.bsa_backward(*bad) == bsa.ERR_INVALID_ARG, i
    bad = list(args)
    bad[9] = 80                              # d
    assert lib.bsa_backward(*bad) == bsa.ERR_UNSUPPORTED
    bad = list(args)
    bad[10] = 24                             # blk
    assert lib.bsa_backward(*bad) == bsa.ERR_UNSUPPORTED
    bad = list(args)
    bad[4] = vp(264)                         # dout misaligned
    assert lib.bsa_backward(*bad) == bsa.ERR_UNSUPPORTED
    bad = list(args)
    bad[8], bad[10] = 4097 * 16, 16          # nb over the backward's 4096
    assert lib.bsa_backward(*bad) == bsa.ERR_UNSUPPORTED
    bad = list(args)
    bad[6], bad[7], bad[8], bad[9], bad[10] = 65535, 1, 4096, 128, 128   # B*H*N*d/8 past 2^31
    assert lib.bsa_backward(*bad) == bsa.ERR_UNSUPPORTED
    bad = list(args)
    bad[13] = float("nan")
    assert lib.bsa_backward(*bad) == bsa.ERR_INVALID_ARG
    bad = list(args)
    bad[17] = None
    assert lib.bsa_backward(*bad) == bsa.ERR_WORKSPACE
    bad = list(args)
    bad[18] = 16
    assert lib.bsa_backward(*bad) == bsa.ERR_WORKSPACE
    bad = list(args)
    bad[17] = vp(272)
    assert lib.bsa_backward(*bad) == bsa.ERR_WORKSPACE


def test_wait_timeout_diagnostic_validation(lib):
    vp = ctypes.c_void_p
    assert lib.bsa_debug_wait_timeout(10_000_000_001, 0, None, None) == bsa.ERR_INVALID_ARG
    assert lib.bsa_debug_wait_timeout(1000, 0, vp(260), None) == bsa.ERR_UNSUPPORTED


def test_host_csr_validator(lib):
    import numpy as np
    # valid: empty row, full row, ragged
    rp = np.array([0, 0, 3, 5], dtype=np.int32)
    ci = np.array([0, 1, 2, 1, 2], dtype=np.int32)
    assert bsa.validate_csr(rp, ci, 3) == -1
    assert bsa.validate_csr(np.zeros(4, dtype=np.int32), np.zeros(0, dtype=np.int32), 3) == -1
    bad_cases = [
        (np.array([1, 1, 3, 5]), ci, 0),                 # row_ptr[0] != 0
        (np.array([0, 3, 2, 5]), ci, 1),                 # decreasing row_ptr
        (np.array([0, 0, 3, 6]), ci, 2),                 # past the end of col_idx
        (rp, np.array([0, 1, 3, 1, 2]), 1),              # id >= nb
        (rp, np.array([0, 1, 2, -1, 2]), 2),             # negative id
        (rp, np.array([0, 2, 1, 1, 2]), 1),              # descending inside a row
        (rp, np.array([0, 1, 2, 2, 2]), 2),              # duplicate
    ]
    for rpb, cib, row in bad_cases:
        assert bsa.validate_csr(np.asarray(rpb, np.int32), np.asarray(cib, np.int32), 3) == row
    vp = ctypes.c_void_p
    assert lib.bsa_validate_csr_host(None, None, 1, 3, 0, None) == bsa.ERR_INVALID_ARG
    assert lib.bsa_validate_csr_host(vp(16), None, 1, 3, 5, None) == bsa.ERR_INVALID_ARG


def test_oracle_masks_pass_the_validator(lib):
    # the oracle's ASA and pattern masks follow the conventions the kernels rely on
    import numpy as np
    import oracle
    from block_sparse_attention_asa_b200 import workloads as W
    w = W.TINY
    q, k, _ = W.make_qkv(w)
    info = oracle.asa_mask(W.as_f64(q), W.as_f64(k), w.blk, w.mode, w.topk, w.mass_tau,
                           w.max_keep_ratio, w.keep_diag, w.n_sink_blocks)
    assert bsa.validate_csr(info.row_ptr.astype(np.int32), info.col_idx, w.nb) == -1
    rp, ci = oracle.pattern_mask([0, 1, 2, 3, 4, 5], 1, 6, 300, 16, 2, 64, -1, 1, 1, 1)
    assert bsa.validate_csr(np.asarray(rp, np.int32), np.asarray(ci, np.int32), 19) == -1


def test_binding_signatures_match_the_header():
    # every function the header declares has a ctypes signature in the binding,
    # with as many arguments as the declaration has parameters
    import re
    with open(bsa.HEADER) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    decls = re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(([^;{}]*?)\)\s*;", text)
    assert decls
    for name, params in decls:
        params = " ".join(params.split())
        n = 0 if params in ("", "void") else params.count(",") + 1
        assert name in bsa._SIGNATURES, f"{name} has no binding signature"
        assert len(bsa._SIGNATURES[name][1]) == n, (name, n, len(bsa._SIGNATURES[name][1]))
    assert {n for n, _ in decls} == set(bsa._SIGNATURES)
