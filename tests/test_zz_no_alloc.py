"""asa_build_mask_noalloc: the ASA mask for callers that may not allocate device
memory (a host framework that owns all GPU memory, or a path that cannot take an
allocation's implicit synchronization).  It uses the library's fixed scratch
array instead of a caller workspace.  Checked through the C ABI against the
workspace entry point (asa_build_mask) on two calls in a row -- with different
shapes, so contents left in the shared array by the first call cannot leak into
the second -- and for the rejection of shapes whose scratch exceeds the array.
The masks are compared exactly: both entry points run the same kernels, which
are deterministic, so the mask tolerance (the 1e-5 band around the cut) is not
needed here.  This file is collected last on purpose."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

MAX_BYTES = 16 << 20


def _noalloc(lib, bsa, q, k, blk, mode, topk, tau, ratio, diag, sink, row_ptr, col_idx):
    B, H, N, d = q.shape
    return lib.asa_build_mask_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), B, H, N, d, blk, mode, topk,
        tau, ratio, diag, sink, 0.0, ctypes.c_void_p(row_ptr.data_ptr()),
        ctypes.c_void_p(col_idx.data_ptr()), col_idx.numel(),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


CASES = [
    # B, H, N, d, blk, mode, topk, tau, ratio, diag, sink -- two different shapes, in this order
    (1, 12, 32760, 128, 64, 1, 0, 0.9, 0.1, 0, 0),   # Wan2.1-shaped layer, mass 0.9 cap 0.1
    (2, 8, 17776, 64, 64, 0, 33, 0.0, 0.0, 1, 4),    # CogVideoX-shaped, top-k + sinks + diag
]


def test_noalloc_matches_workspace_entry_point_twice_in_a_row(cuda_lib):
    lib = cuda_lib.load()
    g = torch.Generator().manual_seed(2024)
    for B, H, N, d, blk, mode, topk, tau, ratio, diag, sink in CASES:
        assert cuda_lib.asa_workspace_size(B, H, N, d, blk) <= MAX_BYTES
        q = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16).cuda()
        k = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16).cuda()
        ref_rp, ref_ci = cuda_lib.asa_build_mask(q, k, blk, mode, topk, tau, ratio, diag, sink)
        assert cuda_lib.check_device_status() == 0
        nb = -(-N // blk)
        cap = cuda_lib.asa_max_nnz(B, H, N, blk, mode, topk, ratio, diag, sink)
        row_ptr = torch.full((B * H * nb + 1,), -1, dtype=torch.int32, device="cuda")
        col_idx = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
        rc = _noalloc(lib, cuda_lib, q, k, blk, mode, topk, tau, ratio, diag, sink, row_ptr, col_idx)
        assert rc == 0, cuda_lib.status_string(rc)
        assert cuda_lib.check_device_status() == 0
        nnz = int(row_ptr[-1])
        assert torch.equal(row_ptr, ref_rp)
        assert torch.equal(col_idx[:nnz], ref_ci)


def test_noalloc_rejects_shapes_beyond_the_array(cuda_lib):
    lib = cuda_lib.load()
    # B1 H24 N118800 d128 blk64 needs 2*44568*128*4 + 44568*59*4 bytes > 16 MiB
    B, H, N, d, blk = 1, 24, 118800, 128, 64
    assert cuda_lib.asa_workspace_size(B, H, N, d, blk) > MAX_BYTES
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    row_ptr = torch.full((B * H * 1857 + 1,), -1, dtype=torch.int32, device="cuda")
    col_idx = torch.full((16,), -1, dtype=torch.int32, device="cuda")
    rc = _noalloc(lib, cuda_lib, q, q, blk, 0, 4, 0.0, 0.0, 0, 0, row_ptr, col_idx)
    assert rc == cuda_lib.ERR_WORKSPACE
    assert cuda_lib.check_device_status() == 0
    assert torch.all(row_ptr == -1) and torch.all(col_idx == -1)   # nothing was launched
