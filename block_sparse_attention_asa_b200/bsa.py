"""Python binding of libbsa_b200.so (include/bsa.h), over ctypes.

Argument marshalling only: torch provides device memory and the current
stream; every step of the computation runs in the library's CUDA kernels.
There is no fallback: without the built library, or without a CUDA device,
the calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
import re
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# The in-tree build; BSA_B200_LIB may name another build of the same library.
LIB_PATH = os.environ.get("BSA_B200_LIB") or os.path.join(_HERE, "libbsa_b200.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "bsa.h")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_CAPACITY = -3
ERR_CUDA = -4
ERR_TIMEOUT = -5
ERR_CSR = -6
ERR_WORKSPACE = -7

MODE_TOPK = 0
MODE_MASS = 1

_c_int, _c_float, _c_size, _c_i64, _vp = (ctypes.c_int, ctypes.c_float, ctypes.c_size_t,
                                          ctypes.c_int64, ctypes.c_void_p)

_SIGNATURES = {
    "asa_build_mask_workspace_size": (_c_size, [_c_int] * 5),
    "asa_build_mask_max_nnz": (_c_i64, [_c_int] * 6 + [_c_float, _c_int, _c_int]),
    "asa_build_mask": (_c_int, [_vp, _vp] + [_c_int] * 7 + [_c_float, _c_float, _c_int, _c_int,
                                                             _c_float, _vp, _vp, _c_i64, _vp,
                                                             _c_size, _vp]),
    "asa_build_mask_noalloc": (_c_int, [_vp, _vp] + [_c_int] * 7 + [_c_float, _c_float, _c_int,
                                                                     _c_int, _c_float, _vp, _vp,
                                                                     _c_i64, _vp]),
    "pattern_mask": (_c_int, [_vp] + [_c_int] * 10 + [_vp, _vp, _c_i64, _vp, _vp]),
    "bsa_forward_workspace_size": (_c_size, [_c_int] * 5),
    "bsa_forward": (_c_int, [_vp, _vp, _vp] + [_c_int] * 5 + [_vp, _vp, _c_float, _vp, _vp, _vp,
                                                              _c_size, _vp]),
    "bsa_forward_residual": (_c_int, [_vp, _vp, _vp] + [_c_int] * 5 + [_vp, _vp, _c_float, _vp, _vp,
                                                                       _vp, _vp, _c_size, _vp]),
    "bsa_backward_workspace_size": (_c_size, [_c_int] * 5),
    "bsa_backward_residual": (_c_int, [_vp] * 7 + [_c_int] * 5 + [_vp, _vp, _c_float, _vp, _vp,
                                                                  _vp, _vp, _c_size, _vp]),
    "bsa_backward": (_c_int, [_vp] * 6 + [_c_int] * 5 + [_vp, _vp, _c_float, _vp, _vp, _vp, _vp,
                                                          _c_size, _vp]),
    "bsa_validate_csr_host": (_c_int, [_vp, _vp, _c_i64, _c_int, _c_i64, _vp]),
    "bsa_check_device_status": (_c_int, [_vp]),
    "bsa_status_string": (ctypes.c_char_p, [_c_int]),
    "bsa_version": (_c_int, []),
    "bsa_debug_exp2_poly": (_c_int, [_vp, _vp, _c_int, _vp]),
    "bsa_debug_wait_timeout": (_c_int, [ctypes.c_ulonglong, _c_int, _vp, _vp]),
    "attention_head_mse_workspace_size": (_c_size, [_c_int] * 4),
    "attention_head_mse": (_c_int, [_vp, _vp] + [_c_int] * 4 + [_vp, _vp, _c_size, _vp]),
    "csr_head_sparsity_workspace_size": (_c_size, [_c_int]),
    "csr_head_sparsity": (_c_int, [_vp, _vp] + [_c_int] * 4 + [_vp, _vp, _c_size, _vp]),
    "pattern_search_select": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, ctypes.c_double,
                                       ctypes.c_double, _vp, _vp]),
}

_lib = None


class BsaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


def header_functions() -> list:
    """Names of the functions include/bsa.h declares."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(",
                                 text, flags=re.M)))


def load(path: str = LIB_PATH):
    """Load the library (once) and declare every exported signature."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libbsa_b200.so is not built ({path}); run "
                           "block_sparse_attention_asa_b200/build.py")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().bsa_status_string(int(code)).decode()


def _check(code: int, where: str):
    if code != OK:
        raise BsaError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if not (isinstance(t, torch.Tensor) and t.is_cuda and t.is_contiguous()):
            raise ValueError("expected contiguous CUDA tensors")


def _shape(q: torch.Tensor):
    if q.dim() != 4 or q.dtype != torch.bfloat16:
        raise ValueError("q/k/v must be bf16 [B, H, N, d]")
    return tuple(int(x) for x in q.shape)


def validate_csr(row_ptr, col_idx, nb: int) -> int:
    """-1 if the CSR block mask (host arrays or tensors) follows the library's
    conventions (rows strictly ascending, ids in [0, nb)), else the first bad row."""
    import numpy as np
    rp = np.ascontiguousarray(torch.as_tensor(row_ptr).cpu().numpy(), dtype=np.int32)
    ci = np.ascontiguousarray(torch.as_tensor(col_idx).cpu().numpy(), dtype=np.int32)
    bad = ctypes.c_int64(-1)
    rc = load().bsa_validate_csr_host(rp.ctypes.data, ci.ctypes.data if ci.size else None,
                                      len(rp) - 1, int(nb), ci.size, ctypes.byref(bad))
    if rc not in (OK, ERR_CSR):
        _check(rc, "bsa_validate_csr_host")
    return int(bad.value)


def check_device_status(stream=None) -> int:
    """Synchronize the stream and return (and clear) the device status word."""
    return int(load().bsa_check_device_status(_stream(stream)))


# ----------------------------------------------------------------------------- ASA
def asa_workspace_size(B: int, H: int, N: int, d: int, blk: int) -> int:
    return int(load().asa_build_mask_workspace_size(B, H, N, d, blk))


def asa_max_nnz(B, H, N, blk, mode, topk=0, max_keep_ratio=0.0, keep_diag=0, n_sink_blocks=0) -> int:
    return int(load().asa_build_mask_max_nnz(B, H, N, blk, mode, topk, max_keep_ratio, keep_diag,
                                            n_sink_blocks))


def asa_build_mask_into(q, k, blk, mode, topk, mass_tau, max_keep_ratio, keep_diag, n_sink_blocks,
                        softmax_scale, row_ptr, col_idx, workspace, stream=None):
    """Raw call into preallocated outputs; asynchronous, no allocation, no sync."""
    B, H, N, d = _shape(q)
    lib = load()
    rc = lib.asa_build_mask(_ptr(q), _ptr(k), B, H, N, d, blk, mode, topk, mass_tau,
                            max_keep_ratio, keep_diag, n_sink_blocks, softmax_scale, _ptr(row_ptr),
                            _ptr(col_idx), col_idx.numel(), _ptr(workspace),
                            workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "asa_build_mask")


def asa_build_mask(q: torch.Tensor, k: torch.Tensor, blk: int, mode: int = MODE_TOPK, topk: int = 0,
                   mass_tau: float = 0.0, max_keep_ratio: float = 0.0, keep_diag: int = 0,
                   n_sink_blocks: int = 0, softmax_scale: float = 0.0, trim: bool = True,
                   stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """CSR (row_ptr, col_idx) of the ASA mask.  trim=True reads nnz back (syncs)."""
    _need_cuda(q, k)
    B, H, N, d = _shape(q)
    nb = -(-N // blk)
    dev = q.device
    cap = asa_max_nnz(B, H, N, blk, mode, topk, max_keep_ratio, keep_diag, n_sink_blocks)
    if cap < 0:
        raise BsaError(ERR_UNSUPPORTED, "asa_build_mask")
    row_ptr = torch.empty(B * H * nb + 1, dtype=torch.int32, device=dev)
    col_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
    ws = torch.empty(max(asa_workspace_size(B, H, N, d, blk), 256), dtype=torch.uint8, device=dev)
    asa_build_mask_into(q, k, blk, mode, topk, mass_tau, max_keep_ratio, keep_diag, n_sink_blocks,
                        softmax_scale, row_ptr, col_idx, ws, stream)
    if trim:
        nnz = int(row_ptr[-1].item())
        col_idx = col_idx[:nnz]
    return row_ptr, col_idx


def asa_build_mask_noalloc_into(q, k, blk, mode, topk, mass_tau, max_keep_ratio, keep_diag,
                                n_sink_blocks, softmax_scale, row_ptr, col_idx, stream=None):
    """The ASA mask into preallocated outputs, with the library's own fixed
    scratch instead of a workspace: for callers that may not allocate device
    memory.  Asynchronous; concurrent calls on one device must be serialized."""
    B, H, N, d = _shape(q)
    rc = load().asa_build_mask_noalloc(_ptr(q), _ptr(k), B, H, N, d, blk, mode, topk, mass_tau,
                                       max_keep_ratio, keep_diag, n_sink_blocks, softmax_scale,
                                       _ptr(row_ptr), _ptr(col_idx), col_idx.numel(),
                                       _stream(stream))
    _check(rc, "asa_build_mask_noalloc")


# ----------------------------------------------------------------------------- patterns
def pattern_mask(head_pattern: Sequence[int], B: int, H: int, N: int, blk: int, band_w: int = 2,
                 frame_tokens: int = 1, f_lo: int = 0, f_hi: int = 0, stripe_blocks: int = 0,
                 tile_global_frames: int = 0, device=None, stream=None):
    """CSR of the per-head fixed patterns (syncs once to size col_idx)."""
    lib = load()
    dev = torch.device("cuda") if device is None else torch.device(device)
    nb = -(-N // blk)
    hp = (ctypes.c_int32 * H)(*[int(x) for x in head_pattern])
    row_ptr = torch.empty(B * H * nb + 1, dtype=torch.int32, device=dev)
    nnz = ctypes.c_int64(0)
    # first pass with zero capacity: counts, scan and the nnz (writes nothing)
    rc = lib.pattern_mask(hp, B, H, N, blk, band_w, frame_tokens, f_lo, f_hi, stripe_blocks,
                          tile_global_frames, _ptr(row_ptr), None, 0, ctypes.byref(nnz),
                          _stream(stream))
    if rc not in (OK, ERR_CAPACITY):
        _check(rc, "pattern_mask")
    col_idx = torch.empty(max(int(nnz.value), 1), dtype=torch.int32, device=dev)
    pattern_mask_into(hp, B, H, N, blk, band_w, frame_tokens, f_lo, f_hi, stripe_blocks,
                      tile_global_frames, row_ptr, col_idx, stream)
    return row_ptr, col_idx[:int(nnz.value)]


def pattern_mask_into(head_pattern, B, H, N, blk, band_w, frame_tokens, f_lo, f_hi, stripe_blocks,
                      tile_global_frames, row_ptr, col_idx, stream=None):
    """Raw asynchronous call into preallocated outputs."""
    lib = load()
    if not isinstance(head_pattern, ctypes.Array):
        head_pattern = (ctypes.c_int32 * H)(*[int(x) for x in head_pattern])
    rc = lib.pattern_mask(head_pattern, B, H, N, blk, band_w, frame_tokens, f_lo, f_hi,
                          stripe_blocks, tile_global_frames, _ptr(row_ptr), _ptr(col_idx),
                          col_idx.numel(), None, _stream(stream))
    _check(rc, "pattern_mask")


# ----------------------------------------------------------------------------- forward
def forward_workspace_size(B: int, H: int, N: int, d: int, blk: int) -> int:
    return int(load().bsa_forward_workspace_size(B, H, N, d, blk))


def bsa_forward_into(q, k, v, blk, row_ptr, col_idx, o, lse=None, softmax_scale=0.0,
                     workspace=None, stream=None, o_residual=None):
    B, H, N, d = _shape(q)
    lib = load()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if o_residual is None:
        rc = lib.bsa_forward(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, blk, _ptr(row_ptr),
                             _ptr(col_idx), softmax_scale, _ptr(o), _ptr(lse), _ptr(workspace),
                             ws_bytes, _stream(stream))
        _check(rc, "bsa_forward")
        return
    rc = lib.bsa_forward_residual(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, blk, _ptr(row_ptr),
                                  _ptr(col_idx), softmax_scale, _ptr(o), _ptr(lse),
                                  _ptr(o_residual), _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "bsa_forward_residual")


def bsa_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, blk: int, row_ptr: torch.Tensor,
                col_idx: torch.Tensor, softmax_scale: float = 0.0, stream=None,
                residual: bool = False):
    """(O bf16 [B,H,N,d], LSE fp32 [B,H,N]) of attention over the CSR's kept blocks;
    with residual=True also O's bf16 rounding residual (O + residual carries the
    fp32 O), for bsa_backward's o_residual."""
    _need_cuda(q, k, v, row_ptr)
    B, H, N, d = _shape(q)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    ws_n = forward_workspace_size(B, H, N, d, blk)
    ws = torch.empty(ws_n, dtype=torch.uint8, device=q.device) if ws_n else None
    if col_idx.numel() == 0:
        col_idx = torch.zeros(1, dtype=torch.int32, device=q.device)
    res = torch.empty_like(q) if residual else None
    bsa_forward_into(q, k, v, blk, row_ptr, col_idx, o, lse, softmax_scale, ws, stream, res)
    return (o, lse, res) if residual else (o, lse)


# ----------------------------------------------------------------------------- backward
def backward_workspace_size(B: int, H: int, N: int, d: int, blk: int) -> int:
    return int(load().bsa_backward_workspace_size(B, H, N, d, blk))


def bsa_backward_into(q, k, v, o, dout, lse, blk, row_ptr, col_idx, dq, dk, dv,
                      softmax_scale=0.0, workspace=None, stream=None, o_residual=None):
    B, H, N, d = _shape(q)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if o_residual is None:
        rc = load().bsa_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), B, H,
                                 N, d, blk, _ptr(row_ptr), _ptr(col_idx), softmax_scale, _ptr(dq),
                                 _ptr(dk), _ptr(dv), _ptr(workspace), ws_bytes, _stream(stream))
        _check(rc, "bsa_backward")
        return
    rc = load().bsa_backward_residual(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(o_residual),
                                      _ptr(dout), _ptr(lse), B, H, N, d, blk, _ptr(row_ptr),
                                      _ptr(col_idx), softmax_scale, _ptr(dq), _ptr(dk), _ptr(dv),
                                      _ptr(workspace), ws_bytes, _stream(stream))
    _check(rc, "bsa_backward_residual")


def bsa_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                 dout: torch.Tensor, lse: torch.Tensor, blk: int, row_ptr: torch.Tensor,
                 col_idx: torch.Tensor, softmax_scale: float = 0.0, stream=None,
                 o_residual: Optional[torch.Tensor] = None):
    """(dQ, dK, dV) bf16 [B,H,N,d] of attention over the CSR's kept blocks for the
    incoming gradient dout; o and lse are bsa_forward's outputs for the same call
    (o_residual: its residual output, so that D comes from the fp32 O)."""
    _need_cuda(q, k, v, o, dout, lse, row_ptr)
    B, H, N, d = _shape(q)
    for t in (k, v, o, dout):
        if tuple(t.shape) != (B, H, N, d) or t.dtype != torch.bfloat16:
            raise ValueError("k, v, o, dout must match q (bf16 [B, H, N, d])")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be float32 [B, H, N]")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(backward_workspace_size(B, H, N, d, blk), 256), dtype=torch.uint8,
                     device=q.device)
    if col_idx.numel() == 0:
        col_idx = torch.zeros(1, dtype=torch.int32, device=q.device)
    if o_residual is not None and (tuple(o_residual.shape) != (B, H, N, d) or
                                   o_residual.dtype != torch.bfloat16):
        raise ValueError("o_residual must match q (bf16 [B, H, N, d])")
    bsa_backward_into(q, k, v, o, dout, lse, blk, row_ptr, col_idx, dq, dk, dv, softmax_scale, ws,
                      stream, o_residual)
    return dq, dk, dv


class _BlockSparseAttention(torch.autograd.Function):
    """bsa_forward / bsa_backward as one autograd node.  The mask is a constant
    of the step and only O is returned, so nothing downstream can depend on an
    undifferentiated LSE.  The forward keeps O's rounding residual for the
    backward, so that D comes from the fp32 O."""

    @staticmethod
    def forward(ctx, q, k, v, blk, row_ptr, col_idx, softmax_scale):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o, lse, res = bsa_forward(q, k, v, blk, row_ptr, col_idx, softmax_scale, residual=True)
        ctx.save_for_backward(q, k, v, o, lse, res, row_ptr, col_idx)
        ctx.blk = blk
        ctx.softmax_scale = softmax_scale
        return o

    @staticmethod
    def backward(ctx, dout):
        q, k, v, o, lse, res, row_ptr, col_idx = ctx.saved_tensors
        dq, dk, dv = bsa_backward(q, k, v, o, dout.contiguous().to(torch.bfloat16), lse, ctx.blk,
                                  row_ptr, col_idx, ctx.softmax_scale, o_residual=res)
        return dq, dk, dv, None, None, None, None


def block_sparse_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, blk: int,
                           row_ptr: torch.Tensor, col_idx: torch.Tensor,
                           softmax_scale: float = 0.0) -> torch.Tensor:
    """Differentiable O of attention over the CSR's kept blocks (bf16 [B,H,N,d]);
    gradients flow to q, k and v, none to the mask."""
    return _BlockSparseAttention.apply(q, k, v, blk, row_ptr, col_idx, softmax_scale)


def head_mse(o_ref: torch.Tensor, o: torch.Tensor, stream=None) -> torch.Tensor:
    """Per-head MSE(O - O_ref) over all B*N*d elements, float64 [H] on the device."""
    _need_cuda(o_ref, o)
    B, H, N, d = _shape(o_ref)
    lib = load()
    mse = torch.empty(H, dtype=torch.float64, device=o_ref.device)
    ws = torch.empty(max(int(lib.attention_head_mse_workspace_size(B, H, N, d)), 256),
                     dtype=torch.uint8, device=o_ref.device)
    _check(lib.attention_head_mse(_ptr(o_ref), _ptr(o), B, H, N, d, _ptr(mse), _ptr(ws),
                                  ws.numel(), _stream(stream)), "attention_head_mse")
    return mse


def head_sparsity(row_ptr: torch.Tensor, col_idx: torch.Tensor, B: int, H: int, N: int, blk: int,
                  stream=None) -> torch.Tensor:
    """Per-head fraction of (query, key) token pairs a CSR block mask skips, float64 [H]."""
    _need_cuda(row_ptr)
    lib = load()
    out = torch.empty(H, dtype=torch.float64, device=row_ptr.device)
    ws = torch.empty(max(int(lib.csr_head_sparsity_workspace_size(H)), 256), dtype=torch.uint8,
                     device=row_ptr.device)
    ci = col_idx if col_idx is not None and col_idx.numel() > 0 else None
    _check(lib.csr_head_sparsity(_ptr(row_ptr), _ptr(ci), B, H, N, blk, _ptr(out), _ptr(ws),
                                 ws.numel(), _stream(stream)), "csr_head_sparsity")
    return out


def search_select(mse, sparsity, candidates: Sequence[int], lam: float, eps: float):
    """Sparse-vDiT selection on host arrays mse, sparsity [P, H]:
    (choice int32 [H], loss float64 [P, H])."""
    import numpy as np
    mse = np.ascontiguousarray(mse, dtype=np.float64)
    sp = np.ascontiguousarray(sparsity, dtype=np.float64)
    P, H = mse.shape
    cand = np.ascontiguousarray(candidates, dtype=np.int32)
    loss = np.empty((P, H), dtype=np.float64)
    choice = np.empty(H, dtype=np.int32)
    _check(load().pattern_search_select(mse.ctypes.data, sp.ctypes.data, cand.ctypes.data, P, H,
                                        float(lam), float(eps), loss.ctypes.data,
                                        choice.ctypes.data), "pattern_search_select")
    return choice, loss


def debug_exp2_poly(x: torch.Tensor, stream=None) -> torch.Tensor:
    """The attention kernel's FMA-pipe 2^x, evaluated on a CUDA float32 tensor."""
    _need_cuda(x)
    y = torch.empty_like(x)
    _check(load().bsa_debug_exp2_poly(_ptr(x), _ptr(y), x.numel(), _stream(stream)),
           "bsa_debug_exp2_poly")
    return y


def debug_wait_timeout(limit_ns: int, arrive_first: bool = False,
                       waited: Optional[torch.Tensor] = None, stream=None) -> None:
    """Run the library's bounded mbarrier wait on a phase that completes only if
    arrive_first; without it the wait gives up after limit_ns and the device
    status reads ERR_TIMEOUT.  waited: optional CUDA int64 [1], the time taken."""
    if waited is not None:
        _need_cuda(waited)
        if waited.dtype != torch.int64 or waited.numel() < 1:
            raise ValueError("waited must be a CUDA int64 tensor")
    _check(load().bsa_debug_wait_timeout(int(limit_ns), int(bool(arrive_first)), _ptr(waited),
                                         _stream(stream)), "bsa_debug_wait_timeout")


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
