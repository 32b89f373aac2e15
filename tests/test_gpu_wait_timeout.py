"""Failure detection on the GPU without a fault (through the C ABI).

Every wait in the library's kernels is an mbarrier wait bounded by
%globaltimer; on expiry the kernel records BSA_ERR_TIMEOUT in the device
status and unwinds.  Here that wait runs out on purpose: one thread waits on
a phase that nothing completes (no trap, no bad address, no endless loop).
The host must read BSA_ERR_TIMEOUT once, the wait must have lasted the limit
and not much longer, the read must clear the status, a wait whose phase does
complete must pass, and the same context must still compute correctly.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_asa_b200 import workloads as W
from tests._compare import compare_attention

pytestmark = pytest.mark.gpu

LIMIT_NS = 20_000_000   # 20 ms


def test_bounded_wait_gives_up_and_the_context_survives(cuda_lib):
    assert cuda_lib.check_device_status() == 0
    waited = torch.zeros(1, dtype=torch.int64, device="cuda")
    cuda_lib.debug_wait_timeout(LIMIT_NS, arrive_first=False, waited=waited)
    assert cuda_lib.check_device_status() == cuda_lib.ERR_TIMEOUT
    w = int(waited.item())
    assert LIMIT_NS <= w < 2_000_000_000, w
    assert cuda_lib.check_device_status() == 0          # the read cleared it
    # a phase that completes: no timeout, and well under the limit
    cuda_lib.debug_wait_timeout(LIMIT_NS, arrive_first=True, waited=waited)
    assert cuda_lib.check_device_status() == 0
    assert int(waited.item()) < LIMIT_NS
    # the context still computes: the tiny ASA layer against the oracle
    tiny = W.TINY
    q, k, v = W.make_qkv(tiny)
    rp, ci = cuda_lib.asa_build_mask(q.cuda(), k.cuda(), tiny.blk, tiny.mode, tiny.topk, tiny.mass_tau,
                                     tiny.max_keep_ratio, tiny.keep_diag, tiny.n_sink_blocks)
    o, lse = cuda_lib.bsa_forward(q.cuda(), k.cuda(), v.cuda(), tiny.blk, rp, ci)
    assert cuda_lib.check_device_status() == 0
    rp_h, ci_h = rp.cpu().numpy().astype(np.int64), ci.cpu().numpy()
    o_ref, l_ref = oracle.masked_attention(W.as_f64(q), W.as_f64(k), W.as_f64(v), tiny.blk, rp_h, ci_h)
    compare_attention(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)
