"""The bench's end-to-end step, with its host copies overlapped with its
compute: mask and forward run per group of (b, h) slices through the public
API on three streams.  Its outputs, copied back to the host, must be the same
bits as one whole-layer call (the mask and the forward treat every (b, h) on
its own, and both are deterministic)."""
import pytest
import torch

import bench
from block_sparse_attention_asa_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,chunks", [("tiny", 2), ("tile3d", 5)])
def test_pipelined_end_to_end_matches_one_call(cuda_lib, name, chunks):
    w = bench.workload(name)
    dev = torch.device("cuda", 0)
    lay = bench.Layer(cuda_lib, w, dev)
    # reference: the whole layer in one mask + forward call
    lay.mask()
    lay.forward()
    torch.cuda.synchronize()
    o_ref, lse_ref = lay.o.cpu(), lay.lse.cpu()
    q_h, k_h, v_h = lay.host
    q_p, k_p, v_p = (x.pin_memory() for x in (q_h, k_h, v_h))
    o_p = torch.zeros(lay.o.shape, dtype=lay.o.dtype).pin_memory()
    lse_p = torch.zeros(lay.lse.shape, dtype=lay.lse.dtype).pin_memory()
    lay.o.zero_()
    lay.lse.zero_()
    ms = bench.time_e2e_pipelined(cuda_lib, lay, q_p, k_p, v_p, o_p, lse_p, steps=2, chunks=chunks)
    assert ms > 0.0
    assert cuda_lib.check_device_status() == 0
    assert torch.equal(o_p, o_ref)
    assert torch.equal(lse_p, lse_ref)
