"""bench.py's host-side helpers (CPU): the flop count of a mask, the clock
summary of nvidia-smi samples inside the timed window, and the traffic table
that only applies to the kernel source it was measured on."""
import importlib.util
import os

import numpy as np
import pytest

from block_sparse_attention_asa_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_block_flops_counts_valid_tokens(bench):
    # N = 40 at blk 16: blocks of 16, 16, 8; one head, d = 64
    w = W.Workload(name="f", B=1, H=1, d=64, frames=1, height=1, width=40, blk=16, seed=0)
    rp = np.array([0, 2, 2, 5])            # rows: {0, 2}, {}, {0, 1, 2}
    ci = np.array([0, 2, 0, 1, 2])
    want = 4 * 64 * (16 * 16 + 16 * 8 + 0 + 8 * 16 + 8 * 16 + 8 * 8)
    assert bench.block_flops(w, rp, ci) == want


def test_clock_summary_keeps_the_timed_window_only(bench):
    c = bench.ClockSampler(0)
    c.t0, c.t1 = 10.0, 11.0
    line = "0, {sm}, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, {cap}"
    c.lines = [
        (9.0, line.format(sm=345, cap="Not Active")),      # before the window
        (10.2, line.format(sm=1965, cap="Not Active")),
        (10.5, line.format(sm=1900, cap="Active")),
        (10.9, line.format(sm=1950, cap="Not Active")),
        (13.0, line.format(sm=210, cap="Active")),         # after it
        (10.6, "garbled"),
    ]
    s = c.summary()
    assert s["sm_mhz"] == 1950 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    empty = bench.ClockSampler(0)
    assert empty.summary()["reasons"] == ["unsampled"]


def test_traffic_applies_to_its_kernel_source_only(bench, monkeypatch):
    assert bench.fwd_traffic("no-such-workload") is None
    monkeypatch.setattr(bench, "FWD_TRAFFIC", {("wan2.1_1.3b_asa", "0" * 64): 1})
    assert bench.fwd_traffic("wan2.1_1.3b_asa") is None


def test_sweep_workload_selection(bench):
    w = bench.workload("sweep", 0.25, 128)
    assert (w.N, w.blk, w.nb, w.topk, w.mode) == (32760, 128, 256, 64, W.MODE_TOPK)
    assert bench.workload("sweep", 1.0, 64).topk == 512        # the dense end of the sweep
    assert bench.workload("wan", 0.25, 128) is W.WAN           # keep / blk apply to the sweep only
    with pytest.raises(ValueError):
        bench.workload("sweep", 0.3, 64)
