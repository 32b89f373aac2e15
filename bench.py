#!/usr/bin/env python
"""Benchmark of the block-sparse attention layer (ASA mask + attention over the
kept blocks) on B200, one process per GPU.

A step is one pass of the hot path over one layer: asa_build_mask (pool, score
and select, CSR) followed by bsa_forward, through the C ABI.  The default
workload is the Wan2.1-1.3B-shaped self-attention layer (B1 H12 N32760 d128,
block 64, cumulative mass 0.9 capped at keep ratio 0.1).  The metric is the
effective TFLOPS over computed blocks: Σ over kept (q-block, kv-block) pairs of
4·n_q·n_k·d with valid tokens only, divided by the step time.

  python bench.py [--gpus N --steps K --warmup W] [--workload wan|cog|hunyuan|tiny]
  python bench.py --workload sweep --keep 0.25 --blk 128   # the keep-ratio sweep
  python bench.py --impl reference      # the fp64 CPU oracle on a bounded sample

On one GPU the same line also carries, under "extra", the other layers timed
the same way with fewer steps (the CogVideoX-shaped layer, the HunyuanVideo-
shaped layer with its fixed patterns, the Wan-shaped layer under the 3D tile,
and the ten keep-ratio x block-size sweep
points on the Wan shape, mask time apart from forward time) and the backward on
the headline layer (--no-extra skips them).

Under torchrun every rank runs its own replica of the layer (the path has no
cross-GPU exchange); the timed region is bracketed by barriers and the maximum
over ranks is reported.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_asa_b200 import workloads as W  # noqa: E402

METRIC = "block-sparse attn effective TFLOPS & % BF16 TC peak; ms/layer at keep ratio"
DATASHEET_BF16_TFLOPS = 2250.0
DATASHEET_HBM_GBS = 8000.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM bytes (read + write) per bsa_fwd_kernel launch, from one ncu capture of
# this script's own `--profile forward` run on that workload, keyed by workload
# and by the sha256 of the kernel source the capture ran: once the kernel
# changes, the figure no longer applies and the bench reports null.
FWD_TRAFFIC = {
    ("wan2.1_1.3b_asa", "4017ae624679036b3512ec6508f53ca5bf413e578eb5360d9a65f4c147c10ea7"):
        303439872 + 84715264,
}


def fwd_traffic(workload_name: str):
    import hashlib
    src = os.path.join(ROOT, "block_sparse_attention_asa_b200", "csrc", "bsa_fwd.cuh")
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    return FWD_TRAFFIC.get((workload_name, sha))


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK), "fallback"


def workload(name: str, keep: float = 0.1, blk: int = 64) -> W.Workload:
    """The named layer; "sweep" is the Wan-shaped layer under top-k with
    k = floor(keep * nb) at block size blk."""
    if name == "sweep":
        if keep not in W.SWEEP_KEEPS or blk not in W.SWEEP_BLKS:
            raise ValueError(f"sweep points: keep in {W.SWEEP_KEEPS}, blk in {W.SWEEP_BLKS}")
        return W.sweep(keep, blk)
    return {"wan": W.WAN, "cog": W.COG, "hunyuan": W.HUNYUAN, "tiny": W.TINY,
            "tile3d": W.WAN_TILE3D}[name]


def block_flops(w: W.Workload, row_ptr: np.ndarray, col_idx: np.ndarray) -> float:
    """Σ over kept (row, kv-block) of 4·n_q·n_k·d on valid tokens."""
    nb = w.nb
    sizes = np.full(nb, w.blk, dtype=np.float64)
    sizes[-1] = w.N - (nb - 1) * w.blk
    rows = len(row_ptr) - 1
    counts = np.diff(row_ptr.astype(np.int64))
    i_of_row = np.arange(rows) % nb
    nq = np.repeat(sizes[i_of_row], counts)
    nk = sizes[col_idx[:int(row_ptr[-1])]]
    return float(4.0 * w.d * np.sum(nq * nk))


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons.

    The sampler is started, and its first sample awaited, before the timed
    region; only samples whose host arrival time lies inside the region set by
    mark_start()/mark_end() are summarised."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 20

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []          # (host time, line)
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.PERIOD_MS)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            deadline = time.monotonic() + 15.0
            while not self.lines and time.monotonic() < deadline and self.proc.poll() is None:
                time.sleep(0.01)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def mark_start(self):
        self.t0 = time.monotonic()

    def mark_end(self):
        self.t1 = time.monotonic()

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(2.0 * self.PERIOD_MS / 1000.0)   # let the last in-region sample arrive
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lo = self.t0 if self.t0 is not None else -float("inf")
        hi = (self.t1 if self.t1 is not None else float("inf")) + self.PERIOD_MS / 1000.0
        for ts, ln in self.lines:
            if not (lo <= ts <= hi):
                continue
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus: int):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- CPU oracle
def oracle_inputs(w: W.Workload, heads: int):
    """fp64 inputs of the first `heads` heads of the layer (drawn like the GPU's)."""
    q, k, v = W.make_qkv(w)
    return tuple(W.as_f64(t[:, :heads].contiguous()) for t in (q, k, v))


def oracle_step(w: W.Workload, qkv, heads: int):
    """One oracle pass (ASA mask + masked attention) over the sample: (seconds, flops)."""
    import oracle
    qf, kf, vf = qkv
    t0 = time.perf_counter()
    m = oracle.asa_mask(qf, kf, w.blk, w.mode, w.topk, w.mass_tau, w.max_keep_ratio, w.keep_diag,
                        w.n_sink_blocks)
    oracle.masked_attention(qf, kf, vf, w.blk, m.row_ptr, m.col_idx)
    dt = time.perf_counter() - t0
    sub = W.Workload(**{**w.__dict__, "H": heads})
    return dt, block_flops(sub, m.row_ptr, m.col_idx)


def run_reference(args, rank, world):
    if rank != 0:
        return
    w = workload(args.workload, args.keep, args.blk)
    if w.source != "asa":
        print(json.dumps({"impl": "reference", "unavailable":
                          "the CPU oracle arm times the ASA workloads only"}), flush=True)
        return
    heads = max(1, min(w.H, args.ref_heads_per_step))
    qkv = oracle_inputs(w, heads)
    for _ in range(args.warmup):
        oracle_step(w, qkv, heads)
    times, fl = [], 0.0
    for _ in range(args.steps):
        dt, fl = oracle_step(w, qkv, heads)
        times.append(dt)
    sec = sum(times) / len(times)
    val = fl / sec / 1e12
    sample = (f"{w.name}: heads 0..{heads - 1} of {w.H} per step "
              f"(ASA mask + masked attention, fp64 numpy)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "blk": w.blk,
                   "sample_heads": heads},
        "cpu_baseline": {"value": val, "unit": "TFLOPS", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": val, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ----------------------------------------------------------------------------- GPU
class Layer:
    """Device buffers of one workload and the two launches of its step (the mask,
    then bsa_forward), through the C ABI."""

    def __init__(self, bsa, w: W.Workload, dev, qkv=None):
        self.bsa, self.w, self.dev = bsa, w, dev
        if qkv is None:
            self.host = W.make_qkv(w)
            qkv = tuple(t.to(dev) for t in self.host)
        else:
            self.host = None
        self.q, self.k, self.v = qkv
        B, H, N, d = self.q.shape
        self.rows = B * H * w.nb
        if w.source == "asa":
            cap = bsa.asa_max_nnz(B, H, N, w.blk, w.mode, w.topk, w.max_keep_ratio, w.keep_diag,
                                  w.n_sink_blocks)
            self.ws = torch.empty(bsa.asa_workspace_size(B, H, N, d, w.blk), dtype=torch.uint8,
                                  device=dev)
            self.hp = None
        else:
            _, ci_probe = bsa.pattern_mask(w.head_pattern, B, H, N, w.blk, w.band_w,
                                           w.frame_tokens, w.f_lo, w.f_hi, w.stripe_blocks,
                                           w.tile_global_frames, device=dev)
            cap = int(ci_probe.numel())
            del ci_probe
            self.ws = None
            import ctypes
            self.hp = (ctypes.c_int32 * H)(*w.head_pattern)
        self.row_ptr = torch.empty(self.rows + 1, dtype=torch.int32, device=dev)
        self.col_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
        self.fws = torch.empty(max(bsa.forward_workspace_size(B, H, N, d, w.blk), 4),
                               dtype=torch.uint8, device=dev)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        # kernels per step: pool and select (ASA) or pattern row_ptr and
        # write; then the forward
        self.launches = 2 + 1

    def mask(self):
        w, b = self.w, self.bsa
        B, H, N, _ = self.q.shape
        if w.source == "asa":
            b.asa_build_mask_into(self.q, self.k, w.blk, w.mode, w.topk, w.mass_tau,
                                  w.max_keep_ratio, w.keep_diag, w.n_sink_blocks, 0.0,
                                  self.row_ptr, self.col_idx, self.ws)
        else:
            b.pattern_mask_into(self.hp, B, H, N, w.blk, w.band_w, w.frame_tokens, w.f_lo,
                                w.f_hi, w.stripe_blocks, w.tile_global_frames, self.row_ptr,
                                self.col_idx)

    def forward(self):
        self.bsa.bsa_forward_into(self.q, self.k, self.v, self.w.blk, self.row_ptr, self.col_idx,
                                  self.o, self.lse, workspace=self.fws)

    def mask_bytes(self, nnz: int) -> float:
        csr = 4.0 * (self.rows + 1) + 4.0 * nnz
        return csr + (2.0 * self.q.numel() * 2 if self.w.source == "asa" else 0.0)


def check_status(bsa, where: str):
    st = bsa.check_device_status()
    if st != 0:
        raise RuntimeError(f"device status {where}: {bsa.status_string(st)}")


def time_layer(layer: Layer, steps: int, warmup: int, local: int, world: int, stream):
    """Warm-up, then `steps` back-to-back steps with per-kernel CUDA events on the
    launching stream and the SM clock sampled inside the timed region."""
    bsa, w = layer.bsa, layer.w
    for _ in range(warmup):
        layer.mask()
        layer.forward()
    check_status(bsa, "after warm-up")
    rp_h = layer.row_ptr.cpu().numpy()
    ci_h = layer.col_idx[:int(rp_h[-1])].cpu().numpy()
    flops = block_flops(w, rp_h, ci_h)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        clk.mark_start()
        t0.record(stream)
        for s in range(steps):
            ev[s][0].record(stream)
            layer.mask()
            ev[s][1].record(stream)
            layer.forward()
            ev[s][2].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
    barrier(world)
    check_status(bsa, "after timing")
    return {
        "total_ms": t0.elapsed_time(t1),
        "mask_ms": [e[0].elapsed_time(e[1]) for e in ev],
        "fwd_ms": [e[1].elapsed_time(e[2]) for e in ev],
        "clocks": clk.summary(), "flops": flops, "nnz": int(rp_h[-1]),
        "keep": float(rp_h[-1]) / (layer.rows * w.nb),
    }


def layer_summary(layer: Layer, t: dict, pk: dict, steps: int) -> dict:
    """Per-layer figures of one timing: ms, TFLOPS and the fractions of the peaks."""
    fwd = statistics.mean(t["fwd_ms"])
    mask = statistics.mean(t["mask_ms"])
    tf = t["flops"] / (fwd * 1e-3) / 1e12
    gbs = layer.mask_bytes(t["nnz"]) / (mask * 1e-3) / 1e9
    return {
        "ms_per_layer": t["total_ms"] / steps, "ms_mask": mask, "ms_forward": fwd,
        "forward_tflops": tf, "frac": tf / float(pk["bf16_tflops"]),
        "mask_kernel": "asa_build_mask" if layer.w.source == "asa" else "pattern_mask",
        "mask_gbs": gbs, "mask_frac": gbs / float(pk["hbm_gbs"]),
        "keep_ratio": t["keep"], "block_flops": t["flops"], "steps": steps,
        "clocks": t["clocks"],
    }


def time_backward(bsa, layer: Layer, flops: float, pk: dict, iters: int = 10, warmup: int = 3):
    """The training path's backward (bsa_backward with the forward's rounding
    residual, as the autograd node runs it) on the layer's mask, O and LSE for a
    seeded dO (CUDA events, median of `iters` calls).  Flops at the usual 2.5x
    the forward's block flops."""
    q, k, v, w = layer.q, layer.k, layer.v, layer.w
    B, H, N, d = q.shape
    g = torch.Generator(device=q.device).manual_seed(5)
    dout = torch.randn(q.shape, generator=g, device=q.device).to(torch.bfloat16)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(bsa.backward_workspace_size(B, H, N, d, w.blk), 4), dtype=torch.uint8,
                     device=q.device)
    res = torch.empty_like(q)
    bsa.bsa_forward_into(q, k, v, w.blk, layer.row_ptr, layer.col_idx, layer.o, layer.lse,
                         workspace=layer.fws, o_residual=res)

    def call():
        bsa.bsa_backward_into(q, k, v, layer.o, dout, layer.lse, w.blk, layer.row_ptr,
                              layer.col_idx, dq, dk, dv, 0.0, ws, o_residual=res)
    for _ in range(warmup):
        call()
    check_status(bsa, "after backward warm-up")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(iters)]
    torch.cuda.synchronize()
    for a, b in evs:
        a.record()
        call()
        b.record()
    torch.cuda.synchronize()
    check_status(bsa, "after backward timing")
    ms = statistics.median(a.elapsed_time(b) for a, b in evs)
    tf = 2.5 * flops / (ms * 1e-3) / 1e12
    return {"workload": w.name, "ms_backward": ms, "tflops_2p5x": tf,
            "frac": tf / float(pk["bf16_tflops"]), "flop_convention": "2.5x forward block flops",
            "d_from": "fp32 O (forward rounding residual)", "iters": iters}


def time_e2e_pipelined(bsa, layer, q_p, k_p, v_p, o_p, lse_p, steps: int, chunks: int = 4):
    """End to end through the public API with pinned host buffers, the step's
    copies overlapped with its compute: the (b, h) slices are split into
    `chunks` groups; group i's H2D copy (copy-in stream), its mask + forward
    (compute stream) and its D2H copy (copy-out stream) are ordered by events,
    so group i+1 is copied in while group i computes and group i-1 is copied
    out.  Every byte of every step still crosses PCIe inside the timed region.
    Returns ms per step (CUDA events, first copy-in to last copy-out)."""
    w = layer.w
    q, k, v, o, lse = layer.q, layer.k, layer.v, layer.o, layer.lse
    B, H, N, d = q.shape
    BH = B * H
    C = max(1, min(chunks, BH))
    bounds = [(BH * i // C, BH * (i + 1) // C) for i in range(C)]
    cmax = max(i1 - i0 for i0, i1 in bounds)
    flat = lambda t: t.view(BH, *t.shape[2:])
    qf, kf, vf, of, lf = flat(q), flat(k), flat(v), flat(o), flat(lse)
    qpf, kpf, vpf, opf, lpf = flat(q_p), flat(k_p), flat(v_p), flat(o_p), flat(lse_p)
    view4 = lambda t, i0, i1: t[i0:i1].view(1, i1 - i0, *t.shape[1:])
    dev = q.device
    nb = w.nb
    row_ptr = torch.empty(cmax * nb + 1, dtype=torch.int32, device=dev)
    if w.source == "asa":
        cap = bsa.asa_max_nnz(1, cmax, N, w.blk, w.mode, w.topk, w.max_keep_ratio, w.keep_diag,
                              w.n_sink_blocks)
        ws = torch.empty(bsa.asa_workspace_size(1, cmax, N, d, w.blk), dtype=torch.uint8, device=dev)
    else:
        cap, ws = layer.col_idx.numel(), None
    col_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
    fws = torch.empty(max(bsa.forward_workspace_size(1, cmax, N, d, w.blk), 4), dtype=torch.uint8,
                      device=dev)
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in bounds]
    ev_cmp = [torch.cuda.Event() for _ in bounds]
    ev_out = [torch.cuda.Event() for _ in bounds]

    def step(first: bool):
        for ci, (i0, i1) in enumerate(bounds):
            c = i1 - i0
            if not first:
                s_in.wait_event(ev_cmp[ci])     # the last step's compute has read these inputs
            with torch.cuda.stream(s_in):
                qf[i0:i1].copy_(qpf[i0:i1], non_blocking=True)
                kf[i0:i1].copy_(kpf[i0:i1], non_blocking=True)
                vf[i0:i1].copy_(vpf[i0:i1], non_blocking=True)
            ev_in[ci].record(s_in)
            s_cmp.wait_event(ev_in[ci])
            if not first:
                s_cmp.wait_event(ev_out[ci])    # the last step's copy-out has read O
            qc, kc, vc = view4(qf, i0, i1), view4(kf, i0, i1), view4(vf, i0, i1)
            if w.source == "asa":
                bsa.asa_build_mask_into(qc, kc, w.blk, w.mode, w.topk, w.mass_tau, w.max_keep_ratio,
                                        w.keep_diag, w.n_sink_blocks, 0.0, row_ptr[:c * nb + 1],
                                        col_idx, ws, stream=s_cmp)
            else:
                hp = [w.head_pattern[bh % H] for bh in range(i0, i1)]
                bsa.pattern_mask_into(hp, 1, c, N, w.blk, w.band_w, w.frame_tokens, w.f_lo, w.f_hi,
                                      w.stripe_blocks, w.tile_global_frames, row_ptr[:c * nb + 1],
                                      col_idx, stream=s_cmp)
            bsa.bsa_forward_into(qc, kc, vc, w.blk, row_ptr[:c * nb + 1], col_idx,
                                 view4(of, i0, i1), view4(lf, i0, i1), workspace=fws, stream=s_cmp)
            ev_cmp[ci].record(s_cmp)
            s_out.wait_event(ev_cmp[ci])
            with torch.cuda.stream(s_out):
                opf[i0:i1].copy_(of[i0:i1], non_blocking=True)
                lpf[i0:i1].copy_(lf[i0:i1], non_blocking=True)
            ev_out[ci].record(s_out)

    torch.cuda.synchronize()
    step(True)                                  # warm-up
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for _ in range(steps):
        step(False)
    e1.record(s_out)
    torch.cuda.synchronize()
    check_status(bsa, "after the pipelined end-to-end steps")
    return e0.elapsed_time(e1) / steps


def run_gpu(args, rank, world, local):
    from block_sparse_attention_asa_b200 import bsa
    w = workload(args.workload, args.keep, args.blk)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    layer = Layer(bsa, w, dev)
    q_h, k_h, v_h = layer.host
    q, o, lse = layer.q, layer.o, layer.lse
    B, H, N, d = q.shape
    rows = layer.rows

    # ---- timed region: K steps, per-kernel events on the launching stream
    t = time_layer(layer, args.steps, args.warmup, local, world, stream)
    total_ms = barrier_max(t["total_ms"], world)
    ms_step = total_ms / args.steps
    flops, keep, nnz = t["flops"], t["keep"], t["nnz"]

    # ---- end to end through the public API with host buffers (pinned), copies timed
    q_p, k_p, v_p = (x.pin_memory() for x in (q_h, k_h, v_h))
    o_p = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    lse_p = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    e2e_steps = max(1, min(args.steps, 20))
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        layer.q.copy_(q_p, non_blocking=True)
        layer.k.copy_(k_p, non_blocking=True)
        layer.v.copy_(v_p, non_blocking=True)
        layer.mask()
        layer.forward()
        o_p.copy_(o, non_blocking=True)
        lse_p.copy_(lse, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_serial_ms = barrier_max(e0.elapsed_time(e1) / e2e_steps, world)
    e2e_ms = barrier_max(time_e2e_pipelined(bsa, layer, q_p, k_p, v_p, o_p, lse_p, e2e_steps), world)
    h2d = 3 * q.numel() * q.element_size()
    d2h = o.numel() * o.element_size() + lse.numel() * lse.element_size()

    pk, pk_kind = peaks()
    summ = layer_summary(layer, t, pk, args.steps)
    achieved = summ["forward_tflops"]
    peak = float(pk["bf16_tflops"])
    value = flops * world / (ms_step * 1e-3) / 1e12
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": w.name, "B": B, "H": H, "N": N, "d": d, "blk": w.blk,
            "mask": (f"mass tau={w.mass_tau} cap={w.max_keep_ratio}" if w.source == "asa" and
                     w.mode == W.MODE_MASS else
                     f"topk k={w.topk} sink={w.n_sink_blocks} diag={w.keep_diag}"
                     if w.source == "asa" else "fixed patterns per head"),
            "keep_ratio": keep, "block_flops": flops,
            "l2": f"inputs larger than L2: Q+K+V = {3 * q.numel() * 2 / 1e6:.0f} MB per step",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
        },
        "ms_mask": summ["ms_mask"], "ms_forward": summ["ms_forward"],
        "roofline": {"bound": "tensor", "kernel": "bsa_fwd_kernel", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_kind": f"{pk_kind} bf16 burst", "traffic": fwd_traffic(w.name),
                     "traffic_unit": "bytes per launch (ncu dram read + write)",
                     "frac_of_sustained": achieved / float(pk.get("bf16_tflops_sustained", peak)),
                     "frac_of_datasheet": achieved / DATASHEET_BF16_TFLOPS},
        "mask_roofline": {"bound": "hbm", "kernel": summ["mask_kernel"],
                          "achieved": summ["mask_gbs"], "peak": float(pk["hbm_gbs"]),
                          "unit": "GB/s", "frac": summ["mask_frac"],
                          "frac_of_8tbs": summ["mask_gbs"] / DATASHEET_HBM_GBS},
        "e2e": {"value": flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOPS",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "how": "public API, pinned host buffers; each step's copies overlapped with its "
                       "compute in 4 groups of (b, h) slices on copy-in, compute and copy-out streams",
                "serial_ms_per_step": e2e_serial_ms,
                "serial_value": flops * world / (e2e_serial_ms * 1e-3) / 1e12},
        "clocks": t["clocks"],
        "gpu_launches": layer.launches * args.steps,
    }
    if world == 1 and not args.no_extra:
        out["extra"] = run_extra(bsa, args, layer, flops, pk, local, stream)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and w.source == "asa":
        heads = max(1, min(w.H, args.ref_heads))
        dt, fl = oracle_step(w, oracle_inputs(w, heads), heads)
        out["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": "TFLOPS", "cores": os.cpu_count(),
                               "kind": "oracle",
                               "sample": f"heads 0..{heads - 1} of {w.H}, one pass, "
                                         f"{dt:.1f} s fp64 numpy"}
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_extra(bsa, args, head_layer: Layer, head_flops: float, pk: dict, local: int, stream):
    """The other layers the workloads name, each timed like the headline (fewer
    steps), plus the backward on the headline layer.  Keys: the workload names,
    "sweep" (keep ratio x block size on the Wan shape, inputs shared with the
    headline layer when it is that shape) and "backward"."""
    ex = {}
    dev = head_layer.dev
    steps, warm = args.extra_steps, 3
    try:
        ex["backward"] = time_backward(bsa, head_layer, head_flops, pk)
    except RuntimeError as e:
        ex["backward"] = {"error": str(e)}
    wan_qkv = (head_layer.q, head_layer.k, head_layer.v) if head_layer.w.name == W.WAN.name else None
    for wl in (W.COG, W.HUNYUAN, W.WAN_TILE3D):
        if wl.name == head_layer.w.name:
            continue
        same = wan_qkv is not None and (wl.B, wl.H, wl.N, wl.d, wl.seed, wl.scale, wl.pe) == (
            W.WAN.B, W.WAN.H, W.WAN.N, W.WAN.d, W.WAN.seed, W.WAN.scale, W.WAN.pe)
        lay = Layer(bsa, wl, dev, wan_qkv if same else None)
        ex[wl.name] = layer_summary(lay, time_layer(lay, steps, warm, local, 1, stream), pk, steps)
        del lay
        torch.cuda.empty_cache()
    sw = {}
    for blk in W.SWEEP_BLKS:
        for kp in W.SWEEP_KEEPS:
            ws = W.sweep(kp, blk)
            lay = Layer(bsa, ws, dev, wan_qkv)
            if wan_qkv is None:
                wan_qkv = (lay.q, lay.k, lay.v)
            sw[f"keep{kp}_blk{blk}"] = layer_summary(lay, time_layer(lay, steps, warm, local, 1,
                                                                     stream), pk, steps)
            del lay
    ex["sweep"] = sw
    return ex


def run_profile(args):
    """One op of the workload run back to back (`--warmup` + `--steps` calls) with
    nothing else around it, for a profiler's launch list or kernel capture:
    `mask` (the layer's mask source), `forward` (on the layer's mask) or
    `backward` (the training path: forward with the rounding residual once,
    then the backward for a seeded dO).  Prints one line; not a benchmark."""
    from block_sparse_attention_asa_b200 import bsa
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = workload(args.workload, args.keep, args.blk)
    lay = Layer(bsa, w, dev)
    lay.mask()
    if args.profile == "mask":
        call = lay.mask
    elif args.profile == "forward":
        call = lay.forward
    else:
        q, k, v = lay.q, lay.k, lay.v
        B, H, N, d = q.shape
        g = torch.Generator(device=dev).manual_seed(5)
        dout = torch.randn(q.shape, generator=g, device=dev).to(torch.bfloat16)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(max(bsa.backward_workspace_size(B, H, N, d, w.blk), 4), dtype=torch.uint8,
                         device=dev)
        res = torch.empty_like(q)
        bsa.bsa_forward_into(q, k, v, w.blk, lay.row_ptr, lay.col_idx, lay.o, lay.lse,
                             workspace=lay.fws, o_residual=res)

        def call():
            bsa.bsa_backward_into(q, k, v, lay.o, dout, lay.lse, w.blk, lay.row_ptr, lay.col_idx,
                                  dq, dk, dv, 0.0, ws, o_residual=res)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        call()
    b.record()
    torch.cuda.synchronize()
    check_status(bsa, f"after {args.profile}")
    print(json.dumps({"profile": args.profile, "workload": w.name, "calls": args.steps,
                      "ms_per_call": a.elapsed_time(b) / args.steps}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="bsa", choices=["bsa", "reference"])
    ap.add_argument("--workload", default="wan", choices=["wan", "cog", "hunyuan", "tiny", "tile3d", "sweep"])
    ap.add_argument("--keep", type=float, default=0.1, help="sweep: keep ratio of the top-k mask")
    ap.add_argument("--blk", type=int, default=64, help="sweep: block size")
    ap.add_argument("--ref-heads", type=int, default=12,
                    help="heads in the cpu_baseline sample of the GPU arm")
    ap.add_argument("--ref-heads-per-step", type=int, default=1,
                    help="heads per step of the --impl reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other layers, the sweep and the backward (1 GPU only)")
    ap.add_argument("--extra-steps", type=int, default=5, help="timed steps of each extra layer")
    ap.add_argument("--profile", choices=["mask", "forward", "backward"], default=None,
                    help="run only this op of the workload back to back, for a profiler (1 GPU)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.profile is not None:
        run_profile(args)
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_gpu(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
