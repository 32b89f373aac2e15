"""Seeded synthetic workloads shaped like the video-DiT attention layers on the pages.

This module is the only code shared by the CUDA path and the fp64 oracle.  It
draws inputs and describes shapes; it holds none of the method's arithmetic
(no pooling, no scores, no selection, no attention).

Inputs: ``numpy.random.default_rng(seed).standard_normal(float32)`` drawn in the
order q, k, v, each ``[B, H, N, d]``; then ``scale * x + PE`` and a
round-to-nearest-even cast to bfloat16 (``torch.Tensor.to``).  The position
embedding is a 3D sinusoid of the token's (t, y, x) coordinate in frame-major
order (x fastest), the usual transformer sinusoid per axis:

* ``d`` is split into ``d_t = d - 2*d_y`` and ``d_y = d_x = 2*floor(d/6)``
  (44/42/42 for d=128, 24/20/20 for d=64), concatenated as [t | y | x];
* an axis part of width ``m`` at position ``p`` is
  ``[sin(p / 10000**(2k/m)) for k < m/2] + [cos(p / 10000**(2k/m)) for k < m/2]``.

Text tokens (the CogVideoX-shaped joint layer puts 226 of them in front of the
video tokens) get no embedding.  The pages fix none of this; it only has to give
the inputs the spatio-temporal structure that content-aware masks react to.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

# Mask-source ids used by the pattern generator (Sparse-vDiT blog, "四种注意力模式"
# table: M0 full, M1 skip, M2 diagonal, M3 multi-diagonal, M4 vertical stripe;
# Efficient-vDiT blog, "3.1 注意力图块化": the 3D attention tile).
PATTERN_FULL = 0
PATTERN_SKIP = 1
PATTERN_DIAG = 2
PATTERN_MULTIDIAG = 3
PATTERN_STRIPE = 4
PATTERN_TILE3D = 5
PATTERN_NAMES = {
    PATTERN_FULL: "full",
    PATTERN_SKIP: "skip",
    PATTERN_DIAG: "diag",
    PATTERN_MULTIDIAG: "multidiag",
    PATTERN_STRIPE: "stripe",
    PATTERN_TILE3D: "tile3d",
}

MODE_TOPK = 0
MODE_MASS = 1


@dataclass(frozen=True)
class Workload:
    """Shape, input recipe and mask parameters of one attention layer."""

    name: str
    B: int
    H: int
    d: int
    frames: int          # latent T
    height: int          # latent H (rows of a frame)
    width: int           # latent W (tokens per row, fastest)
    blk: int
    seed: int
    scale: float = 0.5   # multiplier on the N(0,1) draw
    pe: bool = True      # add the 3D sinusoidal embedding to video tokens
    n_text: int = 0      # text tokens in front of the video tokens
    # mask source: "asa" or "pattern"
    source: str = "asa"
    # ASA parameters
    mode: int = MODE_TOPK
    topk: int = 0
    mass_tau: float = 0.0
    max_keep_ratio: float = 0.0
    keep_diag: int = 0
    n_sink_blocks: int = 0
    # fixed-pattern parameters
    head_pattern: Optional[tuple] = None
    band_w: int = 2
    f_lo: int = -2
    f_hi: int = 2
    stripe_blocks: int = 4
    tile_global_frames: int = 1
    extra: dict = field(default_factory=dict)

    @property
    def frame_tokens(self) -> int:
        return self.height * self.width

    @property
    def N(self) -> int:
        return self.n_text + self.frames * self.height * self.width

    @property
    def nb(self) -> int:
        return -(-self.N // self.blk)


def largest_remainder(total: int, percents) -> list:
    """Integer counts summing to ``total`` in proportion to ``percents``."""
    raw = [total * p / 100.0 for p in percents]
    counts = [int(np.floor(r)) for r in raw]
    left = total - sum(counts)
    order = sorted(range(len(raw)), key=lambda i: (-(raw[i] - counts[i]), i))
    for i in order[:left]:
        counts[i] += 1
    return counts


def assign_head_patterns(H: int, seed: int, shares=((PATTERN_SKIP, 5), (PATTERN_DIAG, 30),
                                                    (PATTERN_MULTIDIAG, 30), (PATTERN_STRIPE, 20),
                                                    (PATTERN_FULL, 15))) -> tuple:
    """Per-head pattern ids: largest-remainder counts, then a seeded permutation."""
    counts = largest_remainder(H, [s for _, s in shares])
    pool = []
    for (pid, _), c in zip(shares, counts):
        pool += [pid] * c
    perm = np.random.default_rng(seed).permutation(H)
    return tuple(int(pool[j]) for j in perm)


def _axis_sinusoid(pos: np.ndarray, m: int) -> np.ndarray:
    half = m // 2
    k = np.arange(half, dtype=np.float64)
    inv = 1.0 / (10000.0 ** (2.0 * k / m))
    ang = pos[:, None].astype(np.float64) * inv[None, :]
    return np.concatenate([np.sin(ang), np.cos(ang)], axis=1)


def position_embedding(frames: int, height: int, width: int, d: int) -> np.ndarray:
    """[frames*height*width, d] float64 3D sinusoid in frame-major token order."""
    dy = 2 * (d // 6)
    dt = d - 2 * dy
    n = frames * height * width
    tok = np.arange(n)
    t = tok // (height * width)
    y = (tok // width) % height
    x = tok % width
    return np.concatenate([_axis_sinusoid(t, dt), _axis_sinusoid(y, dy), _axis_sinusoid(x, dy)], axis=1)


def make_qkv(w: Workload, seed: Optional[int] = None, B: Optional[int] = None, H: Optional[int] = None):
    """Seeded bf16 q, k, v (torch CPU tensors, [B, H, N, d], contiguous)."""
    import torch

    B = w.B if B is None else B
    H = w.H if H is None else H
    rng = np.random.default_rng(w.seed if seed is None else seed)
    shape = (B, H, w.N, w.d)
    pe = None
    if w.pe:
        pe = position_embedding(w.frames, w.height, w.width, w.d).astype(np.float32)
    out = []
    for _ in range(3):
        x = rng.standard_normal(shape, dtype=np.float32)
        if w.scale != 1.0:
            x *= np.float32(w.scale)
        if pe is not None:
            x[:, :, w.n_text:, :] += pe[None, None]
        out.append(torch.from_numpy(x).to(torch.bfloat16).contiguous())
    return tuple(out)


def as_f64(t) -> np.ndarray:
    """bf16 torch tensor -> float64 numpy array (exact widening)."""
    import torch

    return t.to(torch.float32).numpy().astype(np.float64)


# ---------------------------------------------------------------------------
# The layers.  Shapes follow the pages' models (Wan2.1-1.3B, CogVideoX-5B,
# HunyuanVideo); the mask parameters are the ones the workloads are quoted on.
# ---------------------------------------------------------------------------

TINY = Workload(name="tiny_asa", B=1, H=2, d=64, frames=2, height=8, width=8, blk=16, seed=0,
                scale=0.5, mode=MODE_TOPK, topk=3, keep_diag=1)

WAN = Workload(name="wan2.1_1.3b_asa", B=1, H=12, d=128, frames=21, height=30, width=52, blk=64,
               seed=1, scale=0.5, mode=MODE_MASS, mass_tau=0.9, max_keep_ratio=0.1)

COG = Workload(name="cogvideox_5b_asa", B=2, H=48, d=64, frames=13, height=30, width=45, blk=64,
               seed=2, scale=1.0, n_text=226, mode=MODE_TOPK, topk=(278 * 12) // 100,
               n_sink_blocks=-(-226 // 64))

HUNYUAN = Workload(name="hunyuanvideo_patterns", B=1, H=24, d=128, frames=33, height=45, width=80,
                   blk=64, seed=3, scale=1.0, pe=False, source="pattern",
                   head_pattern=assign_head_patterns(24, 3 + 1000), band_w=2, f_lo=-2, f_hi=2,
                   stripe_blocks=4)


# The Efficient-vDiT 3D attention tile ("3.1 注意力图块化") on the Wan shape:
# every head keeps the blocks that share a frame with the query block, plus the
# blocks of the first frame (one global frame), in the given token order.
WAN_TILE3D = Workload(name="wan2.1_1.3b_tile3d", B=1, H=12, d=128, frames=21, height=30,
                      width=52, blk=64, seed=1, scale=0.5, source="pattern",
                      head_pattern=tuple([PATTERN_TILE3D] * 12), tile_global_frames=1)


def sweep(keep: float, blk: int) -> Workload:
    """Wan-shaped layer, top-k with k = floor(keep * nb)."""
    nb = -(-(21 * 30 * 52) // blk)
    return Workload(name=f"wan_sweep_keep{keep}_blk{blk}", B=1, H=12, d=128, frames=21, height=30,
                    width=52, blk=blk, seed=1, scale=0.5, mode=MODE_TOPK,
                    topk=max(1, int(np.floor(keep * nb))))


SWEEP_KEEPS = (1.0, 0.5, 0.25, 0.1, 0.05)
SWEEP_BLKS = (64, 128)
ALL = {w.name: w for w in (TINY, WAN, COG, HUNYUAN, WAN_TILE3D)}
