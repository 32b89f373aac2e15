"""The seeded input generator (block_sparse_attention_asa_b200/workloads.py)
follows the recipe the design states (CPU):

* layer sizes: Wan N 32760 (nb 512, last block 56), CogVideoX N 17776
  (226 text + 13x30x45, nb 278, last 48), HunyuanVideo N 118800 (nb 1857,
  last 16); Cog's top-k is floor(0.12 * 278) = 33 with text sinks 0..3;
* PE: d split as d_t = d - 2*d_y, d_y = d_x = 2*floor(d/6) (24/20/20 at 64,
  44/42/42 at 128); each part is [sin | cos] of p / 10000^(2k/m); tokens in
  frame-major order (t, y, x), x fastest; the t part depends on t alone, etc.;
* make_qkv: scale * N(0,1) + PE on video tokens only, cast to bf16, seeded
  and repeatable, q, k, v drawn in that order;
* Hunyuan heads: largest-remainder counts of 24 x {5, 30, 30, 20, 15}% =
  {skip 1, diag 7, multi 7, stripe 5, full 4}, permuted by the seeded
  generator.
"""
import math

import numpy as np
import torch

from block_sparse_attention_asa_b200 import workloads as W


def test_layer_sizes():
    assert (W.WAN.N, W.WAN.nb, W.WAN.N - (W.WAN.nb - 1) * 64) == (32760, 512, 56)
    assert (W.COG.N, W.COG.nb, W.COG.N - (W.COG.nb - 1) * 64) == (17776, 278, 48)
    assert (W.HUNYUAN.N, W.HUNYUAN.nb, W.HUNYUAN.N - (W.HUNYUAN.nb - 1) * 64) == (118800, 1857, 16)
    assert W.COG.topk == 33 and W.COG.n_sink_blocks == 4 and W.COG.n_text == 226
    assert W.TINY.N == 128 and W.TINY.nb == 8


def test_position_embedding_splits_and_axes():
    for d, (dt, dy) in ((64, (24, 20)), (128, (44, 42))):
        F, Hh, Ww = 3, 4, 5
        pe = W.position_embedding(F, Hh, Ww, d)
        assert pe.shape == (F * Hh * Ww, d)
        t_part, y_part, x_part = pe[:, :dt], pe[:, dt:dt + dy], pe[:, dt + dy:]
        assert x_part.shape[1] == dy
        for tok in range(F * Hh * Ww):
            t, y, x = tok // (Hh * Ww), (tok // Ww) % Hh, tok % Ww
            # each part depends on its own coordinate only
            assert np.array_equal(t_part[tok], t_part[t * Hh * Ww])
            assert np.array_equal(y_part[tok], y_part[y * Ww])
            assert np.array_equal(x_part[tok], x_part[x])
        # position 0: sines 0, cosines 1
        for part, m in ((t_part, dt), (y_part, dy), (x_part, dy)):
            assert np.all(part[0, :m // 2] == 0.0) and np.all(part[0, m // 2:] == 1.0)
        # the first frequency of the x part is 1 (k = 0): sin(x), cos(x)
        xs = np.arange(Ww)
        np.testing.assert_allclose(x_part[xs, 0], np.sin(xs), atol=1e-15)
        np.testing.assert_allclose(x_part[xs, dy // 2], np.cos(xs), atol=1e-15)
        # the last frequency of the t part is 10000^(-2(m/2-1)/m)
        k = dt // 2 - 1
        f = 10000.0 ** (-2.0 * k / dt)
        np.testing.assert_allclose(t_part[Hh * Ww, k], math.sin(f), atol=1e-15)


def test_make_qkv_recipe():
    # scale 0: the draw vanishes, leaving bf16(PE) on video tokens and 0 on text
    w = W.Workload(name="probe", B=1, H=2, d=64, frames=2, height=3, width=4, blk=16, seed=5,
                   scale=0.0, n_text=7)
    q, k, v = W.make_qkv(w)
    assert q.dtype == torch.bfloat16 and q.shape == (1, 2, 7 + 24, 64) and q.is_contiguous()
    pe = torch.from_numpy(W.position_embedding(2, 3, 4, 64).astype(np.float32)).to(torch.bfloat16)
    for t in (q, k, v):
        assert torch.all(t[:, :, :7] == 0)
        assert torch.equal(t[0, 0, 7:], pe) and torch.equal(t[0, 1, 7:], pe)
    # seeded and repeatable; q, k, v are successive draws of one generator
    w1 = W.Workload(name="probe", B=1, H=2, d=64, frames=2, height=3, width=4, blk=16, seed=5,
                    scale=1.0, pe=False)
    a = W.make_qkv(w1)
    b = W.make_qkv(w1)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    rng = np.random.default_rng(5)
    for x in a:
        want = torch.from_numpy(rng.standard_normal((1, 2, 24, 64), dtype=np.float32))
        assert torch.equal(x, want.to(torch.bfloat16))


def test_hunyuan_head_assignment():
    assert W.largest_remainder(24, [5, 30, 30, 20, 15]) == [1, 7, 7, 5, 4]
    hp = W.HUNYUAN.head_pattern
    assert len(hp) == 24
    counts = {p: hp.count(p) for p in set(hp)}
    assert counts == {W.PATTERN_SKIP: 1, W.PATTERN_DIAG: 7, W.PATTERN_MULTIDIAG: 7,
                      W.PATTERN_STRIPE: 5, W.PATTERN_FULL: 4}
    pool = [W.PATTERN_SKIP] + [W.PATTERN_DIAG] * 7 + [W.PATTERN_MULTIDIAG] * 7 + \
        [W.PATTERN_STRIPE] * 5 + [W.PATTERN_FULL] * 4
    perm = np.random.default_rng(3 + 1000).permutation(24)
    assert hp == tuple(pool[j] for j in perm)
