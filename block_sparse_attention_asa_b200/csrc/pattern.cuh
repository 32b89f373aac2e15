// pattern.cuh -- fixed block masks as CSR.
//
// Sparse-vDiT blog, "四种注意力模式": M0 full, M1 skip (output zero), M2 diagonal
// (intra-frame), M3 multi-diagonal (evenly spaced, cross-frame), M4 vertical
// stripe (global tokens); Efficient-vDiT blog, "3.1 注意力图块化": block-wise
// repetition of the 3D attention map (frame tiles).  The rule for each pattern
// is stated on token pairs (see include/bsa.h); below it is evaluated per block
// pair in closed form from the two blocks' token ranges.
//
// One warp per (h, q-block): lanes sweep the candidate kv-blocks, a ballot and
// a popcount prefix give each kept block its position, and the row is written
// once per batch index (the pattern does not depend on b).  Count pass, scan,
// write pass.  Full and diagonal rows are contiguous ranges and skip the
// per-block test; the output is write-bound.
#pragma once
#include "common.cuh"

namespace bsa {

constexpr int kMaxPatternHeads = 1024;

struct PatternParams {
  int B, H, N, blk, nb;
  int band_w, frame_tokens, f_lo, f_hi, stripe_blocks, tile_global_frames;
  int32_t* row_ptr;
  int32_t* col_idx;
  long long capacity;
  int8_t head_pattern[kMaxPatternHeads];
};

// Is kv-block j kept for q-block i under `pattern`?
__device__ __forceinline__ bool pattern_keep(const PatternParams& p, int pattern, int i, int j) {
  switch (pattern) {
    case BSA_PATTERN_FULL:
      return true;
    case BSA_PATTERN_SKIP:
      return false;
    case BSA_PATTERN_DIAG:
      return abs(i - j) <= p.band_w;
    default:
      break;
  }
  // token ranges of the two blocks (N < 2^31, so 32-bit arithmetic is exact)
  const int blk = p.blk, S = p.frame_tokens;
  const int ti_lo = i * blk, ti_hi = min(p.N, ti_lo + blk) - 1;
  const int uj_lo = j * blk, uj_hi = min(p.N, uj_lo + blk) - 1;
  if (pattern == BSA_PATTERN_MULTIDIAG) {
    // offsets u - t over the two blocks: [lo, hi]; frame offset f is hit when
    // [lo, hi] meets [f*S - w*blk, f*S + w*blk] (a few f: no division)
    const long long lo = (long long)uj_lo - ti_hi, hi = (long long)uj_hi - ti_lo;
    const long long wb = (long long)p.band_w * blk;
    if (p.f_hi - p.f_lo <= 8) {
      for (int f = p.f_lo; f <= p.f_hi; ++f) {
        const long long c = (long long)f * S;
        if (lo <= c + wb && hi >= c - wb) return true;
      }
      return false;
    }
    // many offsets: the f range that [lo, hi] can reach, in closed form
    const long long a = lo - wb, bb = hi + wb;
    long long fmin = a >= 0 ? (a + S - 1) / S : -((-a) / S);    // ceil(a / S)
    long long fmax = bb >= 0 ? bb / S : -((-bb + S - 1) / S);   // floor(bb / S)
    fmin = max(fmin, (long long)p.f_lo);
    fmax = min(fmax, (long long)p.f_hi);
    return fmin <= fmax;
  }
  if (pattern == BSA_PATTERN_STRIPE) {
    const int f = uj_lo / S;
    return (long long)(uj_lo - f * S) < (long long)p.stripe_blocks * blk ||
           (long long)(f + 1) * S <= uj_hi;
  }
  if (pattern == BSA_PATTERN_TILE3D) {
    const int fi_lo = ti_lo / S, fi_hi = ti_hi / S, fj_lo = uj_lo / S, fj_hi = uj_hi / S;
    return (fj_lo <= fi_hi && fj_hi >= fi_lo) || fj_lo < p.tile_global_frames;
  }
  return false;
}

__device__ __forceinline__ void pattern_range(const PatternParams& p, int pattern, int i, int& j0,
                                              int& j1) {
  j0 = 0;
  j1 = p.nb;
  if (pattern == BSA_PATTERN_SKIP) {
    j1 = 0;
  } else if (pattern == BSA_PATTERN_DIAG) {
    j0 = max(0, i - p.band_w);
    j1 = min(p.nb, i + p.band_w + 1);
  }
}

// kWrite = false: store the row's count at row_ptr[r+1] for every b.
// kWrite = true : write col_idx[row_ptr[r] ...] for every b.
template <bool kWrite>
__global__ void __launch_bounds__(256) pattern_kernel(const __grid_constant__ PatternParams p) {
  const int lane = threadIdx.x & 31;
  const long long unit = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (unit >= (long long)p.H * p.nb) return;
  const int h = static_cast<int>(unit / p.nb), i = static_cast<int>(unit % p.nb);
  const int pattern = p.head_pattern[h];
  int j0, j1;
  pattern_range(p, pattern, i, j0, j1);
  if (!kWrite) {
    int cnt = 0;
    if (pattern == BSA_PATTERN_FULL || pattern == BSA_PATTERN_SKIP || pattern == BSA_PATTERN_DIAG) {
      cnt = j1 - j0;
    } else {
      for (int j = j0 + lane; j < j1; j += 32) cnt += pattern_keep(p, pattern, i, j) ? 1 : 0;
      cnt = warp_sum(cnt);
    }
    if (lane == 0)
      for (int b = 0; b < p.B; ++b) p.row_ptr[((long long)b * p.H + h) * p.nb + i + 1] = cnt;
    return;
  }
  // Full and diagonal rows are one contiguous range: no per-block test.  The
  // row's bounds are read once per batch index, outside the block sweep.
  const bool contiguous = pattern == BSA_PATTERN_FULL || pattern == BSA_PATTERN_DIAG;
  const unsigned lt = (1u << lane) - 1u;
  for (int b = 0; b < p.B; ++b) {
    const long long r = ((long long)b * p.H + h) * p.nb + i;
    const long long base = p.row_ptr[r], end = p.row_ptr[r + 1];
    int pos = 0;
    for (int jb = j0; jb < j1; jb += 32) {
      const int j = jb + lane;
      const bool keep = j < j1 && (contiguous || pattern_keep(p, pattern, i, j));
      const unsigned m = __ballot_sync(0xffffffffu, keep);
      if (keep) {
        const long long at = base + pos + __popc(m & lt);
        if (at < end) {
          if (at < p.capacity)
            p.col_idx[at] = j;
          else
            record_error(BSA_ERR_CAPACITY);
        }
      }
      pos += __popc(m);
    }
  }
}

}  // namespace bsa
