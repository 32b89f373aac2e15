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
// write pass.  The output is write-bound.
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

__device__ __forceinline__ long long floor_div(long long a, long long b) {
  long long q = a / b;
  return (a % b != 0 && ((a < 0) != (b < 0))) ? q - 1 : q;
}

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
  const long long blk = p.blk, S = p.frame_tokens;
  const long long ti_lo = (long long)i * blk, ti_hi = min((long long)p.N, ti_lo + blk) - 1;
  const long long uj_lo = (long long)j * blk, uj_hi = min((long long)p.N, uj_lo + blk) - 1;
  if (pattern == BSA_PATTERN_MULTIDIAG) {
    // offsets u - t over the two blocks: [lo, hi]; a frame offset f is hit when
    // [lo, hi] meets [f*S - w*blk, f*S + w*blk]
    const long long lo = uj_lo - ti_hi, hi = uj_hi - ti_lo, wb = (long long)p.band_w * blk;
    long long fmin = -floor_div(-(lo - wb), S);  // ceil((lo - wb) / S)
    long long fmax = floor_div(hi + wb, S);
    fmin = max(fmin, (long long)p.f_lo);
    fmax = min(fmax, (long long)p.f_hi);
    return fmin <= fmax;
  }
  if (pattern == BSA_PATTERN_STRIPE) {
    const long long f = uj_lo / S;
    return (uj_lo - f * S) < (long long)p.stripe_blocks * blk || (f + 1) * S <= uj_hi;
  }
  if (pattern == BSA_PATTERN_TILE3D) {
    const long long fi_lo = ti_lo / S, fi_hi = ti_hi / S, fj_lo = uj_lo / S, fj_hi = uj_hi / S;
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
  const int nbatch = p.B;
  int pos = 0;
  for (int jb = j0; jb < j1; jb += 32) {
    const int j = jb + lane;
    const bool keep = j < j1 && pattern_keep(p, pattern, i, j);
    const unsigned m = __ballot_sync(0xffffffffu, keep);
    const int off = pos + __popc(m & ((1u << lane) - 1u));
    if (keep) {
      for (int b = 0; b < nbatch; ++b) {
        const long long r = ((long long)b * p.H + h) * p.nb + i;
        const long long at = (long long)p.row_ptr[r] + off;
        if (at < p.row_ptr[r + 1]) {
          if (at < p.capacity)
            p.col_idx[at] = j;
          else
            record_error(BSA_ERR_CAPACITY);
        }
      }
    }
    pos += __popc(m);
  }
}

}  // namespace bsa
