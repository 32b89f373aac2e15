// pattern.cuh -- fixed block masks as CSR.
//
// Sparse-vDiT blog, "四种注意力模式": M0 full, M1 skip (output zero), M2 diagonal
// (intra-frame), M3 multi-diagonal (evenly spaced, cross-frame), M4 vertical
// stripe (global tokens); Efficient-vDiT blog, "3.1 注意力图块化": block-wise
// repetition of the 3D attention map (frame tiles).  The rule for each pattern
// is stated on token pairs (see include/bsa.h); below, each row's kept blocks
// are runs of consecutive blocks in closed form from the token ranges.
//
// Two kernels: one CTA per head computes the rows' counts in closed form and
// writes row_ptr (offsets from per-pattern totals and a block scan), then each
// warp writes a few rows of one head as runs of consecutive block ids
// (coalesced), once per batch index (the pattern does not depend on b).  The
// output is write-bound.
#pragma once
#include "common.cuh"

namespace bsa {

constexpr int kMaxPatternHeads = 1024;

struct PatternParams {
  int B, H, N, blk, nb;
  int lblk;                       // log2(blk): blk is a power of two
  int band_w, frame_tokens, f_lo, f_hi, stripe_blocks, tile_global_frames;
  int32_t* row_ptr;
  int32_t* col_idx;
  long long capacity;
  int8_t head_pattern[kMaxPatternHeads];
};

// ------------------------------------------------------------------ intervals
// Every rule keeps, for q-block i, a union of a few runs of consecutive
// kv-blocks, given in closed form by the two blocks' token ranges:
//   diag       one run [i - w, i + w];
//   multidiag  one run per frame offset f (the blocks whose offsets u - t can
//              meet [fS - w blk, fS + w blk]);
//   stripe     one run per frame t (the blocks holding tokens [tS, tS + sb blk));
//   tile3d     the blocks sharing a frame with block i, and those holding a
//              token of the first g frames.
// The runs come in ascending order of their first block; touching or
// overlapping runs are merged, so `emit(j0, j1)` sees disjoint ascending runs
// [j0, j1] and the row's blocks are exactly their union.  With stripe_blocks
// = 0 a frame has no stripe tokens and the stripe rule keeps nothing.
// 32-bit arithmetic throughout: N < 2^23 (nb^2 < 2^31 per head, blk <= 128),
// band widths are at most 2^24 tokens and frames at most 2^28 (checked on the
// host), stripe_blocks <= nb and tile_global_frames <= the number of frames
// (clamped on the host; neither clamp changes a mask).  The frame offsets are
// clamped to those whose run can reach [0, nb) before any product f S.
__device__ __forceinline__ int floor_div(int a, int b) { return a >= 0 ? a / b : -((-a + b - 1) / b); }

// floor(a / blk): an arithmetic shift, blk being a power of two
__device__ __forceinline__ int blk_floor(const PatternParams& p, int a) { return a >> p.lblk; }

// Smallest kv-block j whose last token is >= a (nb when none).
__device__ __forceinline__ int first_block_ending_at_or_after(const PatternParams& p, int a) {
  int j = blk_floor(p, a);   // (j+1) blk - 1 >= a  <=>  j >= floor(a / blk)
  if (j < 0) j = 0;
  if (j >= p.nb - 1) return (p.N - 1 >= a) ? p.nb - 1 : p.nb;
  return j;
}

template <typename Emit>
__device__ __forceinline__ void pattern_runs(const PatternParams& p, int pattern, int i,
                                             Emit&& emit) {
  const int nb = p.nb, blk = p.blk, S = p.frame_tokens;
  int ps = -1, pe = -2;   // pending run
  auto add = [&](int j0, int j1) {
    if (j0 < 0) j0 = 0;
    if (j1 > nb - 1) j1 = nb - 1;
    if (j0 > j1) return;
    if (ps >= 0 && j0 <= pe + 1) {
      if (j1 > pe) pe = j1;
      return;
    }
    if (ps >= 0) emit(ps, pe);
    ps = j0;
    pe = j1;
  };
  const int ti_lo = i * blk, ti_hi = min(p.N, ti_lo + blk) - 1;
  switch (pattern) {
    case BSA_PATTERN_FULL:
      add(0, nb - 1);
      break;
    case BSA_PATTERN_SKIP:
      break;
    case BSA_PATTERN_DIAG:
      add(i - p.band_w, i + p.band_w);
      break;
    case BSA_PATTERN_MULTIDIAG: {
      // offsets u - t over the two blocks form [uj_lo - ti_hi, uj_hi - ti_lo];
      // it meets [c - wb, c + wb] (c = f S) iff uj_lo <= c + wb + ti_hi and
      // uj_hi >= c - wb + ti_lo; only the f whose run can reach [0, nb) matter
      const int wb = p.band_w * blk;
      int f0 = p.f_lo, f1 = p.f_hi;
      const int fa = -floor_div(wb + ti_hi, S);                 // ceil((-wb - ti_hi) / S)
      const int fb = floor_div(p.N - 1 + wb - ti_lo, S);
      if (f0 < fa) f0 = fa;
      if (f1 > fb) f1 = fb;
      for (int f = f0; f <= f1; ++f) {
        const int c = f * S;
        add(first_block_ending_at_or_after(p, c - wb + ti_lo), blk_floor(p, c + wb + ti_hi));
      }
      break;
    }
    case BSA_PATTERN_STRIPE: {
      const int L = p.stripe_blocks * blk;
      if (L <= 0) break;
      if (L >= S) {   // every token of every frame is a stripe token
        add(0, nb - 1);
        break;
      }
      for (int t0 = 0; t0 < p.N; t0 += S) add(blk_floor(p, t0), blk_floor(p, min(p.N, t0 + L) - 1));
      break;
    }
    case BSA_PATTERN_TILE3D: {
      if (p.tile_global_frames > 0)   // blocks holding a token of the first g frames
        add(0, blk_floor(p, min(p.N, p.tile_global_frames * S) - 1));
      const int fi_lo = ti_lo / S, fi_hi = ti_hi / S;
      add(first_block_ending_at_or_after(p, fi_lo * S), blk_floor(p, min(p.N, (fi_hi + 1) * S) - 1));
      break;
    }
    default:
      break;
  }
  if (ps >= 0) emit(ps, pe);
}

__device__ __forceinline__ int pattern_count(const PatternParams& p, int pattern, int i) {
  int n = 0;
  pattern_runs(p, pattern, i, [&](int j0, int j1) { n += j1 - j0 + 1; });
  return n;
}

// Row counts with the vertical stripe's taken once: its rows do not depend on
// the q-block (every row keeps the stripe tokens of every frame).
struct PatternCounter {
  int stripe;
  __device__ __forceinline__ explicit PatternCounter(const PatternParams& p)
      : stripe(pattern_count(p, BSA_PATTERN_STRIPE, 0)) {}
  __device__ __forceinline__ int operator()(const PatternParams& p, int pattern, int i) const {
    return pattern == BSA_PATTERN_STRIPE ? stripe : pattern_count(p, pattern, i);
  }
};

constexpr int kPatternScanThreads = 1024;
constexpr int kPatternIds = BSA_PATTERN_TILE3D + 1;

// One CTA per head h: the row counts in closed form, their prefix within the
// head, and the head's offset from the totals of the patterns of the heads
// before it (each pattern's total is computed once) -> row_ptr of every row
// (b, h, i), for all b.  No scratch memory is needed.  A total past INT32_MAX
// is recorded as BSA_ERR_CAPACITY.
__global__ void __launch_bounds__(kPatternScanThreads) pattern_rowptr_kernel(
    const __grid_constant__ PatternParams p) {
  __shared__ long long s_tot[kPatternIds];
  __shared__ long long s_warp[kPatternScanThreads / 32];
  __shared__ long long s_carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.x;
  if (tid < kPatternIds) s_tot[tid] = 0;
  const PatternCounter count(p);
  __syncthreads();
  // totals of the patterns in use
  bool used[kPatternIds] = {};
  for (int hh = 0; hh < p.H; ++hh) used[p.head_pattern[hh]] = true;
  for (int pid = 0; pid < kPatternIds; ++pid) {
    if (!used[pid]) continue;
    long long part = 0;
    for (int i = tid; i < p.nb; i += kPatternScanThreads) part += count(p, pid, i);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) atomicAdd(reinterpret_cast<unsigned long long*>(&s_tot[pid]),
                             static_cast<unsigned long long>(part));
  }
  __syncthreads();
  long long base = 0, total = 0;
  for (int hh = 0; hh < p.H; ++hh) {
    const long long t = s_tot[p.head_pattern[hh]];
    if (hh < h) base += t;
    total += t;
  }
  if ((long long)p.B * total > 0x7fffffffLL) {
    if (tid == 0) record_error(BSA_ERR_CAPACITY);
    return;
  }
  // prefix over the head's rows, kPatternScanThreads rows at a time
  const int pid = p.head_pattern[h];
  if (tid == 0) s_carry = 0;
  __syncthreads();
  for (int i0 = 0; i0 < p.nb; i0 += kPatternScanThreads) {
    const int i = i0 + tid;
    const long long c = i < p.nb ? count(p, pid, i) : 0;
    long long incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const long long w = s_warp[lane];
      long long wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long v = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += v;
      }
      s_warp[lane] = wi - w;
    }
    __syncthreads();
    const long long carry = s_carry;
    const long long end = carry + s_warp[warp] + incl;   // inclusive, within the head
    if (i < p.nb)
      for (int b = 0; b < p.B; ++b)
        p.row_ptr[((long long)b * p.H + h) * p.nb + i + 1] =
            static_cast<int32_t>((long long)b * total + base + end);
    __syncthreads();
    if (tid == kPatternScanThreads - 1) s_carry = end;
    __syncthreads();
  }
  if (h == 0 && tid == 0) p.row_ptr[0] = 0;
}

// Rows of one head per CTA (kPatternRowsPerWarp consecutive rows per warp),
// every b: each row's runs written as consecutive block ids from the row's
// start, coalesced, 32-bit offsets from the row's start (nnz < 2^31).  The
// rows of the full and vertical-stripe patterns do not depend on the q-block:
// a full row is 0..nb-1 and the stripe row is built once per CTA in shared
// memory (when it fits) and copied.  Nothing past the capacity is written.
constexpr int kPatternRowsPerWarp = 4;
constexpr int kPatternWriteWarps = 8;
constexpr int kPatternRowSmem = 4096;   // stripe-row entries kept in shared memory
__global__ void __launch_bounds__(kPatternWriteWarps * 32) pattern_write_kernel(
    const __grid_constant__ PatternParams p) {
  __shared__ int32_t s_row[kPatternRowSmem];
  __shared__ int s_len;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = blockIdx.y;
  const int pattern = p.head_pattern[h];
  const int i0 = (blockIdx.x * kPatternWriteWarps + warp) * kPatternRowsPerWarp;
  bool from_smem = false;
  int s_n = 0;
  if (pattern == BSA_PATTERN_STRIPE) {   // uniform over the CTA
    if (warp == 0) {
      int pos = 0;
      pattern_runs(p, pattern, 0, [&](int j0, int j1) {
        const int n = j1 - j0 + 1;
        for (int k = lane; k < n; k += 32)
          if (pos + k < kPatternRowSmem) s_row[pos + k] = j0 + k;
        pos += n;
      });
      if (lane == 0) s_len = pos;
    }
    __syncthreads();
    s_n = s_len;
    from_smem = s_n <= kPatternRowSmem;
  }
  for (int r = 0; r < kPatternRowsPerWarp; ++r) {
    const int i = i0 + r;
    if (i >= p.nb) break;
    for (int b = 0; b < p.B; ++b) {
      const long long row = ((long long)b * p.H + h) * p.nb + i;
      const long long start = p.row_ptr[row], end = p.row_ptr[row + 1];
      const long long lim = end < p.capacity ? end : p.capacity;
      const int room = lim > start ? static_cast<int>(lim - start) : 0;   // entries it may write
      if (lim < end && lane == 0) record_error(BSA_ERR_CAPACITY);
      if (room == 0) continue;
      int32_t* out = p.col_idx + start;
      if (pattern == BSA_PATTERN_FULL) {
        const int n = min(room, p.nb);
        for (int k = lane; k < n; k += 32) out[k] = k;
      } else if (from_smem) {
        const int n = min(room, s_n);
        for (int k = lane; k < n; k += 32) out[k] = s_row[k];
      } else {
        int pos = 0;
        pattern_runs(p, pattern, i, [&](int j0, int j1) {
          const int n = min(j1 - j0 + 1, room - pos);
          for (int k = lane; k < n; k += 32) out[pos + k] = j0 + k;
          pos += j1 - j0 + 1;
        });
      }
    }
  }
}

}  // namespace bsa
