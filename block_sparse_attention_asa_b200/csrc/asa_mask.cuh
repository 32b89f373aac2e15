// asa_mask.cuh -- BLADE's Adaptive Block-Sparse Attention mask on sm_100a.
//
// BLADE digest (abstract; 方法详解 / 关键设计): ASA builds, per input, a mask that
// keeps the block pairs whose mutual relevance is high.  Reading used here
// (documented in include/bsa.h): mean-pool Q and K per token block, softmax of
// the pooled scores over all kv-blocks, keep by top-k or by the shortest prefix
// reaching a cumulative mass, ties to the lower block index, optional cap and
// forced blocks, CSR out.
//
// Kernels, in launch order:
//   asa_pool_kernel     HBM-bound: streams Q and K once (16-byte loads, fp32
//                       accumulation in a fixed order, one small CTA per
//                       block), writes q̄ [row][d] and k̄ transposed,
//                       k̄ᵀ [bh][d][nb padded to 4].
//   asa_select_kernel   nb <= 1024.  Per CTA, R q-block rows of one (b, h):
//                       the score tile S = q̄ k̄ᵀ as a register-blocked fp32
//                       GEMM (k̄ᵀ streamed through shared memory by cp.async,
//                       double-buffered), then one warp per row with the row's
//                       probabilities in registers: softmax, and the cut found
//                       by bisection over the 32-bit order key with warp
//                       reductions -> selection bitmap and count.
//   asa_select_generic_kernel   any nb: the same arithmetic with the row kept in
//                       shared memory and a radix select on the 64-bit key.
//                       Both select kernels then write the CSR themselves: a
//                       CTA takes its rows in the order of a ticket counter,
//                       publishes its rows' total, finds the total of all
//                       earlier rows by a decoupled look-back over the earlier
//                       CTAs' published totals, writes its row_ptr entries and
//                       expands its bitmaps into ascending col_idx.
#pragma once
#include "common.cuh"
#include "ptx.cuh"
#include <cuda_bf16.h>

namespace bsa {

// ------------------------------------------------------------------ pooling
// One CTA of kPoolWarps warps per (tensor, b, h, block): warp w sums rows
// [w*RW, w*RW + RW) of the block (RW = blk / kPoolWarps rounded up), lane l
// reading 16 bytes (8 elements) of a row, D/8 lanes per row, all of a warp's
// loads issued before the first add.  Partial sums combine in a fixed order
// (rows of a lane, then the lanes of a row group by butterfly, then the warps
// in index order), so the result is deterministic.  Many small CTAs keep the
// HBM stream even to the last wave.
constexpr int kPoolWarps = 4;

template <int D, int BLK>
__global__ void __launch_bounds__(kPoolWarps * 32) asa_pool_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    float* __restrict__ qbar, float* __restrict__ kbarT, int BH, int N, int nb, int kt_ld,
    unsigned long long* __restrict__ scan_flags, unsigned int* __restrict__ scan_ticket,
    int n_flags) {
  // the select kernel's look-back state starts at zero (the grid has more CTAs
  // than there are flags)
  if (threadIdx.x == 0) {
    if (blockIdx.x < static_cast<unsigned>(n_flags)) scan_flags[blockIdx.x] = 0ull;
    if (blockIdx.x == 0) *scan_ticket = 0u;
  }
  constexpr int blk = BLK;
  constexpr int LPR = D / 8;          // lanes per row
  constexpr int RPS = 32 / LPR;       // rows per warp step
  __shared__ float part[kPoolWarps][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long unit = blockIdx.x;
  const bool is_k = unit >= (long long)BH * nb;
  const long long u = is_k ? unit - (long long)BH * nb : unit;
  const long long bh = u / nb;
  const int i = static_cast<int>(u % nb);
  const int r0 = i * blk, nrows = min(blk, N - r0);
  constexpr int rw = (BLK + kPoolWarps - 1) / kPoolWarps;   // rows per warp
  const int wr0 = warp * rw, wr1 = min(nrows, wr0 + rw);
  const __nv_bfloat16* src = (is_k ? k : q) + (bh * N + r0) * D;
  const int sub = lane / LPR, col = (lane % LPR) * 8;
  float acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;
  constexpr int MAXSTEP = (rw + RPS - 1) / RPS;
  uint4 raw[MAXSTEP];
#pragma unroll
  for (int s = 0; s < MAXSTEP; ++s) {
    const int r = wr0 + sub + s * RPS;
    raw[s] = r < wr1 ? __ldg(reinterpret_cast<const uint4*>(src + (long long)r * D + col))
                     : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int s = 0; s < MAXSTEP; ++s) {
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[s]);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float2 f = __bfloat1622float2(h2[c]);
      acc[2 * c] += f.x;
      acc[2 * c + 1] += f.y;
    }
  }
  // combine the row groups (fixed butterfly order)
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], o);
  if (sub == 0) {
#pragma unroll
    for (int c = 0; c < 8; ++c) part[warp][col + c] = acc[c];
  }
  __syncthreads();
  // warps in index order; thread t < D finishes column t
  for (int c = threadIdx.x; c < D; c += kPoolWarps * 32) {
    float v = part[0][c];
#pragma unroll
    for (int w = 1; w < kPoolWarps; ++w) v += part[w][c];
    v /= static_cast<float>(nrows);
    if (!is_k)
      qbar[u * D + c] = v;
    else
      kbarT[(bh * D + c) * (long long)kt_ld + i] = v;
  }
}

// ------------------------------------------------------------------ select
struct SelectParams {
  const float* qbar;      // [BH*nb, D]
  const float* kbarT;     // [BH, D, kt_ld]: k̄ transposed, rows padded to kt_ld
  uint32_t* bitmaps;      // [BH*nb, nbw]
  int32_t* row_ptr;       // [BH*nb + 1]
  int32_t* col_idx;       // [capacity]
  long long capacity;
  unsigned long long* scan_flags;   // [CTAs]: per CTA (total << 2) | state, zeroed before launch
  unsigned int* scan_ticket;        // CTA order, zeroed before launch
  unsigned long long wait_ns;       // bound on the look-back wait
  int groups;             // CTAs per (b, h)
  int nb, nbw, rows_per_cta, nb_pad, kt_ld;
  int dk;                 // asa_select_kernel: k̄ᵀ rows per cp.async stage
  int mode, topk, cap, keep_diag, n_sink;
  float mass_tau, scale;
};

constexpr int kSelWarps = 8;
constexpr int kKChunk = 64;

// Order key: ascending key <=> (p descending, j ascending).  p >= 0, so its
// bit pattern orders like its value.
__device__ __forceinline__ unsigned long long order_key(float p, int j) {
  return (static_cast<unsigned long long>(0xFFFFFFFFu - __float_as_uint(p)) << 32) |
         static_cast<unsigned int>(j);
}

// The m-th smallest order key (1-based m, 1 <= m <= nb <= 65536) of the row
// `pr`, by an 8-bit-digit radix select over the key's significant bytes: the
// four bytes of the p bits, then -- only while elements with equal p remain to
// be split -- the two low bytes of the block index.
__device__ unsigned long long kth_key(const float* pr, int nb, int m, unsigned int* hist) {
  const int lane = threadIdx.x & 31;
  unsigned long long prefix = 0, pmask = 0;
  int remaining = m;
#pragma unroll 1
  for (int pass = 0; pass < 6; ++pass) {
    const int shift = pass < 4 ? 56 - 8 * pass : (pass == 4 ? 8 : 0);
    if (pass == 4) {
      // p settled; if exactly `remaining` elements carry it, take them all
      int eq = 0, last = -1;
      for (int j = lane; j < nb; j += 32)
        if ((order_key(pr[j], j) & pmask) == prefix) {
          ++eq;
          last = j;
        }
      eq = warp_sum(eq);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
      if (eq == remaining) return prefix | static_cast<unsigned int>(last);
    }
#pragma unroll
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int j = lane; j < nb; j += 32) {
      const unsigned long long key = order_key(pr[j], j);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncwarp();
    // lane owns bins [8*lane, 8*lane+8), ascending digit order
    int mine = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b) mine += hist[8 * lane + b];
    const int incl = warp_incl_scan(mine);
    const int excl = incl - mine;
    const unsigned who = __ballot_sync(0xffffffffu, excl < remaining && remaining <= incl);
    const int src = __ffs(who) - 1;
    int digit = 0, below = 0;
    if (lane == src) {
      int c = excl;
      for (int b = 0; b < 8; ++b) {
        const int hb = hist[8 * lane + b];
        if (c + hb >= remaining) {
          digit = 8 * lane + b;
          below = c;
          break;
        }
        c += hb;
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    below = __shfl_sync(0xffffffffu, below, src);
    __syncwarp();
    remaining -= below;
    prefix |= static_cast<unsigned long long>(digit) << shift;
    pmask |= 0xFFull << shift;
  }
  return prefix;
}

// Number of blocks the mass rule keeps: the shortest prefix (in key order)
// whose p sum reaches tau, looked for in chunks of 64 ranks, at most `limit`.
__device__ int mass_count(const float* pr, int nb, float tau, int limit, unsigned int* hist,
                          unsigned long long* buf) {
  const int lane = threadIdx.x & 31;
  float total = 0.f;
  unsigned long long k_lo = 0;  // keys <= k_lo are already counted
  bool have_lo = false;
#pragma unroll 1
  for (int done = 0; done < limit; done += 64) {
    const int upto = min(limit, done + 64);
    const unsigned long long k_hi = kth_key(pr, nb, upto, hist);
    // gather keys in (k_lo, k_hi]
    int n = 0;
    for (int jb = 0; jb < nb; jb += 32) {
      const int j = jb + lane;
      unsigned long long key = 0;
      bool in = false;
      if (j < nb) {
        key = order_key(pr[j], j);
        in = key <= k_hi && (!have_lo || key > k_lo);
      }
      const unsigned msk = __ballot_sync(0xffffffffu, in);
      if (in) buf[n + __popc(msk & ((1u << lane) - 1u))] = key;
      n += __popc(msk);
    }
    __syncwarp();
    // bitonic sort of 64 keys, element x = lane + 32*h
    unsigned long long e0 = lane < n ? buf[lane] : ~0ull;
    unsigned long long e1 = lane + 32 < n ? buf[lane + 32] : ~0ull;
    __syncwarp();
#pragma unroll
    for (int kk = 2; kk <= 64; kk <<= 1) {
#pragma unroll
      for (int jj = kk >> 1; jj > 0; jj >>= 1) {
        if (jj == 32) {
          // partner is the other register of the same lane (x and x+32)
          const bool asc = ((lane & kk) == 0);  // kk == 64 here: always ascending
          const unsigned long long lo = e0 < e1 ? e0 : e1, hi = e0 < e1 ? e1 : e0;
          e0 = asc ? lo : hi;
          e1 = asc ? hi : lo;
        } else {
          const unsigned long long p0 = __shfl_xor_sync(0xffffffffu, e0, jj);
          const unsigned long long p1 = __shfl_xor_sync(0xffffffffu, e1, jj);
          const bool lower = (lane & jj) == 0;
          const bool asc0 = ((lane & kk) == 0);
          const bool asc1 = (((lane + 32) & kk) == 0);
          e0 = (lower == asc0) ? (e0 < p0 ? e0 : p0) : (e0 < p0 ? p0 : e0);
          e1 = (lower == asc1) ? (e1 < p1 ? e1 : p1) : (e1 < p1 ? p1 : e1);
        }
      }
    }
    // p in sorted order; padding keys decode to p = 0
    const float p0 = __uint_as_float(0xFFFFFFFFu - static_cast<unsigned int>(e0 >> 32));
    const float p1 = __uint_as_float(0xFFFFFFFFu - static_cast<unsigned int>(e1 >> 32));
    const float s0 = warp_incl_scan_f(p0);
    const float t0 = __shfl_sync(0xffffffffu, s0, 31);
    const float s1 = warp_incl_scan_f(p1) + t0;
    const unsigned hit0 = __ballot_sync(0xffffffffu, lane < n && total + s0 >= tau);
    const unsigned hit1 = __ballot_sync(0xffffffffu, lane + 32 < n && total + s1 >= tau);
    if (hit0) return done + __ffs(hit0);
    if (hit1) return done + 32 + __ffs(hit1);
    total += __shfl_sync(0xffffffffu, s1, 31);
    k_lo = k_hi;
    have_lo = true;
  }
  return limit;
}

// The CTA that took ticket `lin` and owns rows [i0, i0 + nrow) of (b, h) = bh:
// its rows' counts (cnt, shared memory) are published, the total of every
// earlier row is found by a decoupled look-back, then row_ptr is written and
// the row bitmaps (already in global memory, written by this CTA) are expanded
// into ascending block ids.  Flag word per CTA: (total << 2) | state, state 1 =
// the CTA's own total, 2 = the total through this CTA.  A CTA waits only for
// CTAs with smaller tickets, which started before it, so the wait ends; it is
// bounded all the same (BSA_ERR_TIMEOUT).
__device__ __forceinline__ void csr_write_rows(const SelectParams& p, int lin, int bh, int i0,
                                               int nrow, const int* cnt, long long* s_base) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __syncthreads();   // counts and bitmaps of every row of the CTA are written
  if (warp == 0) {
    long long agg = 0;
    for (int r = lane; r < nrow; r += 32) agg += cnt[r];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) agg += __shfl_xor_sync(0xffffffffu, agg, o);
    volatile unsigned long long* fl = p.scan_flags;
    if (lane == 0) atomicExch(p.scan_flags + lin, (static_cast<unsigned long long>(agg) << 2) |
                                                      (lin == 0 ? 2ull : 1ull));
    long long prefix = 0;
    int j = lin - 1;   // nearest CTA not yet accounted for
    const uint64_t t0 = global_ns();
    while (j >= 0) {
      const int idx = j - lane;
      const unsigned long long f = idx >= 0 ? fl[idx] : 2ull;   // before CTA 0: total 0
      const unsigned st = static_cast<unsigned>(f & 3ull);
      const unsigned incl = __ballot_sync(0xffffffffu, st == 2u);
      const unsigned zero = __ballot_sync(0xffffffffu, st == 0u);
      const int stop = incl ? __ffs(incl) - 1 : 31;           // last lane to add
      const unsigned upto = stop == 31 ? 0xffffffffu : ((2u << stop) - 1u);
      if (zero & upto) {
        if (global_ns() - t0 > p.wait_ns) {
          if (lane == 0) record_error(BSA_ERR_TIMEOUT);
          break;
        }
        continue;
      }
      long long v = lane <= stop ? static_cast<long long>(f >> 2) : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      prefix += v;
      if (incl) break;
      j -= 32;
    }
    if (lin > 0 && lane == 0)
      atomicExch(p.scan_flags + lin, (static_cast<unsigned long long>(prefix + agg) << 2) | 2ull);
    if (lane == 0) *s_base = prefix;
  }
  __syncthreads();
  const long long base = *s_base;
  if (lin == 0 && tid == 0) p.row_ptr[0] = 0;
  // one warp per row: its end in row_ptr, its blocks in ascending order
  for (int rr = warp; rr < nrow; rr += kSelWarps) {
    long long before = 0;
    for (int r = 0; r < rr; ++r) before += cnt[r];
    long long pos = base + before;
    const long long row = (long long)bh * p.nb + i0 + rr;
    if (lane == 0) {
      const long long end = pos + cnt[rr];
      if (end > 0x7fffffffLL) record_error(BSA_ERR_CAPACITY);
      p.row_ptr[row + 1] = static_cast<int32_t>(end > 0x7fffffffLL ? 0x7fffffffLL : end);
    }
    const uint32_t* bmr = p.bitmaps + row * p.nbw;
    for (int w0 = 0; w0 < p.nbw; w0 += 32) {
      const int wd = w0 + lane;
      uint32_t word = wd < p.nbw ? bmr[wd] : 0u;
      const int c = __popc(word);
      const int incl = warp_incl_scan(c);
      long long at = pos + incl - c;
      while (word) {
        const int bit = __ffs(word) - 1;
        word &= word - 1;
        if (at < p.capacity)
          p.col_idx[at] = wd * 32 + bit;
        else
          record_error(BSA_ERR_CAPACITY);
        ++at;
      }
      pos += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(256) asa_select_generic_kernel(const SelectParams p) {
  extern __shared__ __align__(16) unsigned char sel_smem[];
  const int R = p.rows_per_cta;
  float* qs = reinterpret_cast<float*>(sel_smem);                  // [R][D]
  float* kc = qs + R * D;                                          // [64][D+1]
  float* sc = kc + kKChunk * (D + 1);                              // [R][nb_pad]
  unsigned int* hist = reinterpret_cast<unsigned int*>(sc + (size_t)R * p.nb_pad);  // [8][256]
  unsigned long long* buf =
      reinterpret_cast<unsigned long long*>(hist + kSelWarps * 256);  // [8][64]
  __shared__ int s_cnt[64];
  __shared__ long long s_base;
  __shared__ int s_lin;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_lin = static_cast<int>(atomicAdd(p.scan_ticket, 1u));
  __syncthreads();
  const int lin = s_lin;
  const int bh = lin / p.groups, i0 = (lin % p.groups) * R;
  const int nrow = min(R, p.nb - i0);
  const float* qrow = p.qbar + ((long long)bh * p.nb + i0) * D;
  const float* kbh = p.kbarT + (long long)bh * D * p.kt_ld;

  for (int e = tid; e < nrow * D; e += 256) qs[e] = qrow[e];
  // scores: thread (ty, tx) -> row ty, columns tx + 16*m of the chunk
  const int ty = tid >> 4, tx = tid & 15;
  for (int jc = 0; jc < p.nb; jc += kKChunk) {
    __syncthreads();
    const int nj = min(kKChunk, p.nb - jc);
    for (int e = tid; e < nj * D; e += 256) {
      const int dd = e / nj, jj = e - dd * nj;
      kc[jj * (D + 1) + dd] = kbh[(long long)dd * p.kt_ld + jc + jj];
    }
    __syncthreads();
    for (int rr = ty; rr < nrow; rr += 16) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      const float* qv = qs + rr * D;
#pragma unroll 8
      for (int dd = 0; dd < D; ++dd) {
        const float a = qv[dd];
#pragma unroll
        for (int m = 0; m < 4; ++m) acc[m] = fmaf(a, kc[(tx + 16 * m) * (D + 1) + dd], acc[m]);
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int jj = tx + 16 * m;
        if (jj < nj) sc[rr * p.nb_pad + jc + jj] = acc[m] * p.scale;
      }
    }
  }
  __syncthreads();

  unsigned int* myhist = hist + warp * 256;
  unsigned long long* mybuf = buf + warp * 64;
  for (int rr = warp; rr < nrow; rr += kSelWarps) {
    float* pr = sc + rr * p.nb_pad;
    const int i = i0 + rr;
    // softmax over all nb blocks (fixed reduction order)
    float mx = -INFINITY;
    for (int j = lane; j < p.nb; j += 32) mx = fmaxf(mx, pr[j]);
    mx = warp_max(mx);
    float sum = 0.f;
    for (int j = lane; j < p.nb; j += 32) {
      const float e = expf(pr[j] - mx);
      pr[j] = e;
      sum += e;
    }
    sum = warp_sum_f(sum);
    for (int j = lane; j < p.nb; j += 32) pr[j] = pr[j] / sum;
    __syncwarp();
    int m;
    if (p.mode == BSA_MODE_TOPK) {
      m = min(min(p.topk, p.cap), p.nb);
    } else {
      m = mass_count(pr, p.nb, p.mass_tau, min(p.cap, p.nb), myhist, mybuf);
    }
    const unsigned long long kth = kth_key(pr, p.nb, m, myhist);
    const long long r = (long long)bh * p.nb + i;
    uint32_t* dst = p.bitmaps + r * p.nbw;
    int cnt = 0;
    for (int wd = 0; wd < p.nbw; ++wd) {
      const int j = wd * 32 + lane;
      bool keep = false;
      if (j < p.nb) {
        keep = order_key(pr[j], j) <= kth;
        if (p.keep_diag && j == i) keep = true;
        if (j < p.n_sink) keep = true;
      }
      const unsigned word = __ballot_sync(0xffffffffu, keep);
      if (lane == 0) dst[wd] = word;
      cnt += __popc(word);
    }
    if (lane == 0) s_cnt[rr] = cnt;
    __syncwarp();
  }
  csr_write_rows(p, lin, bh, i0, nrow, s_cnt, &s_base);
}

// ------------------------------------------------------------------ select, registers
// Order key of the register path: u = ~bits(p).  p >= 0, so ascending u is
// descending p, and equal u means equal p; ties go to the lower block index.
// Block j of a row sits in register r = j / 32 of lane j % 32; lanes past nb
// hold u = ~0u, which decodes to p = +0 and is never kept.

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Number of blocks of the row with key <= t (row padding counts only at t = ~0u).
template <int NPL>
__device__ __forceinline__ int count_le(const unsigned (&u)[NPL], unsigned t) {
  int c = 0;
#pragma unroll
  for (int r = 0; r < NPL; ++r) c += u[r] <= t ? 1 : 0;
  return __reduce_add_sync(0xffffffffu, c);
}

// Probability mass of the blocks with key <= t (fixed summation order for a given t).
template <int NPL>
__device__ __forceinline__ float mass_le(const unsigned (&u)[NPL], unsigned t) {
  float s = 0.f;
#pragma unroll
  for (int r = 0; r < NPL; ++r) s += u[r] <= t ? __uint_as_float(~u[r]) : 0.f;
  return warp_sum_f(s);
}

// The first m blocks in key order (1 <= m <= nb), as (T, need): every key < T
// and the `need` lowest-index blocks with key == T.  Bisection over the bits
// below the common prefix of lo and hi (the row's smallest and largest key)
// for the smallest t with count_le(t) >= m; it stops early at a t with exactly
// m keys <= t, which then are the answer (T = t + 1, need = 0).
template <int NPL>
__device__ __forceinline__ unsigned cut_by_count(const unsigned (&u)[NPL], int m, unsigned lo,
                                                 unsigned hi, int& need) {
  if (lo == hi) {   // every key equal: the m lowest indices
    need = m;
    return lo;
  }
  const int hb = 31 - __clz(lo ^ hi);
  unsigned t = lo & ~((2u << hb) - 1u);
#pragma unroll 1
  for (int b = hb; b >= 0; --b) {
    const unsigned bit = 1u << b;
    const unsigned cand = t | (bit - 1u);
    const int c = count_le(u, cand);
    if (c == m && cand != 0xFFFFFFFFu) {
      need = 0;
      return cand + 1u;
    }
    if (c < m) t |= bit;
  }
  need = m - (t == 0u ? 0 : count_le(u, t - 1u));
  return t;
}

// Smallest key t in [lo, hi] with mass_le(t) >= tau, given mass_le(hi) >= tau.
template <int NPL>
__device__ __forceinline__ unsigned kth_by_mass(const unsigned (&u)[NPL], float tau, unsigned lo,
                                                unsigned hi) {
  if (lo == hi) return lo;
  const int hb = 31 - __clz(lo ^ hi);
  unsigned t = lo & ~((2u << hb) - 1u);
#pragma unroll 1
  for (int b = hb; b >= 0; --b) {
    const unsigned bit = 1u << b;
    if (mass_le(u, t | (bit - 1u)) < tau) t |= bit;
  }
  return t;
}

// Bit r set <=> this lane's block in register r is among the first blocks in
// key order: every key < T, and the `need` lowest-index blocks with key == T.
template <int NPL>
__device__ __forceinline__ unsigned keep_bits(const unsigned (&u)[NPL], int nb, unsigned T,
                                              int need) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = lanemask_lt();
  unsigned bits = 0u;
  int taken = 0;
#pragma unroll
  for (int r = 0; r < NPL; ++r) {
    const bool tie = r * 32 + lane < nb && u[r] == T;
    const unsigned bal = __ballot_sync(0xffffffffu, tie);
    const bool k = u[r] < T || (tie && taken + __popc(bal & lt) < need);
    bits |= (k ? 1u : 0u) << r;
    taken += __popc(bal);
  }
  return bits;
}

// One warp: softmax of the row's scores, the rule's cut, forced blocks, then
// the row's bitmap words and count.
template <int NPL>
__device__ __forceinline__ void select_row_regs(const float* srow, int i, long long row,
                                                const SelectParams& p, int* cnt_out) {
  const int lane = threadIdx.x & 31;
  const int nb = p.nb;
  float v[NPL];
  float mx = -INFINITY;
#pragma unroll
  for (int r = 0; r < NPL; ++r) {
    const int j = r * 32 + lane;
    v[r] = j < nb ? srow[j] : -INFINITY;
    mx = fmaxf(mx, v[r]);
  }
  mx = warp_max(mx);
  float sum = 0.f;
#pragma unroll
  for (int r = 0; r < NPL; ++r) {
    const float e = r * 32 + lane < nb ? expf(v[r] - mx) : 0.f;
    v[r] = e;
    sum += e;
  }
  sum = warp_sum_f(sum);
  const float inv = 1.0f / sum;
  unsigned u[NPL];
  unsigned lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
  for (int r = 0; r < NPL; ++r) {
    u[r] = 0xFFFFFFFFu;
    if (r * 32 + lane < nb) {
      u[r] = ~__float_as_uint(v[r] * inv);
      lo = min(lo, u[r]);
      hi = max(hi, u[r]);
    }
  }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);

  const int L = min(p.cap, nb);
  const int m0 = p.mode == BSA_MODE_TOPK ? min(p.topk, L) : L;
  int need = 0;
  unsigned T = cut_by_count(u, m0, lo, hi, need);
  if (p.mode == BSA_MODE_MASS) {
    // The top L fall short of tau: the cap binds and the cut is L.  Otherwise
    // the shortest prefix reaching tau ends inside the top L: find its last key.
    const unsigned kb = keep_bits(u, nb, T, need);
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < NPL; ++r) s += (kb >> r) & 1u ? __uint_as_float(~u[r]) : 0.f;
    s = warp_sum_f(s);
    const unsigned top = need == 0 ? T - 1u : T;   // largest key among the top L
    if (s >= p.mass_tau && mass_le(u, top) >= p.mass_tau) {
      const unsigned t = kth_by_mass(u, p.mass_tau, lo, top);
      const int c_lt = t == 0u ? 0 : count_le(u, t - 1u);
      const float f_lt = t == 0u ? 0.f : mass_le(u, t - 1u);
      const int n_tie = count_le(u, t) - c_lt;
      const float pt = __uint_as_float(~t);
      // ties at the cut are taken one at a time, each adding pt
      int n = 1;
      if (pt > 0.f) {
        const float q = (p.mass_tau - f_lt) / pt;
        n = q >= static_cast<float>(n_tie) ? n_tie : max(1, static_cast<int>(ceilf(q)));
      }
      if (c_lt + n <= L) {
        T = t;
        need = n;
      }
    }
  }
  const unsigned kb = keep_bits(u, nb, T, need);
  unsigned myword = 0u;
  int cnt = 0;
#pragma unroll
  for (int r = 0; r < NPL; ++r) {
    const int j = r * 32 + lane;
    const bool forced = j < nb && ((p.keep_diag && j == i) || j < p.n_sink);
    const unsigned w = __ballot_sync(0xffffffffu, ((kb >> r) & 1u) || forced);
    if (lane == r) myword = w;
    cnt += __popc(w);
  }
  if (lane < p.nbw) p.bitmaps[row * p.nbw + lane] = myword;
  if (lane == 0) *cnt_out = cnt;
}

// Tile shape of asa_select_kernel for nb in (128 (NCB-1), 128 NCB], NCB <= 8.
template <int D, int NCB>
struct SelTile {
  static constexpr int NPL = NCB <= 1 ? 4 : NCB <= 2 ? 8 : NCB <= 4 ? 16 : 32;  // p per lane
  static constexpr int NB_PAD = 128 * NCB;                 // score row stride
  static constexpr int R = 8 * (8 / NCB);                  // q-block rows per CTA
  // k̄ᵀ rows per cp.async stage: a power of two, DK * NB_PAD <= 8192 floats
  static constexpr int DK = (D * NB_PAD <= 8192) ? D : (D / 2 * NB_PAD <= 8192) ? D / 2
                            : (D / 4 * NB_PAD <= 8192) ? D / 4 : (D / 8 * NB_PAD <= 8192) ? D / 8
                            : D / 16;
  static constexpr int REGION_A = (2 * DK > R ? 2 * DK : R) * NB_PAD;   // floats
  static constexpr int SMEM = (D * R + REGION_A) * 4;
  static_assert(DK * NB_PAD <= 8192 && D % DK == 0, "stage size");
  static_assert((R / 8) * NCB <= 8, "warp tiles");
};

// nb <= 128 * NCB <= 1024.  R rows per CTA, with (R / 8) * NCB <= 8: warp w
// owns the 8 x 128 score tile (rows 8 * (w / NCB) .., columns 128 * (w % NCB)
// ..), a lane 8 rows x 4 columns, so one k̄ᵀ float4 and two broadcast q̄
// float4 feed 32 FMAs.  Shared memory: qs [D][R] fp32, then region A: two
// stages of DK k̄ᵀ rows (DK * NB_PAD floats each), reused for the
// [R][NB_PAD] scores.
template <int D, int NCB>
__global__ void __launch_bounds__(256, NCB > 4 ? 2 : 3) asa_select_kernel(const SelectParams p) {
  using T = SelTile<D, NCB>;
  constexpr int NPL = T::NPL, R = T::R, nb_pad = T::NB_PAD, DK = T::DK, ncb = NCB;
  extern __shared__ __align__(16) float sel_f[];
  float* qs = sel_f;
  float* ka = sel_f + D * R;
  __shared__ int s_cnt[R];
  __shared__ long long s_base;
  __shared__ int s_lin;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_lin = static_cast<int>(atomicAdd(p.scan_ticket, 1u));
  __syncthreads();
  const int lin = s_lin;
  const int bh = lin / p.groups, i0 = (lin % p.groups) * R;
  const int nrow = min(R, p.nb - i0);
  const int rt = warp / ncb, ct = warp - rt * ncb;
  const bool active = warp < (R >> 3) * ncb && rt * 8 < nrow;
  const float* kt = p.kbarT + (long long)bh * D * p.kt_ld;

  // stage c: k̄ᵀ rows [c*DK, c*DK+DK) -> buffer c&1 (row stride nb_pad; the
  // columns past kt_ld are never read back as scores of real blocks)
  auto stage = [&](int c) {
    const int ld4 = p.kt_ld >> 2;
    const float* src = kt + (long long)c * DK * p.kt_ld;
    float* dst = ka + (c & 1) * DK * nb_pad;
    for (int rr = warp; rr < DK; rr += kSelWarps)
      for (int c4 = lane; c4 < ld4; c4 += 32)
        cp_async16(dst + rr * nb_pad + 4 * c4, src + (long long)rr * p.kt_ld + 4 * c4);
    cp_async_commit();
  };
  stage(0);
  // q̄ rows -> qs[d][row] (absent rows as zeros)
  const float* qg = p.qbar + ((long long)bh * p.nb + i0) * D;
  for (int e = tid; e < R * (D / 4); e += 256) {
    const int rr = e % R, d4 = e / R;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (rr < nrow) v = __ldg(reinterpret_cast<const float4*>(qg + (long long)rr * D) + d4);
    qs[(4 * d4 + 0) * R + rr] = v.x;
    qs[(4 * d4 + 1) * R + rr] = v.y;
    qs[(4 * d4 + 2) * R + rr] = v.z;
    qs[(4 * d4 + 3) * R + rr] = v.w;
  }

  float acc[8][4];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int m = 0; m < 4; ++m) acc[a][m] = 0.f;
  const int nchunks = D / DK;
#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    if (c + 1 < nchunks) {
      stage(c + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (active) {
      const float* kb = ka + (c & 1) * DK * nb_pad + ct * 128 + 4 * lane;
      const float* qb = qs + c * DK * R + rt * 8;
#pragma unroll 4
      for (int dd = 0; dd < DK; ++dd) {
        const float4 kv = *reinterpret_cast<const float4*>(kb + dd * nb_pad);
        const float4 qa = *reinterpret_cast<const float4*>(qb + dd * R);
        const float4 qc = *reinterpret_cast<const float4*>(qb + dd * R + 4);
        const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qc.x, qc.y, qc.z, qc.w};
        const float kk[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
          for (int m = 0; m < 4; ++m) acc[a][m] = fmaf(qv[a], kk[m], acc[a][m]);
      }
    }
    __syncthreads();
  }
  // scores -> region A (every stage has been consumed)
  if (active) {
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      float4 o;
      o.x = acc[a][0] * p.scale;
      o.y = acc[a][1] * p.scale;
      o.z = acc[a][2] * p.scale;
      o.w = acc[a][3] * p.scale;
      *reinterpret_cast<float4*>(ka + (rt * 8 + a) * nb_pad + ct * 128 + 4 * lane) = o;
    }
  }
  __syncthreads();
  for (int rr = warp; rr < nrow; rr += kSelWarps)
    select_row_regs<NPL>(ka + rr * nb_pad, i0 + rr, (long long)bh * p.nb + i0 + rr, p,
                         &s_cnt[rr]);
  csr_write_rows(p, lin, bh, i0, nrow, s_cnt, &s_base);
}

}  // namespace bsa
