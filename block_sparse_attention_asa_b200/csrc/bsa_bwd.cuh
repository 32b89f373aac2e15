// bsa_bwd.cuh -- gradients of attention over the kept blocks of a CSR block mask, sm_100a.
//
// BLADE digest, "技术框架": ASA is trained together with the step distillation,
// so the attention over the kept blocks is differentiated.  The mask is a
// constant of the step and the LSE output receives no gradient.  For a given
// dO, with P_tu = exp(scale q_t.k_u - LSE_t) over the key tokens u of the
// blocks that token t's row lists:
//
//   dV_u  = sum_t P_tu dO_t            dP_tu = dO_t . v_u
//   D_t   = dO_t . O_t                 (equal to sum_u P_tu dP_tu)
//   dS_tu = P_tu (dP_tu - D_t)
//   dQ_t  = scale sum_u dS_tu k_u      dK_u  = scale sum_t dS_tu q_t
//
// Three launches:
//   bwd_delta_kernel     D_t from the forward's O and dO (HBM-bound).
//   bsa_bwd_dq_kernel    item = (b.h, 128-query tile); walks the ascending
//                        union of its q-blocks' rows, 128 keys per step as the
//                        forward does: S = Q K^T and dP = dO V^T into TMEM,
//                        dS (bf16) written over S, dQ += dS K with dS read
//                        from TMEM.  S is double-buffered (the kernel has one
//                        accumulator, so the second one's columns are free):
//                        S(s+1) runs during step s's element-wise pass.
//   bsa_bwd_dkdv_kernel  item = (b.h, 128-key tile); walks the q-blocks whose
//                        rows keep one of the tile's kv-blocks (binary search
//                        in the ascending rows), 128 queries per step:
//                        S^T = K Q^T and dP^T = V dO^T into TMEM, P^T and dS^T
//                        (bf16) written over them, dV += P^T dO and
//                        dK += dS^T Q with P^T and dS^T read from TMEM; at
//                        d = 64 in two halves of 64 queries, so that one
//                        half's element-wise pass overlaps the other half's
//                        MMAs.
// Each tiled kernel keeps its own side's pair of tiles resident in shared
// memory and streams the other side's gathered tiles through a two-deep ring.
// No atomics: each gradient row is written once by the item that owns it, so
// the result does not depend on scheduling.
//
// Warp roles (kBwdThreads threads, one item per CTA): all warps first build
// the item's block list; then warp 0 is the producer (TMA), warp 1 the MMA
// issuer and TMEM owner, warps 4.. the element-wise step and the epilogue
// (warp w owns TMEM lane quarter w % 4 and one contiguous part of the 128
// columns; one tile row per thread).
//
// TMEM columns: S [0,128), dP [128,256), first accumulator [256,256+D),
// second accumulator [384,384+D) (dK/dV kernel) or the odd steps' S (dQ
// kernel).
//
// Ordering facts relied on (as in the forward): the tcgen05.mma ops of one
// thread run in issue order, so the next step's S^T / dP^T may overwrite the
// bf16 operands that this step's accumulating MMAs read; every wait is bounded
// (BSA_ERR_TIMEOUT on expiry), and on the way out the producer waits for its
// loads and the issuer for its MMAs before TMEM is released.
#pragma once
#include "common.cuh"
#include "ptx.cuh"
#include "bsa_fwd.cuh"
#include <cuda_bf16.h>

namespace bsa {

// Element-wise warps: kBwdEltWarps / 4 per TMEM lane quarter, each taking a
// contiguous part of the 128 columns of its rows.
constexpr int kBwdEltWarps = 16;
constexpr int kBwdParts = kBwdEltWarps / 4;
constexpr int kBwdCols = 128 / kBwdParts;          // columns per element-wise warp
constexpr int kBwdThreads = (4 + kBwdEltWarps) * 32;
static_assert(kBwdCols % 32 == 0, "a warp's columns come in 32-column loads");

// TMEM column of the bf16 pair holding column c (0..127) of a 128-wide S or dP
// after the element-wise pass: each warp part packs its columns into the first
// half of its own column range, so no part writes columns another part reads.
__host__ __device__ constexpr int packed_col(int c) {
  return (c / kBwdCols) * kBwdCols + (c % kBwdCols) / 2;
}
constexpr int kBwdMaxNb = 4096;    // blocks per head (the item's list lives in shared memory)
constexpr float kLog2e = 1.4426950408889634f;

struct BwdParams {
  int B, H, N, nb, nbw, ntile;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const float* lse;               // [B*H*N], natural log (forward output)
  const float* delta;             // [B*H*N], D_t
  float scale;                    // softmax scale
  float scale_log2;               // softmax scale * log2(e)
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  unsigned long long wait_ns;     // bound on every wait
};

template <int D, int BLK>
struct BwdCfg {
  static constexpr int G = 128 / BLK;                // blocks per 128-row tile
  static constexpr int NCH = D / 64;                 // 64-column swizzle chunks
  static constexpr int TILE = 128 * D * 2;           // bytes of a 128-row tile
  static constexpr int CHUNK = 128 * 128;            // bytes of one 128x64 chunk
  static constexpr int NR = 2;                       // ring depth
  static constexpr int RES_OFF = 0;                  // two resident tiles
  static constexpr int RA_OFF = 2 * TILE;            // ring A (NR tiles)
  static constexpr int RB_OFF = RA_OFF + NR * TILE;  // ring B (NR tiles)
  static constexpr int BAR_OFF = RB_OFF + NR * TILE;
  static constexpr int BAR_BYTES = 256;
  static constexpr int NBARS = 1 + 2 * NR + 8;
  static_assert(NBARS * 8 <= BAR_BYTES, "mbarriers must fit their area");
  static constexpr int META_OFF = BAR_OFF + BAR_BYTES;     // NR step entries
  static constexpr int META_INTS = 24;                     // [0] nvalid [1..8] ids [9..16] keep
  static constexpr int MISC_OFF = META_OFF + NR * META_INTS * 4;
  static constexpr int MISC_BYTES = 128;                   // tmem base, abort, total, counts[warps]
  static constexpr int STAGE_OFF = MISC_OFF + MISC_BYTES;  // 2 x (128 LSE + 128 D) floats
  static constexpr int STAGE_BYTES = 2 * 2 * 128 * 4;
  static constexpr int BM_OFF = STAGE_OFF + STAGE_BYTES;   // q-block bitmaps (dQ kernel)
  static constexpr int BM_BYTES = 4096;
  static constexpr int LIST_OFF = BM_OFF + BM_BYTES;
  static constexpr int SMEM = LIST_OFF + kBwdMaxNb * 4 + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory over the per-CTA limit");
  static_assert(G * kBwdMaxNb / 32 * 4 <= BM_BYTES, "bitmaps must fit their area");
  static constexpr uint32_t S_COL = 0, DP_COL = 128, ACC0_COL = 256, ACC1_COL = 384;
};

// D_t = dO_t . O_t, fp32; D/8 lanes per token, 16-byte loads.  With o_res
// (the forward's rounding residual) O_t is taken as O_t + o_res_t, which
// carries the forward's fp32 result.
template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                        const __nv_bfloat16* __restrict__ o_res,
                                                        const __nv_bfloat16* __restrict__ dout,
                                                        long long tokens, float* __restrict__ delta) {
  constexpr int TPT = D / 8;
  const long long tok = ((long long)blockIdx.x * 256 + threadIdx.x) / TPT;
  const int part = threadIdx.x % TPT;
  float acc = 0.f;
  if (tok < tokens) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + tok * D) + part);
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(dout + tok * D) + part);
    const __nv_bfloat162* ha = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fa = __bfloat1622float2(ha[e]), fb = __bfloat1622float2(hb[e]);
      acc = fmaf(fa.x, fb.x, acc);
      acc = fmaf(fa.y, fb.y, acc);
    }
    if (o_res != nullptr) {
      const uint4 c = __ldg(reinterpret_cast<const uint4*>(o_res + tok * D) + part);
      const __nv_bfloat162* hc = reinterpret_cast<const __nv_bfloat162*>(&c);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fc = __bfloat1622float2(hc[e]), fb = __bfloat1622float2(hb[e]);
        acc = fmaf(fc.x, fb.x, acc);
        acc = fmaf(fc.y, fb.y, acc);
      }
    }
  }
#pragma unroll
  for (int off = TPT / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (tok < tokens && part == 0) delta[tok] = acc;
}

// Bits (over kv-blocks j0 .. j0+ng-1) that CSR row r keeps; the row is ascending.
__device__ __forceinline__ uint32_t row_keep_bits(const int32_t* __restrict__ row_ptr,
                                                  const int32_t* __restrict__ col_idx, long long r,
                                                  int j0, int ng) {
  int lo = row_ptr[r];
  const int e1 = row_ptr[r + 1];
  int hi = e1;
  while (lo < hi) {   // first entry >= j0
    const int mid = lo + ((hi - lo) >> 1);
    if (col_idx[mid] < j0)
      lo = mid + 1;
    else
      hi = mid;
  }
  uint32_t keep = 0;
  for (int e = lo; e < e1; ++e) {
    const int c = col_idx[e];
    if (c >= j0 + ng) break;
    if (c >= j0) keep |= 1u << (c - j0);
  }
  return keep;
}

// Zero the gradient rows [t0, t0 + 128) ∩ [0, N) of one head: a tile no row reaches.
template <int D>
__device__ __forceinline__ void zero_rows(__nv_bfloat16* g, long long bh, int t0, int N) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < 128; r += kBwdThreads / 32) {
    const int token = t0 + r;
    if (token >= N) break;
    uint4* dst = reinterpret_cast<uint4*>(g + (bh * N + token) * D);
    for (int c = lane; c < D / 8; c += 32) dst[c] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Store NC columns of one accumulator row (this thread's TMEM lane) as bf16,
// times `mul`.
template <int NC>
__device__ __forceinline__ void store_acc_row(uint32_t taddr, float mul, __nv_bfloat16* dst,
                                              bool store) {
  static_assert(NC % 16 == 0, "16-column loads");
  constexpr int EC = NC % 32 == 0 ? 32 : 16;   // columns per TMEM load
#pragma unroll 1
  for (int c = 0; c < NC / EC; ++c) {
    uint32_t r[32];
    if constexpr (EC == 32) {
      tmem_ld32(taddr + c * EC, r);
    } else {
      uint32_t r16[16];
      tmem_ld16(taddr + c * EC, r16);
#pragma unroll
      for (int e = 0; e < 16; ++e) r[e] = r16[e];
    }
    tmem_wait_ld();
    uint32_t packed[16];
#pragma unroll
    for (int e = 0; e < EC / 2; ++e) {
      __nv_bfloat162 hb = __floats2bfloat162_rn(__uint_as_float(r[2 * e]) * mul,
                                                __uint_as_float(r[2 * e + 1]) * mul);
      packed[e] = *reinterpret_cast<uint32_t*>(&hb);
    }
    if (store) {
      uint4* d4 = reinterpret_cast<uint4*>(dst + c * EC);
#pragma unroll
      for (int e = 0; e < EC / 8; ++e)
        d4[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
    }
  }
}

// ============================================================================ dK, dV
template <int D, int BLK>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bsa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_k,    // box 128 rows
                        const __grid_constant__ CUtensorMap tm_v,    // box 128 rows
                        const __grid_constant__ CUtensorMap tm_q,    // box BLK rows
                        const __grid_constant__ CUtensorMap tm_do,   // box BLK rows
                        const BwdParams p) {
  using C = BwdCfg<D, BLK>;
  // d = 64: each step's 128 queries are two halves of 64 (X = 0, 1): S^T_X and
  // dP^T_X (N = 64 MMAs) into columns [64X, 64X + 64) of S^T and of dP^T,
  // then dV += P^T_X dO_X and dK += dS^T_X Q_X (K = 64).  The element-wise
  // warps of half X (the parts 2X and 2X + 1 of each lane quarter) depend only
  // on half X's MMAs, so one half's element-wise pass runs while the tensor
  // pipe works on the other half (measured on B200: CogVideoX backward 10.74
  // -> 10.16 ms).  d = 128 keeps whole steps: there the half-rate N = 64 MMAs
  // cost more than the overlap gains (Wan 3.62 -> 3.72 ms).
  constexpr int NHALF = D == 64 ? 2 : 1;
  constexpr int QH = 128 / NHALF;                // queries per half
  constexpr int HW = kBwdEltWarps / NHALF;       // element-wise warps per half
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* res_full = bars;                     // resident K, V
  uint64_t* ring_full = res_full + 1;            // [NR] Q, dO of a step
  uint64_t* ring_free = ring_full + C::NR;       // [NR]
  uint64_t* s_full = ring_free + C::NR;          // [2 halves] S^T_X, dP^T_X in TMEM
  uint64_t* p_full = s_full + 2;                 // [2 halves] P^T_X, dS^T_X in TMEM
  uint64_t* acc_done = p_full + 2;               // dV, dK complete
  uint64_t* stage_bar = acc_done + 1;            // [2 halves] LSE/D of the half staged
  uint64_t* drain = stage_bar + 2;
  int* meta = reinterpret_cast<int*>(smem + C::META_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  int* abort_flag = reinterpret_cast<int*>(smem + C::MISC_OFF + 4);
  int* wcount = reinterpret_cast<int*>(smem + C::MISC_OFF + 16);    // [warps]
  float* stage = reinterpret_cast<float*>(smem + C::STAGE_OFF);     // [2][LSE 128 | D 128]
  uint32_t* list = reinterpret_cast<uint32_t*>(smem + C::LIST_OFF);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x / p.ntile, kt = blockIdx.x % p.ntile;
  const int j0 = kt * C::G;
  const int ng = min(C::G, p.nb - j0);

  // ---- q-blocks whose rows keep one of kv-blocks [j0, j0 + ng), ascending,
  // each with its keep bits over those kv-blocks
  int total = 0;
  for (int base = 0; base < p.nb; base += kBwdThreads) {
    const int i = base + tid;
    uint32_t keep = 0;
    if (i < p.nb) keep = row_keep_bits(p.row_ptr, p.col_idx, (long long)bh * p.nb + i, j0, ng);
    const unsigned m = __ballot_sync(0xffffffffu, keep != 0u);
    if (lane == 0) wcount[warp] = __popc(m);
    __syncthreads();
    int before = 0, round = 0;
#pragma unroll
    for (int w = 0; w < kBwdThreads / 32; ++w) {
      const int c = wcount[w];
      round += c;
      before += w < warp ? c : 0;
    }
    if (keep) list[total + before + __popc(m & ((1u << lane) - 1u))] = static_cast<uint32_t>(i) | (keep << 16);
    total += round;
    __syncthreads();
  }
  if (total == 0) {
    zero_rows<D>(p.dk, bh, kt * 128, p.N);
    zero_rows<D>(p.dv, bh, kt * 128, p.N);
    return;
  }
  const int nsteps = (total + C::G - 1) / C::G;

  if (tid == 0) {
    mbar_init(res_full, 1);
    for (int s = 0; s < C::NR; ++s) {
      mbar_init(&ring_full[s], 1);
      mbar_init(&ring_free[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], HW);                 // the half's warps
      mbar_init(&stage_bar[x], HW);
    }
    mbar_init(acc_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(res_full, 2 * C::TILE);
#pragma unroll
      for (int c = 0; c < C::NCH; ++c) {
        tma_load_3d(smem + C::RES_OFF + c * C::CHUNK, &tm_k, res_full, c * 64, kt * 128, bh);
        tma_load_3d(smem + C::RES_OFF + C::TILE + c * C::CHUNK, &tm_v, res_full, c * 64, kt * 128, bh);
      }
      int s = 0;
      for (; s < nsteps; ++s) {
        const int slot = s % C::NR;
        if (s >= C::NR && !mbar_wait(&ring_free[slot], ((s / C::NR) - 1) & 1, p.wait_ns)) {
          ok = false;
          break;
        }
        int* me = meta + slot * C::META_INTS;
        const int pos = s * C::G, nvalid = min(C::G, total - pos);
        const uint32_t e0 = list[pos];
        me[0] = nvalid;
#pragma unroll
        for (int sl = 0; sl < C::G; ++sl) {
          const uint32_t e = sl < nvalid ? list[pos + sl] : e0;   // unused: reload a listed block
          me[1 + sl] = static_cast<int>(e & 0xFFFFu);
          me[9 + sl] = sl < nvalid ? static_cast<int>(e >> 16) : 0;
        }
        mbar_arrive_expect_tx(&ring_full[slot], 2 * C::TILE);
#pragma unroll
        for (int sl = 0; sl < C::G; ++sl)
#pragma unroll
          for (int c = 0; c < C::NCH; ++c) {
            const int row = me[1 + sl] * BLK;
            tma_load_3d(smem + C::RA_OFF + slot * C::TILE + c * C::CHUNK + sl * BLK * 128, &tm_q,
                        &ring_full[slot], c * 64, row, bh);
            tma_load_3d(smem + C::RB_OFF + slot * C::TILE + c * C::CHUNK + sl * BLK * 128, &tm_do,
                        &ring_full[slot], c * 64, row, bh);
          }
      }
      if (!ok) {
        record_error(BSA_ERR_TIMEOUT);
        *(volatile int*)abort_flag = 1;
      }
      // every load issued lands before the CTA exits
      mbar_wait(res_full, 0, p.wait_ns);
      for (int t = s > C::NR ? s - C::NR : 0; t < s; ++t)
        mbar_wait(&ring_full[t % C::NR], (t / C::NR) & 1, p.wait_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, 0, 1);
      const uint64_t d_k = smem_desc(smem_u32(smem + C::RES_OFF), 16, 1024);
      const uint64_t d_v = smem_desc(smem_u32(smem + C::RES_OFF + C::TILE), 16, 1024);
      const uint64_t d_q = smem_desc(smem_u32(smem + C::RA_OFF), 16, 1024);          // K-major
      const uint64_t d_do = smem_desc(smem_u32(smem + C::RB_OFF), 16, 1024);         // K-major
      const uint64_t d_q_mn = smem_desc(smem_u32(smem + C::RA_OFF), C::CHUNK, 1024); // MN-major
      const uint64_t d_do_mn = smem_desc(smem_u32(smem + C::RB_OFF), C::CHUNK, 1024);
      constexpr uint32_t idesc_h = idesc_bf16_f32(128, QH, 0, 0);   // N = the half's queries
      const uint32_t t_s = tmem + C::S_COL, t_dp = tmem + C::DP_COL;
      const uint32_t t_dv = tmem + C::ACC0_COL, t_dk = tmem + C::ACC1_COL;
      // S^T_X = K Q_X^T and dP^T_X = V dO_X^T (M = 128 keys, N = 64 queries,
      // K = D): Q_X, dO_X are rows 64X .. 64X+63 of the step's tiles
      auto issue_sdp = [&](int s, int x) {
        const uint64_t ro = static_cast<uint64_t>(((s % C::NR) * C::TILE + x * QH * 128) >> 4);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::CHUNK + (kk & 3) * 32) >> 4);
          mma_ss(t_s + QH * x, d_k + off, d_q + ro + off, idesc_h, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::CHUNK + (kk & 3) * 32) >> 4);
          mma_ss(t_dp + QH * x, d_v + off, d_do + ro + off, idesc_h, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[x]);
      };
      // dV += P^T_X dO_X, dK += dS^T_X Q_X (M = 128 keys, N = D, K = 64 queries)
      auto issue_acc = [&](int s, int x) {
        const uint64_t ro = static_cast<uint64_t>(((s % C::NR) * C::TILE) >> 4);
        tc_fence_after();
#pragma unroll
        for (int k4 = 0; k4 < QH / 16; ++k4) {
          const int kk = (QH / 16) * x + k4;          // 16-query group of the step
          mma_ts(t_dv, t_s + packed_col(kk * 16), d_do_mn + ro + static_cast<uint64_t>((kk * 2048) >> 4),
                 idesc_acc, (s > 0 || kk > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int k4 = 0; k4 < QH / 16; ++k4) {
          const int kk = (QH / 16) * x + k4;
          mma_ts(t_dk, t_dp + packed_col(kk * 16), d_q_mn + ro + static_cast<uint64_t>((kk * 2048) >> 4),
                 idesc_acc, (s > 0 || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(res_full, 0, p.wait_ns) && mbar_wait(&ring_full[0], 0, p.wait_ns);
      bool issued = false;
      if (ok) {
        for (int x = 0; x < NHALF; ++x) issue_sdp(0, x);
        issued = true;
      }
      // order: ... acc_0(s), sdp_0(s+1), acc_1(s), sdp_1(s+1), ...  Each half's
      // S^T/dP^T columns are rewritten only after that half's accumulating
      // MMAs have been issued (same thread: they run in order).
      for (int s = 0; ok && s < nsteps; ++s) {
        const int slot = s % C::NR;
        const int s1 = s + 1;
        for (int x = 0; x < NHALF; ++x) {
          if (!mbar_wait(&p_full[x], s & 1, p.wait_ns)) {
            ok = false;
            break;
          }
          issue_acc(s, x);
          if (x == NHALF - 1) mma_commit(&ring_free[slot]);   // the step's last reads of Q and dO
          if (s1 < nsteps) {
            if (x == 0 && !mbar_wait(&ring_full[s1 % C::NR], (s1 / C::NR) & 1, p.wait_ns)) {
              ok = false;
              break;
            }
            issue_sdp(s1, x);
          }
        }
      }
      if (ok) {
        mma_commit(acc_done);
      } else {
        record_error(BSA_ERR_TIMEOUT);
        *(volatile int*)abort_flag = 1;
      }
      if (issued) {
        mma_commit(drain);
        mbar_wait(drain, 0, p.wait_ns);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ================================================================ P^T, dS^T, epilogue
    // warp (q, part): TMEM lane quarter q = warp % 4, query columns
    // [part * kBwdCols, part * kBwdCols + kBwdCols) of each step
    const int wq = warp & 3;
    const int part = (warp - 4) >> 2;
    const int half = part / (4 / NHALF);         // query half of the step (d = 64: parts 2X, 2X+1)
    const int cbase = part * kBwdCols;
    const int sbase = cbase / BLK;                // first q slot of this part
    const int u = wq * 32 + lane;                 // key row of the tile
    const int key = kt * 128 + u;
    const bool key_ok = key < p.N;
    const int kvb = u / BLK;                      // its kv-block in the tile
    const int gt = tid - 128;                     // 0 .. kBwdEltWarps*32 - 1
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float c2 = p.scale_log2;
    auto warp_arrive = [&](uint64_t* bar) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    bool ok = true;
    for (int s = 0; s < nsteps; ++s) {
      const int slot = s % C::NR;
      bool w_ok = mbar_wait(&ring_full[slot], (s / C::NR) & 1, p.wait_ns) && !*(volatile int*)abort_flag;
      if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
      const int* me = meta + slot * C::META_INTS;
      const int nvalid = me[0];
      // stage LSE (log2 units) and D of the step's 128 queries; a query past N
      // or in an unused slot gets LSE = +inf (P = 0)
      float* st = stage + (s & 1) * 256;
      {
        // the half's queries, staged by the half's first QH threads
        const int ht = gt - half * HW * 32;
        if (ht < QH) {
          const int qi = half * QH + ht;          // query of the step
          const int sl = qi / BLK;
          const int tok = me[1 + sl] * BLK + qi % BLK;
          const bool valid = sl < nvalid && tok < p.N;
          st[qi] = valid ? p.lse[(long long)bh * p.N + tok] * kLog2e : INFINITY;
          st[128 + qi] = valid ? p.delta[(long long)bh * p.N + tok] : 0.f;
        }
      }
      uint32_t live = 0;   // q slots of the step whose q-block keeps this row's kv-block
#pragma unroll
      for (int sl = 0; sl < C::G; ++sl)
        if (sl < nvalid && ((me[9 + sl] >> kvb) & 1)) live |= 1u << sl;
      if (!key_ok) live = 0;
      const uint32_t live_p = live >> sbase;      // bit j: slot sbase + j
      warp_arrive(&stage_bar[half]);
      w_ok = mbar_wait(&stage_bar[half], s & 1, p.wait_ns);
      if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
      w_ok = mbar_wait(&s_full[half], s & 1, p.wait_ns);
      if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
      tc_fence_after();
      const float* stl = st + cbase;
      const uint32_t s_col = C::S_COL;
#pragma unroll
      for (int cc = 0; cc < kBwdCols / 32; ++cc) {
        uint32_t rs[32], rd[32];
        tmem_ld32(t_lane + s_col + cbase + cc * 32, rs);
        tmem_ld32(t_lane + C::DP_COL + cbase + cc * 32, rd);
        tmem_wait_ld();
        uint32_t pp[16], pd[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c0 = cc * 32 + 2 * e, c1 = c0 + 1;     // columns within the part
          const bool l0 = (live_p >> (c0 / BLK)) & 1u, l1 = (live_p >> (c1 / BLK)) & 1u;
          const float p0 = l0 ? fast_ex2(__uint_as_float(rs[2 * e]) * c2 - stl[c0]) : 0.f;
          const float p1 = l1 ? fast_ex2(__uint_as_float(rs[2 * e + 1]) * c2 - stl[c1]) : 0.f;
          const float d0 = p0 * (__uint_as_float(rd[2 * e]) - stl[128 + c0]);
          const float d1 = p1 * (__uint_as_float(rd[2 * e + 1]) - stl[128 + c1]);
          __nv_bfloat162 hp = __floats2bfloat162_rn(p0, p1);
          __nv_bfloat162 hd = __floats2bfloat162_rn(d0, d1);
          pp[e] = *reinterpret_cast<uint32_t*>(&hp);
          pd[e] = *reinterpret_cast<uint32_t*>(&hd);
        }
        // bf16 pairs into the first half of this part's columns, over fp32
        // columns this warp has already read
        tmem_st16(t_lane + s_col + packed_col(cbase + cc * 32), pp);
        tmem_st16(t_lane + C::DP_COL + packed_col(cbase + cc * 32), pd);
      }
      tmem_wait_st();
      warp_arrive(&p_full[half]);
    }
    if (ok) {
      const bool w_ok = mbar_wait(acc_done, 0, p.wait_ns);
      ok = __all_sync(0xffffffffu, w_ok);
    }
    if (ok) {
      tc_fence_after();
      constexpr int NC = D / kBwdParts;           // accumulator columns per part
      const long long row = ((long long)bh * p.N + key) * D + part * NC;
      store_acc_row<NC>(t_lane + C::ACC0_COL + part * NC, 1.0f, p.dv + row, key_ok);
      store_acc_row<NC>(t_lane + C::ACC1_COL + part * NC, p.scale, p.dk + row, key_ok);
    } else {
      record_error(BSA_ERR_TIMEOUT);
      *(volatile int*)abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ============================================================================ dQ
template <int D, int BLK>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bsa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,     // box 128 rows
                      const __grid_constant__ CUtensorMap tm_do,    // box 128 rows
                      const __grid_constant__ CUtensorMap tm_k,     // box BLK rows
                      const __grid_constant__ CUtensorMap tm_v,     // box BLK rows
                      const BwdParams p) {
  using C = BwdCfg<D, BLK>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* res_full = bars;                     // resident Q, dO
  uint64_t* ring_full = res_full + 1;            // [NR] K, V of a step
  uint64_t* ring_free = ring_full + C::NR;       // [NR]
  uint64_t* s_full = ring_free + C::NR;          // [2] S (by step parity) and dP in TMEM
  uint64_t* p_full = s_full + 2;                 // dS in TMEM (element-wise warps)
  uint64_t* acc_done = p_full + 1;               // dQ complete
  uint64_t* drain = acc_done + 1;
  int* meta = reinterpret_cast<int*>(smem + C::META_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  int* abort_flag = reinterpret_cast<int*>(smem + C::MISC_OFF + 4);
  int* total_s = reinterpret_cast<int*>(smem + C::MISC_OFF + 8);
  uint32_t* bm = reinterpret_cast<uint32_t*>(smem + C::BM_OFF);      // [G][nbw]
  uint32_t* list = reinterpret_cast<uint32_t*>(smem + C::LIST_OFF);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x / p.ntile, qt = blockIdx.x % p.ntile;
  const int qb0 = qt * C::G;
  const int nq = min(C::G, p.nb - qb0);
  const int nbw = p.nbw;

  // ---- the tile's rows as bitmaps, then their ascending union with keep bits
  // over the tile's q-blocks
  for (int e = tid; e < C::G * nbw; e += kBwdThreads) bm[e] = 0u;
  __syncthreads();
  for (int qq = 0; qq < nq; ++qq) {
    const long long r = (long long)bh * p.nb + qb0 + qq;
    const int e0 = p.row_ptr[r], e1 = p.row_ptr[r + 1];
    for (int e = e0 + tid; e < e1; e += kBwdThreads) {
      const int c = p.col_idx[e];
      if (c >= 0 && c < p.nb)
        atomicOr(&bm[qq * nbw + (c >> 5)], 1u << (c & 31));
      else
        record_error(BSA_ERR_CSR);
    }
  }
  __syncthreads();
  if (warp == 0) {
    int n = 0;
    for (int wb = 0; wb < nbw; wb += 32) {
      const int wd = wb + lane;
      uint32_t u = 0;
      if (wd < nbw)
        for (int qq = 0; qq < nq; ++qq) u |= bm[qq * nbw + wd];
      const int c = __popc(u);
      const int incl = warp_incl_scan(c);
      const int tot = __shfl_sync(0xffffffffu, incl, 31);
      int at = n + incl - c;
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1;
        uint32_t keep = 0;
        for (int qq = 0; qq < nq; ++qq) keep |= ((bm[qq * nbw + wd] >> bit) & 1u) << qq;
        list[at++] = static_cast<uint32_t>(wd * 32 + bit) | (keep << 16);
      }
      n += tot;
    }
    if (lane == 0) *total_s = n;
  }
  __syncthreads();
  const int total = *total_s;
  if (total == 0) {
    zero_rows<D>(p.dq, bh, qt * 128, p.N);
    return;
  }
  const int nsteps = (total + C::G - 1) / C::G;

  if (tid == 0) {
    mbar_init(res_full, 1);
    for (int s = 0; s < C::NR; ++s) {
      mbar_init(&ring_full[s], 1);
      mbar_init(&ring_free[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_full, kBwdEltWarps);
    mbar_init(acc_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(res_full, 2 * C::TILE);
#pragma unroll
      for (int c = 0; c < C::NCH; ++c) {
        tma_load_3d(smem + C::RES_OFF + c * C::CHUNK, &tm_q, res_full, c * 64, qt * 128, bh);
        tma_load_3d(smem + C::RES_OFF + C::TILE + c * C::CHUNK, &tm_do, res_full, c * 64, qt * 128, bh);
      }
      int s = 0;
      for (; s < nsteps; ++s) {
        const int slot = s % C::NR;
        if (s >= C::NR && !mbar_wait(&ring_free[slot], ((s / C::NR) - 1) & 1, p.wait_ns)) {
          ok = false;
          break;
        }
        int* me = meta + slot * C::META_INTS;
        const int pos = s * C::G, nvalid = min(C::G, total - pos);
        const uint32_t e0 = list[pos];
        me[0] = nvalid;
#pragma unroll
        for (int sl = 0; sl < C::G; ++sl) {
          const uint32_t e = sl < nvalid ? list[pos + sl] : e0;
          me[1 + sl] = static_cast<int>(e & 0xFFFFu);
          me[9 + sl] = sl < nvalid ? static_cast<int>(e >> 16) : 0;
        }
        mbar_arrive_expect_tx(&ring_full[slot], 2 * C::TILE);
#pragma unroll
        for (int sl = 0; sl < C::G; ++sl)
#pragma unroll
          for (int c = 0; c < C::NCH; ++c) {
            const int row = me[1 + sl] * BLK;
            tma_load_3d(smem + C::RA_OFF + slot * C::TILE + c * C::CHUNK + sl * BLK * 128, &tm_k,
                        &ring_full[slot], c * 64, row, bh);
            tma_load_3d(smem + C::RB_OFF + slot * C::TILE + c * C::CHUNK + sl * BLK * 128, &tm_v,
                        &ring_full[slot], c * 64, row, bh);
          }
      }
      if (!ok) {
        record_error(BSA_ERR_TIMEOUT);
        *(volatile int*)abort_flag = 1;
      }
      mbar_wait(res_full, 0, p.wait_ns);
      for (int t = s > C::NR ? s - C::NR : 0; t < s; ++t)
        mbar_wait(&ring_full[t % C::NR], (t / C::NR) & 1, p.wait_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, 0, 1);
      const uint64_t d_q = smem_desc(smem_u32(smem + C::RES_OFF), 16, 1024);
      const uint64_t d_do = smem_desc(smem_u32(smem + C::RES_OFF + C::TILE), 16, 1024);
      const uint64_t d_k = smem_desc(smem_u32(smem + C::RA_OFF), 16, 1024);           // K-major
      const uint64_t d_v = smem_desc(smem_u32(smem + C::RB_OFF), 16, 1024);           // K-major
      const uint64_t d_k_mn = smem_desc(smem_u32(smem + C::RA_OFF), C::CHUNK, 1024);  // MN-major
      // S is double-buffered (S of step s in the columns of parity s; the
      // dQ kernel leaves the second accumulator's columns free), so S(s+1) =
      // Q K(s+1)^T runs while the element-wise warps work on step s; dP has
      // one buffer, so dP(s+1) follows the element-wise pass of step s.
      const uint32_t t_dp = tmem + C::DP_COL, t_dq = tmem + C::ACC0_COL;
      auto t_s = [&](int s) -> uint32_t { return tmem + ((s & 1) ? C::ACC1_COL : C::S_COL); };
      auto issue_s = [&](int s) {
        const uint64_t ro = static_cast<uint64_t>(((s % C::NR) * C::TILE) >> 4);
        tc_fence_after();
        // S = Q K^T (M = 128 queries, N = 128 keys, K = D)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::CHUNK + (kk & 3) * 32) >> 4);
          mma_ss(t_s(s), d_q + off, d_k + ro + off, idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_dp = [&](int s) {
        const uint64_t ro = static_cast<uint64_t>(((s % C::NR) * C::TILE) >> 4);
        // dP = dO V^T
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::CHUNK + (kk & 3) * 32) >> 4);
          mma_ss(t_dp, d_do + off, d_v + ro + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[s & 1]);   // S(s) and dP(s)
      };
      bool ok = mbar_wait(res_full, 0, p.wait_ns) && mbar_wait(&ring_full[0], 0, p.wait_ns);
      bool issued = false;
      if (ok) {
        issue_s(0);
        issue_dp(0);
        issued = true;
      }
      for (int s = 0; ok && s < nsteps; ++s) {
        const int slot = s % C::NR;
        const int s1 = s + 1, slot1 = s1 % C::NR;
        // S(s+1) now if its K is already here (its buffer last held dS(s-1),
        // read by dQ(s-1), issued before)
        bool s1_done = false;
        if (s1 < nsteps && mbar_test_wait(&ring_full[slot1], (s1 / C::NR) & 1)) {
          issue_s(s1);
          s1_done = true;
        }
        if (!mbar_wait(p_full, s & 1, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // dQ += dS K (M = 128 queries, N = D, K = 128 keys)
        {
          const uint64_t ro = static_cast<uint64_t>((slot * C::TILE) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(t_dq, t_s(s) + packed_col(kk * 16),
                   d_k_mn + ro + static_cast<uint64_t>((kk * 2048) >> 4), idesc_acc,
                   (s > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&ring_free[slot]);
        if (s1 < nsteps) {
          if (!s1_done) {
            if (!mbar_wait(&ring_full[slot1], (s1 / C::NR) & 1, p.wait_ns)) {
              ok = false;
              break;
            }
            issue_s(s1);
          }
          issue_dp(s1);   // dP's buffer: the element-wise pass of step s has read dP(s)
        }
      }
      if (ok) {
        mma_commit(acc_done);
      } else {
        record_error(BSA_ERR_TIMEOUT);
        *(volatile int*)abort_flag = 1;
      }
      if (issued) {
        mma_commit(drain);
        mbar_wait(drain, 0, p.wait_ns);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ================================================================ dS, epilogue
    // warp (q, part): TMEM lane quarter q = warp % 4, key columns
    // [part * kBwdCols, part * kBwdCols + kBwdCols) of each step
    constexpr int SPP = kBwdCols >= BLK ? kBwdCols / BLK : 1;   // kv slots per part
    const int wq = warp & 3;
    const int part = (warp - 4) >> 2;
    const int cbase = part * kBwdCols;
    const int sbase = cbase / BLK;                // first kv slot of this part
    const int koff = cbase % BLK;                 // key offset inside that slot's block
    const int r = wq * 32 + lane;                 // query row of the tile
    const int token = qt * 128 + r;
    const bool row_ok = token < p.N;
    const int qq = r / BLK;                       // its q-block in the tile
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float c2 = p.scale_log2;
    const float lse2 = row_ok ? p.lse[(long long)bh * p.N + token] * kLog2e : INFINITY;
    const float dlt = row_ok ? p.delta[(long long)bh * p.N + token] : 0.f;
    auto warp_arrive = [&](uint64_t* bar) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    bool ok = true;
    for (int s = 0; s < nsteps; ++s) {
      const int slot = s % C::NR;
      bool w_ok = mbar_wait(&ring_full[slot], (s / C::NR) & 1, p.wait_ns) && !*(volatile int*)abort_flag;
      if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
      const int* me = meta + slot * C::META_INTS;
      const int nvalid = me[0];
      // this part's kv slots: kept by this row, and their valid keys (the
      // last block may be partial)
      uint32_t live = 0;
      int nk[SPP];
#pragma unroll
      for (int j = 0; j < SPP; ++j) {
        const int sl = sbase + j;
        if (row_ok && sl < nvalid && ((me[9 + sl] >> qq) & 1)) live |= 1u << j;
        nk[j] = min(BLK, p.N - me[1 + sl] * BLK);
      }
      w_ok = mbar_wait(&s_full[s & 1], (s >> 1) & 1, p.wait_ns);
      if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
      tc_fence_after();
      const uint32_t s_col = (s & 1) ? C::ACC1_COL : C::S_COL;   // S of this step
#pragma unroll
      for (int cc = 0; cc < kBwdCols / 32; ++cc) {
        uint32_t rs[32], rd[32];
        tmem_ld32(t_lane + s_col + cbase + cc * 32, rs);
        tmem_ld32(t_lane + C::DP_COL + cbase + cc * 32, rd);
        tmem_wait_ld();
        uint32_t pd[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c0 = cc * 32 + 2 * e, c1 = c0 + 1;     // columns within the part
          const bool l0 = ((live >> (c0 / BLK)) & 1u) && koff + (c0 % BLK) < nk[c0 / BLK];
          const bool l1 = ((live >> (c1 / BLK)) & 1u) && koff + (c1 % BLK) < nk[c1 / BLK];
          const float p0 = l0 ? fast_ex2(__uint_as_float(rs[2 * e]) * c2 - lse2) : 0.f;
          const float p1 = l1 ? fast_ex2(__uint_as_float(rs[2 * e + 1]) * c2 - lse2) : 0.f;
          const float d0 = p0 * (__uint_as_float(rd[2 * e]) - dlt);
          const float d1 = p1 * (__uint_as_float(rd[2 * e + 1]) - dlt);
          __nv_bfloat162 hd = __floats2bfloat162_rn(d0, d1);
          pd[e] = *reinterpret_cast<uint32_t*>(&hd);
        }
        // dS (bf16 pairs) into the first half of this part's columns
        tmem_st16(t_lane + s_col + packed_col(cbase + cc * 32), pd);
      }
      tmem_wait_st();
      warp_arrive(p_full);
    }
    if (ok) {
      const bool w_ok = mbar_wait(acc_done, 0, p.wait_ns);
      ok = __all_sync(0xffffffffu, w_ok);
    }
    if (ok) {
      tc_fence_after();
      constexpr int NC = D / kBwdParts;
      store_acc_row<NC>(t_lane + C::ACC0_COL + part * NC, p.scale,
                        p.dq + ((long long)bh * p.N + token) * D + part * NC, row_ok);
    } else {
      record_error(BSA_ERR_TIMEOUT);
      *(volatile int*)abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace bsa
