// bsa_fwd.cuh -- attention over the kept blocks of a CSR block mask, sm_100a.
//
// Sparse-vDiT blog, "核心公式": O = softmax(Q Kᵀ/√d) V per head; BLADE digest,
// abstract: the computation is restricted to the blocks the mask keeps.  The
// online (running max / running sum) softmax is the FlashAttention scheme that
// both blogs build on.
//
// One CTA per (b·h, 128-query tile).  A 128-row tile holds S = 128/blk q-blocks;
// it walks the ascending UNION of their CSR rows, 128 keys (S kv-blocks) per
// step, and masks, per row, the kv-blocks its own q-block does not list.  On
// B200 an M=64 or N=64 tcgen05.mma runs at half the rate of M=N=128, so a
// 128x128 tile with some masked work beats exact 64-row tiles.
//
// Warp roles (256 threads):
//   warp 0      TMA producer: Q tile once, then per step S gathered K and V
//               blocks (one box per kv-block and 64-column chunk, 128B swizzle)
//               into a ring of NST stages.
//   warp 1      MMA issuer (one thread): S_j = Q K_jᵀ into TMEM (double
//               buffered), then O += P_{j-1} V_{j-1} with P read from TMEM.
//   warp 2      TMEM allocation / release.
//   warps 4-7   softmax: thread = query row = TMEM lane.  Loads S_j, masks,
//               running max (rescale of O only when the max grows by more than
//               2^8, else the stale max is kept -- exact, since the final
//               normalisation uses the same max), exponentials, P (bf16) back
//               into TMEM over S_j, epilogue O / l and LSE.
//
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D).  P_j occupies the
// first 64 columns of S_{j%2} (two bf16 per 32-bit column).
#pragma once
#include "common.cuh"
#include "ptx.cuh"
#include <cuda_bf16.h>

namespace bsa {

struct FwdParams {
  int B, H, N, nb, nbw, nqt;      // nqt: number of 128-query tiles
  const int32_t* row_ptr;
  const int32_t* col_idx;
  float scale_log2;               // softmax scale * log2(e)
  __nv_bfloat16* o;
  float* lse;
  unsigned long long wait_ns;     // bound on every wait
};

template <int D, int BLK>
struct FwdCfg {
  static constexpr int BM = 128, BN = 128;
  static constexpr int SLOTS = BN / BLK;            // kv-blocks per step
  static constexpr int QB = BM / BLK;               // q-blocks per tile
  static constexpr int NCH = D / 64;                // 64-column swizzle chunks
  static constexpr int TILE = 128 * D * 2;          // bytes of a 128-row tile
  static constexpr int CHUNK = 128 * 128;           // bytes of one 128x64 chunk
  static constexpr int NST = D == 128 ? 2 : 4;      // K/V ring depth
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = TILE;
  static constexpr int V_OFF = K_OFF + NST * TILE;
  static constexpr int AUX_OFF = V_OFF + NST * TILE;
  // aux: barriers (32 x 8 B), tmem base + flags (64 B), stage meta, bitmaps
  static constexpr int BAR_BYTES = 256;
  static constexpr int META_OFF = AUX_OFF + BAR_BYTES + 64;
  static constexpr int META_STRIDE = 16 + 8 * 8;    // nvalid + blocks[8] + keep[8]
  static constexpr int BM_OFF = META_OFF + NST * META_STRIDE * 4;
  static constexpr int kMaxBitmapBytes = 16384;
  static constexpr int SMEM = BM_OFF + kMaxBitmapBytes + 1024;  // + alignment slack
  static constexpr int O_COL = 256;
};

template <int D, int BLK>
__global__ void __launch_bounds__(256, 1)
    bsa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<D, BLK>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::AUX_OFF);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;                 // [NST]
  uint64_t* v_full = bars + 1 + C::NST;        // [NST]
  uint64_t* kv_empty = bars + 1 + 2 * C::NST;  // [NST]
  uint64_t* s_full = bars + 1 + 3 * C::NST;    // [2]
  uint64_t* p_full = s_full + 2;               // [2]
  uint64_t* o_done = p_full + 2;               // [2]
  uint64_t* mma_drain = o_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::AUX_OFF + C::BAR_BYTES);
  int* n_union = reinterpret_cast<int*>(tmem_slot + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 2);
  int* meta = reinterpret_cast<int*>(smem + C::META_OFF);
  uint32_t* bm = reinterpret_cast<uint32_t*>(smem + C::BM_OFF);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = blockIdx.x, bh = blockIdx.y;
  const int qb0 = qt * C::QB;                         // first q-block of the tile
  const int nqb = min(C::QB, p.nb - qb0);             // q-blocks present
  const int nbw = p.nbw;

  // ---- setup: barriers, TMEM, per-q-block bitmaps of the CSR rows, union size
  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128);
      mbar_init(&o_done[b], 1);
    }
    mbar_init(mma_drain, 1);
    *n_union = 0;
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  for (int e = tid; e < C::QB * nbw; e += 256) bm[e] = 0u;
  __syncthreads();
  for (int qq = warp; qq < nqb; qq += 8) {
    const long long r = (long long)bh * p.nb + qb0 + qq;
    const int e0 = p.row_ptr[r], e1 = p.row_ptr[r + 1];
    for (int e = e0 + lane; e < e1; e += 32) {
      const int c = p.col_idx[e];
      if (c >= 0 && c < p.nb)
        atomicOr(&bm[qq * nbw + (c >> 5)], 1u << (c & 31));
      else
        record_error(BSA_ERR_CSR);
    }
  }
  __syncthreads();
  {
    int cnt = 0;
    for (int w = tid; w < nbw; w += 256) {
      uint32_t u = 0;
      for (int qq = 0; qq < nqb; ++qq) u |= bm[qq * nbw + w];
      cnt += __popc(u);
    }
    cnt = warp_sum(cnt);
    if (lane == 0 && cnt) atomicAdd(n_union, cnt);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ntiles = (*n_union + C::SLOTS - 1) / C::SLOTS;

  if (warp == 0) {
    // ================================================================ producer
    if (lane == 0 && ntiles > 0) {
      const int row0 = qt * 128;
      mbar_arrive_expect_tx(q_full, C::TILE);
#pragma unroll
      for (int c = 0; c < C::NCH; ++c)
        tma_load_3d(smem + C::Q_OFF + c * C::CHUNK, &tm_q, q_full, c * 64, row0, bh);
      int w = 0, issued = 0;
      uint32_t word = 0;
      for (int qq = 0; qq < nqb; ++qq) word |= bm[qq * nbw];
      for (int j = 0; j < ntiles && !*(volatile int*)abort_flag; ++j) {
        const int st = j % C::NST;
        if (j >= C::NST && !mbar_wait(&kv_empty[st], ((j / C::NST) - 1) & 1, p.wait_ns)) {
          record_error(BSA_ERR_TIMEOUT);
          *(volatile int*)abort_flag = 1;
          break;
        }
        int* mt = meta + st * C::META_STRIDE;
        int nvalid = 0, first = 0;
#pragma unroll
        for (int s = 0; s < C::SLOTS; ++s) {
          while (word == 0 && w + 1 < nbw) {
            ++w;
            for (int qq = 0; qq < nqb; ++qq) word |= bm[qq * nbw + w];
          }
          int blkid = -1;
          if (word) {
            const int bit = __ffs(word) - 1;
            word &= word - 1;
            blkid = w * 32 + bit;
          }
          if (s == 0) first = blkid;
          int keep = 0;
          if (blkid >= 0) {
            ++nvalid;
            for (int qq = 0; qq < nqb; ++qq)
              keep |= ((bm[qq * nbw + (blkid >> 5)] >> (blkid & 31)) & 1u) << qq;
          }
          mt[1 + s] = blkid >= 0 ? blkid : first;  // unused slots reload a valid block
          mt[9 + s] = keep;
        }
        mt[0] = nvalid;
        mbar_arrive_expect_tx(&k_full[st], C::TILE);
#pragma unroll
        for (int s = 0; s < C::SLOTS; ++s)
#pragma unroll
          for (int c = 0; c < C::NCH; ++c)
            tma_load_3d(smem + C::K_OFF + st * C::TILE + c * C::CHUNK + s * BLK * 128, &tm_k,
                        &k_full[st], c * 64, mt[1 + s] * BLK, bh);
        mbar_arrive_expect_tx(&v_full[st], C::TILE);
#pragma unroll
        for (int s = 0; s < C::SLOTS; ++s)
#pragma unroll
          for (int c = 0; c < C::NCH; ++c)
            tma_load_3d(smem + C::V_OFF + st * C::TILE + c * C::CHUNK + s * BLK * 128, &tm_v,
                        &v_full[st], c * 64, mt[1 + s] * BLK, bh);
        issued = j + 1;
      }
      // drain: the loads of the last NST issued steps (and Q) must land before exit
      mbar_wait(q_full, 0, p.wait_ns);
      for (int t = issued > C::NST ? issued - C::NST : 0; t < issued; ++t) {
        const int st = t % C::NST;
        mbar_wait(&k_full[st], (t / C::NST) & 1, p.wait_ns);
        mbar_wait(&v_full[st], (t / C::NST) & 1, p.wait_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0 && ntiles > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q_base = smem_u32(smem + C::Q_OFF);
      bool ok = mbar_wait(q_full, 0, p.wait_ns);
      tc_fence_after();
      auto issue_pv = [&](int jj) -> bool {
        const int sb = jj & 1, st = jj % C::NST;
        if (!mbar_wait(&p_full[sb], (jj >> 1) & 1, p.wait_ns)) return false;
        if (!mbar_wait(&v_full[st], (jj / C::NST) & 1, p.wait_ns)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(smem + C::V_OFF + st * C::TILE);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t db = smem_desc(v_base + kk * 2048, C::CHUNK, 1024);
          mma_ts(tmem + C::O_COL, tmem + sb * 128 + kk * 8, db, idesc_pv, (jj > 0 || kk > 0));
        }
        mma_commit(&kv_empty[st]);
        mma_commit(&o_done[sb]);
        return true;
      };
      for (int j = 0; ok && j < ntiles; ++j) {
        const int st = j % C::NST, sb = j & 1;
        if (!mbar_wait(&k_full[st], (j / C::NST) & 1, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_base = smem_u32(smem + C::K_OFF + st * C::TILE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
          mma_ss(tmem + sb * 128, smem_desc(q_base + off, 16, 1024),
                 smem_desc(k_base + off, 16, 1024), idesc_qk, kk > 0);
        }
        mma_commit(&s_full[sb]);
        if (j >= 1 && !issue_pv(j - 1)) ok = false;
      }
      if (ok) ok = issue_pv(ntiles - 1);
      if (!ok) {
        record_error(BSA_ERR_TIMEOUT);
        *(volatile int*)abort_flag = 1;
      }
      // every MMA this thread issued completes before the CTA releases TMEM
      mma_commit(mma_drain);
      mbar_wait(mma_drain, 0, p.wait_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ================================================================ softmax
    const int wq = warp - 4;                 // TMEM lane quarter
    const int row = wq * 32 + lane;          // query row in the tile
    const int qq = row / BLK;                // its q-block in the tile
    const int token = qt * 128 + row;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int sb = j & 1, st = j % C::NST;
      bool w_ok = mbar_wait(&s_full[sb], (j >> 1) & 1, p.wait_ns) &&
                  mbar_wait(&k_full[st], (j / C::NST) & 1, p.wait_ns) &&
                  !*(volatile int*)abort_flag;
      if (!__all_sync(0xffffffffu, w_ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int* mt = meta + st * C::META_STRIDE;
      float x[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(t_lane + sb * 128 + c * 32, r);
#pragma unroll
        for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(r[e]);
      }
      tmem_wait_ld();
      const int nvalid = mt[0];
      float tmax = -INFINITY;
#pragma unroll
      for (int s = 0; s < C::SLOTS; ++s) {
        const bool live = s < nvalid && ((mt[9 + s] >> qq) & 1);
        const int nkeys = live ? min(BLK, p.N - mt[1 + s] * BLK) : 0;
#pragma unroll
        for (int e = 0; e < BLK; ++e) {
          const int c = s * BLK + e;
          x[c] = e < nkeys ? x[c] * p.scale_log2 : -INFINITY;
          tmax = fmaxf(tmax, x[c]);
        }
      }
      // lazy rescale, decided per warp (tcgen05.ld/st are warp-collective)
      const float m_new = fmaxf(m_run, tmax);
      const bool grow = m_new > m_run + 8.0f;
      const bool any_grow = __any_sync(0xffffffffu, grow);
      float alpha = 1.0f;
      if (grow) {
        alpha = (m_run == -INFINITY) ? 0.0f : exp2f(m_run - m_new);
        m_run = m_new;
      }
      if (any_grow && j > 0) {
        // O holds the sum of PV up to step j-1: wait for it, then scale by alpha
        w_ok = mbar_wait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, p.wait_ns);
        if (!__all_sync(0xffffffffu, w_ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(t_lane + C::O_COL + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(t_lane + C::O_COL + c * 32, r);
        }
      }
      const float m_use = m_run;
      const bool dead = m_use == -INFINITY;
      float rsum = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int col = half * 64 + 2 * c;
          const float p0 = dead ? 0.f : exp2f(x[col] - m_use);
          const float p1 = dead ? 0.f : exp2f(x[col + 1] - m_use);
          rsum += p0 + p1;
          __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
          pk[c] = *reinterpret_cast<uint32_t*>(&h);
        }
        tmem_st32(t_lane + sb * 128 + half * 32, pk);
      }
      l_run = l_run * alpha + rsum;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[sb]);
    }
    if (!ok) {
      record_error(BSA_ERR_TIMEOUT);
      *(volatile int*)abort_flag = 1;
    }
    // ---- epilogue
    bool have_o = ok && ntiles > 0;
    if (have_o) {
      const int jl = ntiles - 1;
      const bool w_ok = mbar_wait(&o_done[jl & 1], (jl >> 1) & 1, p.wait_ns);
      if (!__all_sync(0xffffffffu, w_ok)) {
        record_error(BSA_ERR_TIMEOUT);
        *(volatile int*)abort_flag = 1;
        have_o = false;
      }
      tc_fence_after();
    }
    const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
    __nv_bfloat16* orow = p.o + ((long long)bh * p.N + token) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t r[32];
      if (have_o) {
        tmem_ld32(t_lane + C::O_COL + c * 32, r);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = 0u;
      }
      uint32_t packed[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[2 * e]) * inv_l,
                                                 __uint_as_float(r[2 * e + 1]) * inv_l);
        packed[e] = *reinterpret_cast<uint32_t*>(&h);
      }
      if (token < p.N) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dst[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
      }
    }
    if (p.lse != nullptr && token < p.N)
      p.lse[(long long)bh * p.N + token] =
          l_run > 0.f ? (m_run * 0.69314718055994531f + logf(l_run)) : -INFINITY;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
}

}  // namespace bsa
