// bsa_fwd.cuh -- attention over the kept blocks of a CSR block mask, sm_100a.
//
// Sparse-vDiT blog, "核心公式": O = softmax(Q Kᵀ/√d) V per head; BLADE digest,
// abstract: the computation is restricted to the blocks the mask keeps.  The
// online (running max / running sum) softmax is the FlashAttention scheme that
// both blogs build on.
//
// Work item = (b·h, 128-query tile).  A tile holds 128/blk q-blocks and walks the
// ascending UNION of their CSR rows, 128 keys (128/blk gathered kv-blocks) per
// step, masking per row the kv-blocks its own q-block does not list.  On B200
// an M=64 or N=64 tcgen05.mma runs at half the rate of M=N=128, so a 128x128
// step with some masked work beats exact 64-row tiles.
//
// Persistent CTAs (one per SM), each running ONE stream of steps over its
// items, with the score tile S double-buffered in TMEM so that the tensor pipe
// runs the next step's QK (and the previous step's PV) while the softmax works
// on the current step, and with O and Q double-buffered per item so that the
// stream does not stop at item boundaries.  CTA c starts on item c; every later
// item comes from a grid-wide counter, so the SMs that run faster take more
// items (without a counter, items c + kG of a static deal, G = grid size).
//
// Warp roles (384 threads, 12 warps):
//   warp 3      scheduler: per item builds the q-block bitmaps of its CSR rows
//               and the ascending union list (block id + keep bits) in shared
//               memory, in segments, double-buffered, and prefetches the
//               item's Q tile into L2.
//   warp 0      producer (one lane, state in registers): per step takes up to
//               128/blk list entries, publishes a step entry (first/last, block
//               ids, keep bits) and the gathered K boxes (TMA, 128B swizzle)
//               into a K ring; the V boxes follow on a separate front, since V
//               is needed one step later than K.  Q tiles go into two buffers,
//               by item parity.
//   warp 1      MMA issuer (one thread): S(t) = Q Kᵀ into S buffer t%2 and
//               O += P(t-1) V for the previous step (P read from TMEM), in
//               whichever order their inputs arrive.  It and the producer
//               poll with non-blocking barrier tests, so waiting on one
//               barrier never delays their response to another.
//   warp 2      allocates and releases TMEM.
//   warps 4-11  softmax + epilogue.  Warp (q, h): rows 32q..32q+31 (TMEM lane
//               quarter q), keys 64h..64h+63 of each 128-key step; the two
//               halves of a row exchange their maxima through shared memory.
//               Raw-score max (3-input max), packed f32x2 scale/shift and sums,
//               one ex2 per score, lazy rescale of O (only when the max grows
//               by more than 2^kLazyRescaleLog2; exact because the final
//               normalisation uses the same stale max), P (bf16) written over
//               S in TMEM.  A half whose keys all belong to blocks its q-block
//               does not list writes P = 0 without exponentials.  An item's
//               epilogue (O / l to bf16, LSE) runs after the next item's first
//               step, by which time its last PV has long finished.
//
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [384,384+D).
//
// The single MMA thread issues step t's pair, QK(t) into S(t%2) and PV(t-1),
// in either order, and only after step t-1's pair.  Ordering facts:
//   * tcgen05.mma ops issued by one thread execute in order.  QK(t) overwrites
//     S(t%2) after PV(t-2) read P(t-2) from it (PV(t-2) was issued first, and
//     waited for the softmax to finish step t-2);
//   * when the softmax sees S(t) ready, QK(t), and so PV(t-2), have completed:
//     only PV(t-1) may still run.  A rescale of O at step t (same item) waits
//     for PV(t-1) (pv_done, one phase per PV, so the wait is unambiguous);
//   * per-buffer barriers (S ready, P stored, O done/free, Q full/free) are
//     indexed by step or item parity; each phase is waited for before the
//     buffer can be reused, so every parity wait is unambiguous;
//   * ring index s reuses K and V slots NK and NV indices later; the PV that
//     frees the V slot of a step is issued as soon as the step's P is stored,
//     and needs no K tile the producer has not loaded, so the producer never
//     waits on work that needs its own next step;
//   * the producer never stops its V front while it waits on consumer
//     progress (a free K slot is polled; the Q buffer, released by the last QK
//     of the item two before, is waited for with the V front running),
//     because that progress may itself need a V tile only this thread's V
//     front loads;
//   * every wait is bounded (BSA_ERR_TIMEOUT on expiry, then the CTA unwinds).
#pragma once
#include "common.cuh"
#include "ptx.cuh"
#include <cuda_bf16.h>

namespace bsa {

struct FwdParams {
  int B, H, N, nb, nbw, nqt, n_items;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  float scale_log2;               // softmax scale * log2(e)
  float scale;                    // softmax scale
  __nv_bfloat16* o;
  float* lse;
  __nv_bfloat16* o_res;           // optional: the fp32 O minus its bf16 rounding, as bf16
  unsigned long long wait_ns;     // bound on every wait
  int* item_counter;              // zeroed before launch; null: items dealt statically
};

// Softmax warps: two per TMEM lane quarter, 64 keys each, the two halves
// exchanging their row maxima.
constexpr int kSoftmaxWarps = 8;
constexpr int kFwdThreads = (4 + kSoftmaxWarps) * 32;

// Lazy rescale: a row keeps its running max m (and the scale of O and of its
// sum) until a step's max exceeds m by more than this many exp2 units, so P =
// 2^((s - m) c) stays below 2^kLazyRescaleLog2.  Any value is exact (the final
// O/l and LSE use the same m); the bound only keeps the fp32 sums finite: l
// and O (l times a convex combination of V) stay below 2^kLazyRescaleLog2
// times the number of keys (at most 2^23) times max|v|.  2^8 rescaled O on 14%
// of the CogVideoX layer's steps (measured on B200); 2^20 almost never does.
constexpr float kLazyRescaleLog2 = 20.0f;

template <int D, int BLK>
struct FwdCfg {
  static constexpr int SLOTS = 128 / BLK;            // kv-blocks per step
  static constexpr int QB = 128 / BLK;               // q-blocks per tile
  static constexpr int NCH = D / 64;                 // 64-column swizzle chunks
  static constexpr int TILE = 128 * D * 2;           // bytes of a 128-row tile
  static constexpr int CHUNK = 128 * 128;            // bytes of one 128x64 chunk
  static constexpr int NK = D == 128 ? 2 : 4;        // K ring depth
  static constexpr int NV = D == 128 ? 2 : 4;        // V ring depth
  static constexpr int NM = 8;                       // step entries
  static constexpr int LCAP = 512;                   // union entries per list segment
  static constexpr int RW = LCAP / 32;               // bitmap words per fill round (<= LCAP bits)
  static_assert(RW >= 1 && RW <= 32, "fill round must fit one warp and one segment");
  static_assert(NM > NK + 2, "a step entry is reused only after its step's P is stored");
  static constexpr int Q_OFF = 0;                    // Q0, Q1 (item parity)
  static constexpr int K_OFF = 2 * TILE;
  static constexpr int V_OFF = K_OFF + NK * TILE;
  static constexpr int AUX_OFF = V_OFF + NV * TILE;
  static constexpr int BAR_BYTES = 512;
  // k/v full+free, q full/free, s_full, p_full, o done/free, m_full, l
  // full/free, drain, pair, pv_done
  static constexpr int NBARS = 2 * NK + 2 * NV + 2 * 6 + NM + 4 + 1 + 4 + 1;
  static_assert(NBARS * 8 <= BAR_BYTES, "mbarriers must fit their area");
  static constexpr int SMETA_OFF = AUX_OFF + BAR_BYTES;          // NM step entries
  static constexpr int SMETA_INTS = 24;
  static constexpr int VQ = 8;                                   // V-front queue entries
  static constexpr int VQ_INTS = VQ * 12;                        // producer V-front queue
  static constexpr int HDR_OFF = SMETA_OFF + (NM * SMETA_INTS + VQ_INTS) * 4;   // 2 headers x 8 ints
  static constexpr int MISC_OFF = HDR_OFF + 2 * 8 * 4;
  static constexpr int LIST_OFF = MISC_OFF + 64;                 // 2 bufs x LCAP
  static constexpr int BM_OFF = LIST_OFF + 2 * LCAP * 4;         // q-block bitmaps
  static constexpr int kMaxBitmapBytes = 4096;
  static constexpr int XCH_OFF = BM_OFF + kMaxBitmapBytes;       // row max / sum exchange
  static constexpr int XCH_BYTES = (2 * 2 * 128 + 2 * 128) * 4;
  static constexpr int SMEM = XCH_OFF + XCH_BYTES + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory over the per-CTA limit");
  static constexpr int S_COL = 0, O_COL = 256;
};

// entry kinds (list headers and step entries)
constexpr int kEntryNormal = 0, kEntryEnd = 2;

// list segment header (ints): [0] kind (0 segment, 2 end) [1] bh [2] qt [3] nq
//                             [4] count [5] first segment [6] last segment
// list entry: kv-block id | (keep bits over the tile's q-blocks) << 16

// step entry, as ints:
//  [0] kind (0 normal, 2 end)  [1] first  [2] last  [3] nvalid  [4] bh  [5] qt
//  [6..13] block ids          [14..21] keep bits (q-blocks of the tile)
//  [22] ring index of the step (K slot = ring % NK, V slot = ring % NV)
__device__ __forceinline__ float fast_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe (Cody-Waite reduction, then a minimax polynomial):
// n = round(x) through the 1.5*2^23 rounding constant, f = x - n in [-1/2, 1/2],
// 2^f ~ c0 + f(c1 + f(c2 + f c3)) (relative error 7.5e-5, fitted by
// fit_exp2_poly.py), and 2^n added into the exponent field.  x is clamped to
// [-126, ...] so the exponent add cannot wrap; below x = -125 the result is a
// non-negative value under 2^-124 (exact exp2 there is below 3e-38).  Used for a share of the softmax
// exponentials so that the MUFU pipe is not the bottleneck.
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -126.0f);
  const float t = x + 12582912.0f;
  const float f = x - (t - 12582912.0f);
  const float q = fmaf(fmaf(fmaf(0.0551716685295105f, f, 0.2426111251115799f), f,
                            0.6932609677314758f),
                       f, 0.9999280571937561f);
  return __int_as_float(__float_as_int(q) + (__float_as_int(t) << 23));
}

// Packed two-wide fp32 arithmetic (one instruction for two scores).
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Pairs (of 16 per 32-column chunk) whose exponentials go to the FMA pipe.
// Measured on B200: the polynomial costs ~9.5 issue cycles per warp-element
// against MUFU's 8-cycle pipe occupancy, so it only pays once the softmax is
// MUFU-bound with idle issue slots; off for now.
constexpr int kPolyPairs = 0;

__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap* m, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

// Producer state (kept in registers).
struct ProdSlot {
  int sc = 0;         // list segments consumed so far
  int pos = 0, count = 0;
  int bh = 0, qt = 0, nq = 0;
  int qcount = 0;     // Q tiles loaded
  bool have = false, lastseg = false, first_tile = false, flushed = false;
  bool need_q = false;  // the current item's Q tile is not loaded yet
};

// Scheduler state.
struct SchedSlot {
  int item = 0;       // current item
  int fills = 0;      // segments published
  int wpos = 0;       // next bitmap word of the current item
  int bh = 0, qt = 0, nq = 0;
  int total = 0, emitted = 0;   // union size of the current item, entries published
  bool mid = false;   // current item has more segments
  bool done = false;
};

// RES: also write O's rounding residual (p.o_res); a separate instantiation so
// that the plain forward carries none of its code.
template <int D, int BLK, bool RES>
__global__ void __launch_bounds__(kFwdThreads, 1)
    bsa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<D, BLK>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::AUX_OFF);
  uint64_t* k_full = bars;                       // [NK]
  uint64_t* k_free = k_full + C::NK;             // [NK]
  uint64_t* v_full = k_free + C::NK;             // [NV]
  uint64_t* v_free = v_full + C::NV;             // [NV]
  uint64_t* q_full = v_free + C::NV;             // [2] by item parity
  uint64_t* q_free = q_full + 2;                 // [2]
  uint64_t* s_full = q_free + 2;                 // [2] by step parity
  uint64_t* p_full = s_full + 2;                 // [2] by step parity
  uint64_t* o_done = p_full + 2;                 // [2] by item parity
  uint64_t* o_free = o_done + 2;                 // [2]
  uint64_t* m_full = o_free + 2;                 // [NM]
  uint64_t* l_full = m_full + C::NM;             // [2]
  uint64_t* l_free = l_full + 2;                 // [2]
  uint64_t* mma_drain = l_free + 2;              // [1]
  uint64_t* pair_bar = mma_drain + 1;            // [4 lane quarters]
  uint64_t* pv_done = pair_bar + 4;              // [1] one phase per PV
  int* smeta = reinterpret_cast<int*>(smem + C::SMETA_OFF);
  int* hdr = reinterpret_cast<int*>(smem + C::HDR_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  int* abort_flag = reinterpret_cast<int*>(smem + C::MISC_OFF + 4);
  uint32_t* lists = reinterpret_cast<uint32_t*>(smem + C::LIST_OFF);
  uint32_t* bm = reinterpret_cast<uint32_t*>(smem + C::BM_OFF);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nbw = p.nbw;

  if (tid == 0) {
    for (int s = 0; s < C::NK; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_free[s], 1);
    }
    for (int s = 0; s < C::NV; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_free[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&q_full[x], 1);
      mbar_init(&q_free[x], 1);
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], kSoftmaxWarps);   // one arrive per softmax warp
      mbar_init(&o_done[x], 1);
      mbar_init(&o_free[x], kSoftmaxWarps);
      mbar_init(&l_full[x], 1);
      mbar_init(&l_free[x], 1);
    }
    for (int s = 0; s < C::NM; ++s) mbar_init(&m_full[s], 1);
    mbar_init(mma_drain, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&pair_bar[i], 2);   // one arrive per warp
    mbar_init(pv_done, 1);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 3) {
    // ================================================================ scheduler
    // Next item, its q-block bitmaps, then the ascending union list in
    // segments of at most LCAP entries.  CTA c starts on item c; later items
    // come from a grid-wide counter, so SMs that run faster take more items
    // (without a counter: round-robin, c + kG).
    SchedSlot st;
    st.item = blockIdx.x;
    auto next_item = [&](int cur) -> int {
      if (p.item_counter == nullptr) return cur + static_cast<int>(gridDim.x);
      int v = 0;
      if (lane == 0) v = static_cast<int>(gridDim.x) + atomicAdd(p.item_counter, 1);
      return __shfl_sync(0xffffffffu, v, 0);
    };
    uint64_t t_last = global_ns();
    auto publish = [&]() -> bool {
      // returns true if a segment (or the end marker) was published
      const int b = st.fills & 1;
      if (st.fills >= 2) {
        // one lane polls, the warp follows its answer
        bool ready = lane == 0 && mbar_test_wait(&l_free[b], ((st.fills >> 1) - 1) & 1);
        if (!__shfl_sync(0xffffffffu, ready, 0)) return false;
      }
      int* h = hdr + b * 8;
      uint32_t* list = lists + b * C::LCAP;
      bool first_seg = false;
      while (!st.mid) {
        if (st.item >= p.n_items) {
          if (lane == 0) {
            h[0] = kEntryEnd;
            mbar_arrive(&l_full[b]);
          }
          __syncwarp();
          st.done = true;
          ++st.fills;
          return true;
        }
        st.bh = st.item / p.nqt;
        st.qt = st.item % p.nqt;
        const int qb0 = st.qt * C::QB;
        st.nq = min(C::QB, p.nb - qb0);
        for (int e = lane; e < C::QB * nbw; e += 32) bm[e] = 0u;
        __syncwarp();
        for (int qq = 0; qq < st.nq; ++qq) {
          const long long r = (long long)st.bh * p.nb + qb0 + qq;
          const int e0 = p.row_ptr[r], e1 = p.row_ptr[r + 1];
          for (int e = e0 + lane; e < e1; e += 32) {
            const int c = p.col_idx[e];
            if (c >= 0 && c < p.nb)
              atomicOr(&bm[qq * nbw + (c >> 5)], 1u << (c & 31));
            else
              record_error(BSA_ERR_CSR);
          }
        }
        __syncwarp();
        int cnt = 0;
        for (int wd = lane; wd < nbw; wd += 32) {
          uint32_t u = 0;
          for (int qq = 0; qq < st.nq; ++qq) u |= bm[qq * nbw + wd];
          cnt += __popc(u);
        }
        cnt = warp_sum(cnt);
        st.item = next_item(st.item);
        if (cnt == 0) {
          // no row of this tile lists anything: O = 0, LSE = -inf
          for (int r = 0; r < 128; ++r) {
            const int token = st.qt * 128 + r;
            if (token >= p.N) break;
            uint4* dst = reinterpret_cast<uint4*>(p.o + ((long long)st.bh * p.N + token) * D);
            for (int c = lane; c < D / 8; c += 32) dst[c] = make_uint4(0u, 0u, 0u, 0u);
            if (RES) {
              uint4* dr = reinterpret_cast<uint4*>(p.o_res + ((long long)st.bh * p.N + token) * D);
              for (int c = lane; c < D / 8; c += 32) dr[c] = make_uint4(0u, 0u, 0u, 0u);
            }
            if (lane == 0 && p.lse) p.lse[(long long)st.bh * p.N + token] = -INFINITY;
          }
          continue;
        }
        if (lane == 0)
          for (int c = 0; c < C::NCH; ++c) tma_prefetch_l2_3d(&tm_q, c * 64, st.qt * 128, st.bh);
        st.mid = true;
        st.wpos = 0;
        st.total = cnt;
        st.emitted = 0;
        first_seg = true;
      }
      // fill the segment from the union, RW bitmap words per round; a round
      // holds at most RW * 32 = LCAP blocks, so an empty segment always takes
      // at least one round
      int n = 0;
      while (st.wpos < nbw) {
        const int wd = st.wpos + lane;
        uint32_t u = 0;
        if (lane < C::RW && wd < nbw)
          for (int qq = 0; qq < st.nq; ++qq) u |= bm[qq * nbw + wd];
        const int c = __popc(u);
        const int incl = warp_incl_scan(c);
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        if (n + total > C::LCAP) break;  // rest goes to the next segment
        int at = n + incl - c;
        while (u) {
          const int bit = __ffs(u) - 1;
          u &= u - 1;
          const int blk = wd * 32 + bit;
          uint32_t keep = 0;
          for (int qq = 0; qq < st.nq; ++qq) keep |= ((bm[qq * nbw + wd] >> bit) & 1u) << qq;
          list[at++] = static_cast<uint32_t>(blk) | (keep << 16);
        }
        n += total;
        st.wpos += C::RW;
      }
      st.emitted += n;
      const bool last_seg = st.emitted >= st.total;   // never an empty tail segment
      __syncwarp();
      if (lane == 0) {
        h[0] = 0;
        h[1] = st.bh;
        h[2] = st.qt;
        h[3] = st.nq;
        h[4] = n;
        h[5] = first_seg;
        h[6] = last_seg;
        mbar_arrive(&l_full[b]);
      }
      __syncwarp();
      st.mid = !last_seg;
      ++st.fills;
      return true;
    };
    while (!st.done) {
      if (__any_sync(0xffffffffu, *(volatile int*)abort_flag != 0)) break;
      if (publish()) {
        t_last = global_ns();
      } else if (global_ns() - t_last > p.wait_ns) {
        if (lane == 0) record_error(BSA_ERR_TIMEOUT);
        *(volatile int*)abort_flag = 1;
        break;
      }
    }
  } else if (warp == 0) {
    // ================================================================ producer
    // Two fronts over the ring: the K front publishes entry sk (step entry, K
    // boxes) once K slot sk % NK is free; the V front loads the V boxes of
    // entry sv < sk once V slot sv % NV is free.  V is needed one entry later
    // than K, so a PV still running never holds back the next K.
    if (lane == 0) {
      ProdSlot P;
      int sk = 0, sv = 0;  // next ring index for K / for V
      bool ok = true;
      int* vq = smeta + C::NM * C::SMETA_INTS;   // V-front queue: VQ entries x 12 ints
      bool used_ring = false;
      // One pass of the V front: loads every V tile whose slot is free.
      auto v_front = [&]() -> bool {
        bool moved = false;
        while (sv < sk && (sv < C::NV || mbar_test_wait(&v_free[sv % C::NV], ((sv / C::NV) - 1) & 1))) {
          const int* vqe = vq + (sv % C::VQ) * 12;
          const int vs = sv % C::NV;
          mbar_arrive_expect_tx(&v_full[vs], C::TILE);
#pragma unroll
          for (int sl = 0; sl < C::SLOTS; ++sl)
#pragma unroll
            for (int c = 0; c < C::NCH; ++c)
              tma_load_3d(smem + C::V_OFF + vs * C::TILE + c * C::CHUNK + sl * BLK * 128, &tm_v,
                          &v_full[vs], c * 64, vqe[2 + sl] * BLK, vqe[1]);
          ++sv;
          moved = true;
        }
        return moved;
      };
      // One K-front entry.  Returns false on a wait that gave up.
      auto k_step = [&]() -> bool {
        used_ring = false;
        int* vqe = vq + (sk % C::VQ) * 12;
        if (!P.have || P.pos == P.count) {
          if (P.have) {
            mbar_arrive(&l_free[(P.sc - 1) & 1]);
            P.have = false;
          }
          const int b = P.sc & 1;
          if (!mbar_wait(&l_full[b], (P.sc >> 1) & 1, p.wait_ns)) return false;
          const int* h = hdr + b * 8;
          ++P.sc;
          if (h[0] == kEntryEnd) {
            // stream finished: END entry for the softmax and MMA threads (no ring slot)
            int* sm = smeta + (sk % C::NM) * C::SMETA_INTS;
            sm[0] = kEntryEnd;
            mbar_arrive(&m_full[sk % C::NM]);
            P.flushed = true;
            return true;
          }
          P.have = true;
          P.pos = 0;
          P.count = h[4];
          P.lastseg = h[6] != 0;
          if (P.count == 0) return false;   // never published; refuse to spin on it
          if (h[5]) {
            P.bh = h[1];
            P.qt = h[2];
            P.nq = h[3];
            P.first_tile = true;
            P.need_q = true;
          }
        }
        if (P.need_q) {
          // Q tile into buffer qcount % 2, after the last QK of the item two
          // before.  While waiting, keep the V front going: that QK follows a
          // PV whose V tile this same thread's V front may still have to load.
          const int qb = P.qcount & 1;
          if (P.qcount >= 2 && !mbar_test_wait(&q_free[qb], ((P.qcount >> 1) - 1) & 1)) {
            const uint64_t t0 = global_ns();
            while (!mbar_test_wait(&q_free[qb], ((P.qcount >> 1) - 1) & 1)) {
              v_front();
              if (global_ns() - t0 > p.wait_ns) return false;
            }
          }
          mbar_arrive_expect_tx(&q_full[qb], C::TILE);
#pragma unroll
          for (int c = 0; c < C::NCH; ++c)
            tma_load_3d(smem + C::Q_OFF + qb * C::TILE + c * C::CHUNK, &tm_q, &q_full[qb], c * 64,
                        P.qt * 128, P.bh);
          ++P.qcount;
          P.need_q = false;
        }
        const uint32_t* list = lists + ((P.sc - 1) & 1) * C::LCAP;
        int* sm = smeta + (sk % C::NM) * C::SMETA_INTS;
        const int nvalid = min(C::SLOTS, P.count - P.pos);
        const uint32_t e0 = list[P.pos];
#pragma unroll
        for (int sl = 0; sl < C::SLOTS; ++sl) {
          const uint32_t e = sl < nvalid ? list[P.pos + sl] : e0;   // unused: reload a listed block
          const int blk = static_cast<int>(e & 0xFFFFu);
          sm[6 + sl] = blk;
          sm[14 + sl] = sl < nvalid ? static_cast<int>(e >> 16) : 0;
          vqe[2 + sl] = blk;
        }
        vqe[0] = kEntryNormal;
        vqe[1] = P.bh;
        P.pos += nvalid;
        const int first = P.first_tile ? 1 : 0;
        const int lastt = (P.lastseg && P.pos == P.count) ? 1 : 0;
        P.first_tile = false;
        sm[0] = kEntryNormal;
        sm[1] = first;
        sm[2] = lastt;
        sm[3] = nvalid;
        sm[4] = P.bh;
        sm[5] = P.qt;
        sm[22] = sk;   // ring index: K slot sk % NK, V slot sk % NV
        mbar_arrive(&m_full[sk % C::NM]);
        used_ring = true;
        const int ks = sk % C::NK;
        mbar_arrive_expect_tx(&k_full[ks], C::TILE);
#pragma unroll
        for (int sl = 0; sl < C::SLOTS; ++sl)
#pragma unroll
          for (int c = 0; c < C::NCH; ++c)
            tma_load_3d(smem + C::K_OFF + ks * C::TILE + c * C::CHUNK + sl * BLK * 128, &tm_k,
                        &k_full[ks], c * 64, vqe[2 + sl] * BLK, P.bh);
        return true;
      };
      uint64_t t_last = global_ns();
      while (ok) {
        if (*(volatile int*)abort_flag) break;
        bool prog = false;
        // ---- K front
        // (the K front stays less than VQ entries ahead of the V front, whose
        // queue entry it writes; entry sk reuses the step entry of sk - NM,
        // whose step's P was stored before QK(sk - NK) was issued)
        if (!P.flushed && sk - sv < C::VQ &&
            (sk < C::NK || mbar_test_wait(&k_free[sk % C::NK], ((sk / C::NK) - 1) & 1))) {
          ok = k_step();
          if (!ok) break;
          if (used_ring) ++sk;
          prog = true;
        }
        // ---- V front
        if (v_front()) prog = true;
        if (P.flushed && sv == sk) break;
        if (prog) {
          t_last = global_ns();
        } else if (global_ns() - t_last > p.wait_ns) {
          ok = false;
          break;
        }
      }
      if (!ok) {
        record_error(BSA_ERR_TIMEOUT);
        *(volatile int*)abort_flag = 1;
      }
      // drain: the loads of the last ring entries (and Q) land before exit
      for (int t = sk > C::NK ? sk - C::NK : 0; t < sk; ++t)
        mbar_wait(&k_full[t % C::NK], (t / C::NK) & 1, p.wait_ns);
      for (int t = sv > C::NV ? sv - C::NV : 0; t < sv; ++t)
        mbar_wait(&v_full[t % C::NV], (t / C::NV) & 1, p.wait_ns);
      for (int t = P.qcount > 2 ? P.qcount - 2 : 0; t < P.qcount; ++t)
        mbar_wait(&q_full[t & 1], (t >> 1) & 1, p.wait_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    // One thread issues every MMA of the CTA, step by step: QK(t) needs only
    // K(t) (and, on an item's first step, its Q tile), so the tensor pipe
    // computes S(t) while the softmax works on step t-1; PV(t-1) needs that
    // step's P.  Whichever is ready first goes first.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      // descriptor bases; per-instruction offsets are compile-time adds to the
      // address field (addresses stay below 2^18, so the 14-bit field never carries)
      const uint64_t dq0 = smem_desc(smem_u32(smem + C::Q_OFF), 16, 1024);
      const uint64_t dk0 = smem_desc(smem_u32(smem + C::K_OFF), 16, 1024);
      const uint64_t dv0 = smem_desc(smem_u32(smem + C::V_OFF), C::CHUNK, 1024);
      int pend = -1, pend_first = 0, pend_last = 0, pend_item = 0;
      int items = 0, cur_item = -1;
      bool ok = true, issued = false;
      // PV of the pending step: its V tile, its P and (first step of an item)
      // the O buffer, all polled without blocking
      auto pv_ready = [&]() -> bool {
        const int sp = pend;
        if (!mbar_test_wait(&v_full[sp % C::NV], (sp / C::NV) & 1)) return false;
        // the first PV of an item overwrites its O buffer: the epilogue of
        // the item two before must have read it
        if (pend_first && pend_item >= 2 &&
            !mbar_test_wait(&o_free[pend_item & 1], ((pend_item >> 1) - 1) & 1))
          return false;
        return mbar_test_wait(&p_full[sp & 1], (sp >> 1) & 1);
      };
      auto issue_pv = [&]() {
        const int sp = pend;
        const int ob = pend_item & 1;
        tc_fence_after();
        const uint32_t t_o = tmem + C::O_COL + ob * 128;
        const uint32_t t_p = tmem + C::S_COL + (sp & 1) * 128;   // P over S
        const uint64_t dv = dv0 + static_cast<uint64_t>(((sp % C::NV) * C::TILE) >> 4);
        const uint32_t acc0 = pend_first ? 0u : 1u;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(t_o, t_p + kk * 8, dv + static_cast<uint64_t>((kk * 2048) >> 4), idesc_pv,
                 kk == 0 ? acc0 : 1u);
        mma_commit(&v_free[sp % C::NV]);
        mma_commit(pv_done);
        if (pend_last) mma_commit(&o_done[ob]);
        pend = -1;
      };
      // Step t's slot holds QK(t) and PV(t-1), issued in whichever order
      // their inputs arrive (QK(t) needs PV(t-2) issued before it, which the
      // previous slot guarantees; PV(t-1) needs QK(t-1), likewise).
      for (int t = 0; ok; ++t) {
        const int mi = t % C::NM;
        bool have = false, end = false, qk_done = false;
        int first = 0, lastt = 0, s = 0;
        uint64_t t0 = global_ns();
        while (true) {
          bool prog = false;
          if (!have && mbar_test_wait(&m_full[mi], (t / C::NM) & 1)) {
            const int* sm = smeta + mi * C::SMETA_INTS;
            have = true;
            end = sm[0] == kEntryEnd;
            first = sm[1];
            lastt = sm[2];
            s = sm[22];
            prog = true;
          }
          if (have && !end && !qk_done && mbar_test_wait(&k_full[s % C::NK], (s / C::NK) & 1) &&
              (!first || mbar_test_wait(&q_full[items & 1], (items >> 1) & 1))) {
            if (first) cur_item = items++;
            tc_fence_after();
            // S(t % 2) was last read as P(t-2) by PV(t-2), issued before this QK
            const int ks = s % C::NK;
            const uint32_t t_s = tmem + C::S_COL + (t & 1) * 128;
            const uint64_t dq = dq0 + static_cast<uint64_t>(((cur_item & 1) * C::TILE) >> 4);
            const uint64_t dk = dk0 + static_cast<uint64_t>((ks * C::TILE) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::CHUNK + (kk & 3) * 32) >> 4);
              mma_ss(t_s, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
            }
            issued = true;
            mma_commit(&k_free[ks]);
            if (lastt) mma_commit(&q_free[cur_item & 1]);
            mma_commit(&s_full[t & 1]);
            qk_done = true;
            prog = true;
          }
          if (pend >= 0 && pv_ready()) {
            issue_pv();
            prog = true;
          }
          if (pend < 0 && have && (end || qk_done)) break;
          if (prog) {
            t0 = global_ns();
          } else if (global_ns() - t0 > p.wait_ns) {
            ok = false;
            break;
          }
        }
        if (!ok || end) break;
        pend = s;
        pend_first = first;
        pend_last = lastt;
        pend_item = cur_item;
      }
      if (!ok) {
        record_error(BSA_ERR_TIMEOUT);
        *(volatile int*)abort_flag = 1;
      }
      if (issued) {
        mma_commit(mma_drain);
        mbar_wait(mma_drain, 0, p.wait_ns);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ================================================================ softmax
    // Warp (q, h): q = TMEM lane quarter (rows 32q..32q+31), h = key part
    // (keys KW*h .. KW*h+KW-1 of each 128-key step).  The two halves of a row
    // agree on the running max through shared memory and a two-warp mbarrier.
    constexpr int NH = kSoftmaxWarps / 4;     // key parts per row
    constexpr int KW = 128 / NH;              // keys per warp and step
    constexpr int DW = D / NH;                // O columns per warp in rescale and epilogue
    static_assert(NH == 2, "the max exchange pairs two warps");
    const int h = (warp - 4) >> 2;
    const int wq = warp & 3;                  // TMEM lane quarter
    const int row = wq * 32 + lane;           // query row in the tile
    const int qq = row / BLK;                 // its q-block in the tile
    uint64_t* pbar = &pair_bar[wq];           // the two warps of this lane quarter
    int puse = 0;
    // every lane's prior shared-memory writes and tcgen05 operations are
    // ordered before lane 0's arrive by the warp barrier
    auto warp_arrive = [&](uint64_t* bar) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    auto pair_sync = [&]() -> bool {
      warp_arrive(pbar);
      const bool r = mbar_wait(pbar, puse & 1, p.wait_ns);
      ++puse;
      tc_fence_after();
      return __all_sync(0xffffffffu, r);
    };
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    float* xmax = reinterpret_cast<float*>(smem + C::XCH_OFF);        // [2 step parity][2 halves][128]
    float* xsum = xmax + 2 * 2 * 128;                                 // [2 halves][128]
    const float c2 = p.scale_log2;
    float m_run = -INFINITY;   // running max of raw scores (same in every part of a row)
    float l_run = 0.f;         // this part's running sum
    int items = 0, cur_item = -1;
    bool ok = true;
    // an item's epilogue, deferred until the next item's first step is done
    bool pe = false;
    int pe_item = 0, pe_bh = 0, pe_qt = 0;
    float pe_m = 0.f, pe_l = 0.f;
    auto epilogue = [&]() -> bool {
      const int ob = pe_item & 1;
      const uint32_t o_col = C::O_COL + ob * 128;
      const int token = pe_qt * 128 + row;
      bool w_ok = mbar_wait(&o_done[ob], (pe_item >> 1) & 1, p.wait_ns);
      if (!__all_sync(0xffffffffu, w_ok)) return false;
      tc_fence_after();
      float* xs = xsum;
      xs[h * 128 + row] = pe_l;
      if (!pair_sync()) return false;
      const float l_tot = pe_l + xs[(h ^ 1) * 128 + row];
      const float inv_l = l_tot > 0.f ? 1.0f / l_tot : 0.f;
      __nv_bfloat16* orow = p.o + ((long long)pe_bh * p.N + token) * D + h * DW;
#pragma unroll 1
      for (int c = 0; c < DW / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(t_lane + o_col + h * DW + c * 32, r);
        tmem_wait_ld();
        uint32_t packed[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          __nv_bfloat162 hb = __floats2bfloat162_rn(__uint_as_float(r[2 * e]) * inv_l,
                                                    __uint_as_float(r[2 * e + 1]) * inv_l);
          packed[e] = *reinterpret_cast<uint32_t*>(&hb);
        }
        if (token < p.N) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2],
                                packed[4 * e + 3]);
        }
        if (RES && token < p.N) {
          // the rounding residual of each element, so that O + residual
          // carries the fp32 result to about 2^-16
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float a = __uint_as_float(r[2 * e]) * inv_l;
            const float b = __uint_as_float(r[2 * e + 1]) * inv_l;
            const float2 hi = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&packed[e]));
            __nv_bfloat162 lo = __floats2bfloat162_rn(a - hi.x, b - hi.y);
            packed[e] = *reinterpret_cast<uint32_t*>(&lo);
          }
          uint4* dr = reinterpret_cast<uint4*>(p.o_res + ((long long)pe_bh * p.N + token) * D +
                                               h * DW + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dr[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2],
                               packed[4 * e + 3]);
        }
      }
      warp_arrive(&o_free[ob]);
      if (h == 0 && p.lse != nullptr && token < p.N)
        p.lse[(long long)pe_bh * p.N + token] =
            l_tot > 0.f ? (pe_m * p.scale + logf(l_tot)) : -INFINITY;
      pe = false;
      return true;
    };
    // kv-block slots overlapping this warp's keys
    constexpr int SPW = BLK <= KW ? KW / BLK : 1;
    const int sl0 = BLK <= KW ? h * SPW : 0;
    const uint32_t warp_mask = ((1u << SPW) - 1u) << sl0;
    for (int t = 0;; ++t) {
      const int mi = t % C::NM;
      bool w_ok = mbar_wait(&m_full[mi], (t / C::NM) & 1, p.wait_ns) && !*(volatile int*)abort_flag;
      if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
      // the entry stays valid until this step's P is published; bh/qt are kept
      // in registers for the epilogue, which runs later
      const int* sm = smeta + mi * C::SMETA_INTS;
      if (sm[0] == kEntryEnd) break;
      const int first = sm[1], lastt = sm[2], nvalid = sm[3];
      const int e_bh = sm[4], e_qt = sm[5];
      // which slots of the step this row keeps, and the one partial block (the
      // last, < blk keys) if present; read before S lands
      uint32_t live_bits = 0;
      int part_slot = -1, part_keys = BLK;
#pragma unroll
      for (int sl = 0; sl < C::SLOTS; ++sl) {
        if (sl < nvalid && ((sm[14 + sl] >> qq) & 1)) {
          live_bits |= 1u << sl;
          const int nk = p.N - sm[6 + sl] * BLK;
          if (nk < BLK) {
            part_slot = sl;
            part_keys = nk;
          }
        }
      }
      const bool live_all = (live_bits & warp_mask) == warp_mask &&
                            (part_slot < sl0 || part_slot >= sl0 + SPW);
      if (first) {
        cur_item = items++;
        m_run = -INFINITY;
        l_run = 0.f;
      }
      const uint32_t s_col = C::S_COL + (t & 1) * 128;
      const uint32_t o_col = C::O_COL + (cur_item & 1) * 128;
      w_ok = mbar_wait(&s_full[t & 1], (t >> 1) & 1, p.wait_ns);
      if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
      tc_fence_after();
      // This warp's keys all belong to blocks the row's q-block does not list
      // (warp-uniform when blk >= 32: a warp's rows share one q-block): no
      // exponentials, P = 0.
      const bool part_dead = !__any_sync(0xffffffffu, (live_bits & warp_mask) != 0u);
      float x[KW];
#pragma unroll
      for (int c = 0; c < KW / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(t_lane + s_col + h * KW + c * 32, r);
#pragma unroll
        for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(r[e]);
      }
      tmem_wait_ld();
      float hmax = -INFINITY;
      if (!part_dead) {
        // masking: slots this row's q-block does not list, unused slots, keys >= N
        if (!__all_sync(0xffffffffu, live_all)) {
          // valid keys of each block in this warp's range, counted from the
          // range's first key of that block
          constexpr int SPAN = BLK < KW ? BLK : KW;
          int nk_loc[KW / SPAN];
#pragma unroll
          for (int b = 0; b < KW / SPAN; ++b) {
            const int sl = BLK <= KW ? sl0 + b : 0;
            const int nk = ((live_bits >> sl) & 1u) ? (sl == part_slot ? part_keys : BLK) : 0;
            nk_loc[b] = BLK <= KW ? nk : nk - h * KW;
          }
#pragma unroll
          for (int c = 0; c < KW; ++c)
            if (c % SPAN >= nk_loc[c / SPAN]) x[c] = -INFINITY;
        }
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < KW; c += 8) {
          mx0 = fmax3(mx0, x[c], x[c + 1]);
          mx1 = fmax3(mx1, x[c + 2], x[c + 3]);
          mx2 = fmax3(mx2, x[c + 4], x[c + 5]);
          mx3 = fmax3(mx3, x[c + 6], x[c + 7]);
        }
        hmax = fmax3(fmax3(mx0, mx1, mx2), mx3, mx3);
      }
      // agree on the row max with the other half (double-buffered by step
      // parity); the barrier also orders both halves' S reads before any P write
      float* xm = xmax + (t & 1) * 2 * 128;
      xm[h * 128 + row] = hmax;
      if (!pair_sync()) { ok = false; break; }
      const float tmax = fmaxf(hmax, xm[(h ^ 1) * 128 + row]);
      // lazy rescale (decided per warp: tcgen05.ld/st are warp-collective)
      const float m_new = fmaxf(m_run, tmax);
      const bool grow = m_run == -INFINITY ? (m_new > -INFINITY)
                                           : ((m_new - m_run) * c2 > kLazyRescaleLog2);
      float alpha = 1.0f;
      if (grow) {
        alpha = (m_run == -INFINITY) ? 0.0f : fast_ex2((m_run - m_new) * c2);
        m_run = m_new;
      }
      if (!first && __any_sync(0xffffffffu, grow)) {
        // O holds PV up to step t-2; wait for PV(t-1), then scale this warp's
        // columns before the PV of this step
        w_ok = mbar_wait(pv_done, (t - 1) & 1, p.wait_ns);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < DW / 16; ++c) {
          uint32_t r[16];
          tmem_ld16(t_lane + o_col + h * DW + c * 16, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st16(t_lane + o_col + h * DW + c * 16, r);
        }
      }
      const float neg_m = m_run == -INFINITY ? 0.f : -m_run * c2;
      const uint64_t c2x2 = pack2(c2, c2), nmx2 = pack2(neg_m, neg_m);
      uint64_t ls2a = pack2(0.f, 0.f), ls2b = pack2(0.f, 0.f);
      const bool emu = kPolyPairs > 0 && __all_sync(0xffffffffu, live_all);
#pragma unroll
      for (int q2 = 0; q2 < KW / 32; ++q2) {
        uint32_t pk[16];
        if (part_dead) {
#pragma unroll
          for (int c = 0; c < 16; ++c) pk[c] = 0u;
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int col = q2 * 32 + 2 * c;
            float a0, a1;
            unpack2(ffma2(pack2(x[col], x[col + 1]), c2x2, nmx2), a0, a1);
            float p0, p1;
            if (emu && (c & 15) >= 16 - kPolyPairs) {
              p0 = exp2_poly(a0);
              p1 = exp2_poly(a1);
            } else {
              p0 = fast_ex2(a0);
              p1 = fast_ex2(a1);
            }
            if (c & 1)
              ls2b = fadd2(ls2b, pack2(p0, p1));
            else
              ls2a = fadd2(ls2a, pack2(p0, p1));
            __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
            pk[c] = *reinterpret_cast<uint32_t*>(&hb);
          }
        }
        // P (bf16 pairs) over S: keys KW h + 32 q2 .. +31 -> columns KW/2 h + 16 q2
        tmem_st16(t_lane + s_col + h * (KW / 2) + q2 * 16, pk);
      }
      float la0, la1, lb0, lb1;
      unpack2(ls2a, la0, la1);
      unpack2(ls2b, lb0, lb1);
      l_run = l_run * alpha + ((la0 + la1) + (lb0 + lb1));
      tmem_wait_st();
      warp_arrive(&p_full[t & 1]);
      if (pe && !epilogue()) { ok = false; break; }
      if (lastt) {
        pe = true;
        pe_item = cur_item;
        pe_bh = e_bh;
        pe_qt = e_qt;
        pe_m = m_run;
        pe_l = l_run;
      }
    }
    if (ok && pe && !epilogue()) ok = false;
    if (!ok) {
      record_error(BSA_ERR_TIMEOUT);
      *(volatile int*)abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
}

}  // namespace bsa
