// bsa_api.cu -- the C ABI of include/bsa.h: host-side validation, TMA tensor
// maps and kernel launches.  Every compute step runs in the kernels included
// below; this file only checks arguments, sizes grids and launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cmath>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>

#include "../../include/bsa.h"
#include "common.cuh"
#include "pattern.cuh"
#include "asa_mask.cuh"
#include "bsa_fwd.cuh"
#include "bsa_bwd.cuh"
#include "search.cuh"

namespace {

using bsa::FwdCfg;

constexpr unsigned long long kWaitNs = 1000000000ull;  // 1 s bound on device waits

inline cudaStream_t as_cuda(bsa_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

inline int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline bool blk_ok(int blk) { return blk == 16 || blk == 32 || blk == 64 || blk == 128; }

inline int check_launch() { return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA; }

int common_shape_checks(int B, int H, int N, int blk) {
  if (B <= 0 || H <= 0 || N <= 0 || blk <= 0) return BSA_ERR_INVALID_ARG;
  if (!blk_ok(blk)) return BSA_ERR_UNSUPPORTED;
  const long long nb = (N + blk - 1) / blk;
  if ((long long)B * H * nb * nb >= (1LL << 31)) return BSA_ERR_UNSUPPORTED;
  if ((long long)B * H > 65535) return BSA_ERR_UNSUPPORTED;  // grid.y
  return BSA_OK;
}

// ---- tensor maps ------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [B*H, N, d] bf16 viewed as a 3D tensor {d, N, B*H}; box {64, rows, 1}, 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, int BH, int N, int d, int rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---- per-device one-time settings --------------------------------------------
// Flags and cached values are atomics: host threads may make their first calls
// concurrently; repeating the setting is harmless, a data race would not be.
constexpr int kMaxDevices = 64;
using DeviceFlags = std::atomic<bool>[kMaxDevices];

// Raise a kernel's dynamic shared-memory limit once per device; `done` is that
// kernel's flag array.
template <typename K>
bool allow_smem(K kernel, int bytes, DeviceFlags& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
  if (dev < kMaxDevices && done[dev].load(std::memory_order_acquire)) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  if (dev < kMaxDevices) done[dev].store(true, std::memory_order_release);
  return true;
}

// ---- forward launch -----------------------------------------------------------
int sm_count() {
  static std::atomic<int> counts[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  int n = counts[dev].load(std::memory_order_acquire);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    counts[dev].store(n, std::memory_order_release);
  }
  return n;
}

template <int D, int BLK>
int launch_fwd(const void* q, const void* k, const void* v, int B, int H, int N,
               const int32_t* row_ptr, const int32_t* col_idx, float scale, void* o, float* lse,
               void* o_res, int* item_counter, cudaStream_t stream) {
  using C = FwdCfg<D, BLK>;
  const int nb = (N + BLK - 1) / BLK;
  const int nbw = (nb + 31) / 32;
  if ((long long)C::QB * nbw * 4 > C::kMaxBitmapBytes) return BSA_ERR_UNSUPPORTED;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, B * H, N, D, 128) || !make_map(&mk, k, B * H, N, D, BLK) ||
      !make_map(&mv, v, B * H, N, D, BLK))
    return BSA_ERR_CUDA;
  static DeviceFlags smem_set, smem_set_res;
  if (!allow_smem(bsa::bsa_fwd_kernel<D, BLK, false>, C::SMEM, smem_set) ||
      !allow_smem(bsa::bsa_fwd_kernel<D, BLK, true>, C::SMEM, smem_set_res))
    return BSA_ERR_CUDA;
  bsa::FwdParams p;
  p.B = B;
  p.H = H;
  p.N = N;
  p.nb = nb;
  p.nbw = nbw;
  p.nqt = ceil_div(N, 128);
  p.n_items = B * H * p.nqt;
  p.row_ptr = row_ptr;
  p.col_idx = col_idx;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.o_res = static_cast<__nv_bfloat16*>(o_res);
  p.wait_ns = kWaitNs;
  p.item_counter = item_counter;
  const int sms = sm_count();
  if (sms <= 0) return BSA_ERR_CUDA;
  // persistent: one CTA per SM, one stream of items per CTA
  const int grid = std::min(sms, p.n_items);
  if (o_res != nullptr)
    bsa::bsa_fwd_kernel<D, BLK, true><<<grid, bsa::kFwdThreads, C::SMEM, stream>>>(mq, mk, mv, p);
  else
    bsa::bsa_fwd_kernel<D, BLK, false><<<grid, bsa::kFwdThreads, C::SMEM, stream>>>(mq, mk, mv, p);
  return check_launch();
}

template <int D>
int launch_fwd_blk(int blk, const void* q, const void* k, const void* v, int B, int H, int N,
                   const int32_t* rp, const int32_t* ci, float scale, void* o, float* lse,
                   void* o_res, int* ctr, cudaStream_t s) {
  switch (blk) {
    case 16: return launch_fwd<D, 16>(q, k, v, B, H, N, rp, ci, scale, o, lse, o_res, ctr, s);
    case 32: return launch_fwd<D, 32>(q, k, v, B, H, N, rp, ci, scale, o, lse, o_res, ctr, s);
    case 64: return launch_fwd<D, 64>(q, k, v, B, H, N, rp, ci, scale, o, lse, o_res, ctr, s);
    case 128: return launch_fwd<D, 128>(q, k, v, B, H, N, rp, ci, scale, o, lse, o_res, ctr, s);
  }
  return BSA_ERR_UNSUPPORTED;
}

// ---- ASA mask sizes -------------------------------------------------------------
// Workspace: q̄ [rows][d] fp32 | k̄ᵀ [B*H][d][kt_ld] fp32 | bitmaps [rows][nbw] u32,
// each part starting on a 256-byte boundary.
struct AsaLayout {
  long long nb, nbw, rows, kt_ld;
  size_t qbar_off, kbar_off, bitmap_off, scan_off, total;
};

AsaLayout asa_layout(int B, int H, int N, int d, int blk) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  AsaLayout L;
  L.nb = (N + blk - 1) / blk;
  L.nbw = (L.nb + 31) / 32;
  L.rows = (long long)B * H * L.nb;
  L.kt_ld = (L.nb + 3) / 4 * 4;   // 16-byte rows for cp.async
  L.qbar_off = 0;
  L.kbar_off = up((size_t)L.rows * d * sizeof(float));
  L.bitmap_off = L.kbar_off + up((size_t)B * H * d * L.kt_ld * sizeof(float));
  // the select kernels' look-back state: a ticket, then one flag word per CTA
  // (at most one CTA per row)
  L.scan_off = L.bitmap_off + up((size_t)L.rows * L.nbw * sizeof(uint32_t));
  L.total = L.scan_off + 256 + up((size_t)L.rows * sizeof(unsigned long long));
  return L;
}

int select_cap(int nb, float ratio) {
  if (!(ratio > 0.f)) return nb;
  const int c = static_cast<int>(std::floor(static_cast<double>(ratio) * nb));
  return c < 1 ? 1 : (c > nb ? nb : c);
}

template <int D>
size_t select_generic_smem(int R, int nb_pad) {
  return (size_t)R * D * 4 + (size_t)bsa::kKChunk * (D + 1) * 4 + (size_t)R * nb_pad * 4 +
         (size_t)bsa::kSelWarps * 256 * 4 + (size_t)bsa::kSelWarps * 64 * 8;
}

template <int D, int NCB>
int launch_select_regs(bsa::SelectParams sp, int BH, cudaStream_t stream) {
  using T = bsa::SelTile<D, NCB>;
  sp.nb_pad = T::NB_PAD;
  sp.rows_per_cta = T::R;
  sp.dk = T::DK;
  sp.groups = static_cast<int>(ceil_div(sp.nb, T::R));
  static DeviceFlags done;
  if (!allow_smem(bsa::asa_select_kernel<D, NCB>, T::SMEM, done)) return BSA_ERR_CUDA;
  const dim3 grid(static_cast<unsigned>((long long)sp.groups * BH));
  bsa::asa_select_kernel<D, NCB><<<grid, 256, T::SMEM, stream>>>(sp);
  return check_launch() ? BSA_ERR_CUDA : BSA_OK;
}

template <int D>
int launch_asa(const void* q, const void* k, int B, int H, int N, int blk, int mode, int topk,
               float tau, float ratio, int keep_diag, int n_sink, float scale, int32_t* row_ptr,
               int32_t* col_idx, long long cap_entries, void* ws, cudaStream_t stream) {
  const AsaLayout L = asa_layout(B, H, N, D, blk);
  const int nb = static_cast<int>(L.nb), nbw = static_cast<int>(L.nbw);
  const int BH = B * H;
  if (BH > 65535) return BSA_ERR_UNSUPPORTED;
  char* base = static_cast<char*>(ws);
  float* qbar = reinterpret_cast<float*>(base + L.qbar_off);
  float* kbarT = reinterpret_cast<float*>(base + L.kbar_off);
  uint32_t* bitmaps = reinterpret_cast<uint32_t*>(base + L.bitmap_off);
  auto* scan_ticket = reinterpret_cast<unsigned int*>(base + L.scan_off);
  auto* scan_flags = reinterpret_cast<unsigned long long*>(base + L.scan_off + 256);
  const int n_flags = static_cast<int>(L.rows);
  // 1. pooling (also zeroes the select kernel's look-back state)
  {
    const long long units = 2LL * BH * nb;
    const auto* qq = static_cast<const __nv_bfloat16*>(q);
    const auto* kk = static_cast<const __nv_bfloat16*>(k);
    const int ld = static_cast<int>(L.kt_ld);
    const dim3 g(static_cast<unsigned>(units)), b(bsa::kPoolWarps * 32);
    switch (blk) {
      case 16: bsa::asa_pool_kernel<D, 16><<<g, b, 0, stream>>>(qq, kk, qbar, kbarT, BH, N, nb, ld, scan_flags, scan_ticket, n_flags); break;
      case 32: bsa::asa_pool_kernel<D, 32><<<g, b, 0, stream>>>(qq, kk, qbar, kbarT, BH, N, nb, ld, scan_flags, scan_ticket, n_flags); break;
      case 64: bsa::asa_pool_kernel<D, 64><<<g, b, 0, stream>>>(qq, kk, qbar, kbarT, BH, N, nb, ld, scan_flags, scan_ticket, n_flags); break;
      case 128: bsa::asa_pool_kernel<D, 128><<<g, b, 0, stream>>>(qq, kk, qbar, kbarT, BH, N, nb, ld, scan_flags, scan_ticket, n_flags); break;
      default: return BSA_ERR_UNSUPPORTED;
    }
    if (check_launch()) return BSA_ERR_CUDA;
  }
  // 2. scores + selection
  {
    bsa::SelectParams sp;
    sp.qbar = qbar;
    sp.kbarT = kbarT;
    sp.bitmaps = bitmaps;
    sp.row_ptr = row_ptr;
    sp.col_idx = col_idx;
    sp.capacity = cap_entries;
    sp.scan_flags = scan_flags;
    sp.scan_ticket = scan_ticket;
    sp.wait_ns = kWaitNs;
    sp.nb = nb;
    sp.nbw = nbw;
    sp.kt_ld = static_cast<int>(L.kt_ld);
    sp.dk = 0;
    sp.mode = mode;
    sp.topk = topk;
    sp.cap = select_cap(nb, ratio);
    sp.keep_diag = keep_diag;
    sp.n_sink = n_sink;
    sp.mass_tau = tau;
    sp.scale = scale;
    int rc = BSA_OK;
    const int ncb = (nb + 127) / 128;   // 128-column score blocks
    switch (ncb) {
      case 1: rc = launch_select_regs<D, 1>(sp, BH, stream); break;
      case 2: rc = launch_select_regs<D, 2>(sp, BH, stream); break;
      case 3: rc = launch_select_regs<D, 3>(sp, BH, stream); break;
      case 4: rc = launch_select_regs<D, 4>(sp, BH, stream); break;
      case 5: rc = launch_select_regs<D, 5>(sp, BH, stream); break;
      case 6: rc = launch_select_regs<D, 6>(sp, BH, stream); break;
      case 7: rc = launch_select_regs<D, 7>(sp, BH, stream); break;
      case 8: rc = launch_select_regs<D, 8>(sp, BH, stream); break;
      default: break;
    }
    if (ncb > 8) {
      const int nb_pad = (nb + 31) / 32 * 32;
      const size_t budget = 200 * 1024;
      int R = 16;
      while (R > 1 && select_generic_smem<D>(R, nb_pad) > budget) --R;
      const size_t smem = select_generic_smem<D>(R, nb_pad);
      if (smem > budget) return BSA_ERR_UNSUPPORTED;
      static DeviceFlags done;
      if (!allow_smem(bsa::asa_select_generic_kernel<D>, 220 * 1024, done)) return BSA_ERR_CUDA;
      sp.rows_per_cta = R;
      sp.nb_pad = nb_pad;
      sp.groups = static_cast<int>(ceil_div(nb, R));
      const dim3 grid(static_cast<unsigned>((long long)sp.groups * BH));
      bsa::asa_select_generic_kernel<D><<<grid, 256, smem, stream>>>(sp);
      rc = check_launch() ? BSA_ERR_CUDA : BSA_OK;
    }
    return rc;
  }
}

// ---- backward launches ---------------------------------------------------------
template <int D, int BLK>
int launch_bwd(const void* q, const void* k, const void* v, const void* dout, int B, int H,
               int N, const int32_t* row_ptr, const int32_t* col_idx, const float* lse,
               const float* delta, float scale, void* dq, void* dk, void* dv,
               cudaStream_t stream) {
  using C = bsa::BwdCfg<D, BLK>;
  const int nb = (N + BLK - 1) / BLK;
  const int nbw = (nb + 31) / 32;
  if (nb > bsa::kBwdMaxNb || C::G * nbw * 4 > C::BM_BYTES) return BSA_ERR_UNSUPPORTED;
  const int BH = B * H;
  // resident tiles: 128-row boxes; gathered blocks: blk-row boxes
  CUtensorMap q128, do128, k128, v128, qb, dob, kb, vb;
  if (!make_map(&q128, q, BH, N, D, 128) || !make_map(&do128, dout, BH, N, D, 128) ||
      !make_map(&k128, k, BH, N, D, 128) || !make_map(&v128, v, BH, N, D, 128) ||
      !make_map(&qb, q, BH, N, D, BLK) || !make_map(&dob, dout, BH, N, D, BLK) ||
      !make_map(&kb, k, BH, N, D, BLK) || !make_map(&vb, v, BH, N, D, BLK))
    return BSA_ERR_CUDA;
  static DeviceFlags dq_set, dkdv_set;
  if (!allow_smem(bsa::bsa_bwd_dq_kernel<D, BLK>, C::SMEM, dq_set) ||
      !allow_smem(bsa::bsa_bwd_dkdv_kernel<D, BLK>, C::SMEM, dkdv_set))
    return BSA_ERR_CUDA;
  bsa::BwdParams p;
  p.B = B;
  p.H = H;
  p.N = N;
  p.nb = nb;
  p.nbw = nbw;
  p.ntile = ceil_div(N, 128);
  p.row_ptr = row_ptr;
  p.col_idx = col_idx;
  p.lse = lse;
  p.delta = delta;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.wait_ns = kWaitNs;
  const int items = BH * p.ntile;   // one 128-row tile per CTA, either side
  bsa::bsa_bwd_dq_kernel<D, BLK><<<items, bsa::kBwdThreads, C::SMEM, stream>>>(q128, do128, kb,
                                                                             vb, p);
  if (check_launch()) return BSA_ERR_CUDA;
  bsa::bsa_bwd_dkdv_kernel<D, BLK><<<items, bsa::kBwdThreads, C::SMEM, stream>>>(k128, v128, qb,
                                                                               dob, p);
  return check_launch();
}

template <int D>
int launch_bwd_blk(int blk, const void* q, const void* k, const void* v, const void* dout, int B,
                   int H, int N, const int32_t* rp, const int32_t* ci, const float* lse,
                   const float* delta, float scale, void* dq, void* dk, void* dv,
                   cudaStream_t s) {
  switch (blk) {
    case 16: return launch_bwd<D, 16>(q, k, v, dout, B, H, N, rp, ci, lse, delta, scale, dq, dk, dv, s);
    case 32: return launch_bwd<D, 32>(q, k, v, dout, B, H, N, rp, ci, lse, delta, scale, dq, dk, dv, s);
    case 64: return launch_bwd<D, 64>(q, k, v, dout, B, H, N, rp, ci, lse, delta, scale, dq, dk, dv, s);
    case 128: return launch_bwd<D, 128>(q, k, v, dout, B, H, N, rp, ci, lse, delta, scale, dq, dk, dv, s);
  }
  return BSA_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

int bsa_version(void) { return 100; }

const char* bsa_status_string(int status) {
  switch (status) {
    case BSA_OK: return "ok";
    case BSA_ERR_INVALID_ARG: return "invalid argument";
    case BSA_ERR_UNSUPPORTED: return "unsupported shape, block size, head dim or alignment";
    case BSA_ERR_CAPACITY: return "col_idx capacity too small for the mask";
    case BSA_ERR_CUDA: return "CUDA runtime or launch error";
    case BSA_ERR_TIMEOUT: return "a device-side wait gave up";
    case BSA_ERR_CSR: return "CSR block index outside [0, nb)";
    case BSA_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
  }
  return "unknown status";
}

// ---- Sparse-vDiT offline search quantities -----------------------------------
size_t attention_head_mse_workspace_size(int B, int H, int N, int d) {
  if (B <= 0 || H <= 0 || N <= 0 || (d != 64 && d != 128)) return 0;
  const size_t chunks = (N + bsa::kMseTokens - 1) / bsa::kMseTokens;
  return (((size_t)B * H * chunks * sizeof(double)) + 255) & ~static_cast<size_t>(255);
}

int attention_head_mse(const void* o_ref, const void* o, int B, int H, int N, int d, double* mse,
                       void* workspace, size_t ws_bytes, bsa_stream_t stream) {
  if (!o_ref || !o || !mse) return BSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || N <= 0) return BSA_ERR_INVALID_ARG;
  if ((long long)B * H > 65535) return BSA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return BSA_ERR_UNSUPPORTED;
  if (!aligned(o_ref, 16) || !aligned(o, 16) || !aligned(mse, 8)) return BSA_ERR_UNSUPPORTED;
  const size_t need = attention_head_mse_workspace_size(B, H, N, d);
  if (!workspace || ws_bytes < need || !aligned(workspace, 256)) return BSA_ERR_WORKSPACE;
  const int chunks = (N + bsa::kMseTokens - 1) / bsa::kMseTokens;
  cudaStream_t s = as_cuda(stream);
  double* partial = static_cast<double*>(workspace);
  bsa::head_mse_partial_kernel<<<dim3(chunks, B * H), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(o_ref), static_cast<const __nv_bfloat16*>(o), N, d, chunks,
      partial);
  if (check_launch()) return BSA_ERR_CUDA;
  bsa::head_mse_final_kernel<<<ceil_div(H, 128), 128, 0, s>>>(partial, B, H, N, d, chunks, mse);
  return check_launch();
}

size_t csr_head_sparsity_workspace_size(int H) {
  if (H <= 0) return 0;
  return ((size_t)H * sizeof(unsigned long long) + 255) & ~static_cast<size_t>(255);
}

int csr_head_sparsity(const int32_t* row_ptr, const int32_t* col_idx, int B, int H, int N, int blk,
                      double* sparsity, void* workspace, size_t ws_bytes, bsa_stream_t stream) {
  if (!row_ptr || !sparsity) return BSA_ERR_INVALID_ARG;
  int rc = common_shape_checks(B, H, N, blk);
  if (rc != BSA_OK) return rc;
  if (!aligned(sparsity, 8)) return BSA_ERR_UNSUPPORTED;
  if (!workspace || ws_bytes < csr_head_sparsity_workspace_size(H) || !aligned(workspace, 256))
    return BSA_ERR_WORKSPACE;
  const int nb = (N + blk - 1) / blk;
  const long long rows = (long long)B * H * nb;
  cudaStream_t s = as_cuda(stream);
  auto* kept = static_cast<unsigned long long*>(workspace);
  if (cudaMemsetAsync(kept, 0, (size_t)H * sizeof(unsigned long long), s) != cudaSuccess)
    return BSA_ERR_CUDA;
  if (col_idx != nullptr) {
    bsa::csr_pairs_kernel<<<ceil_div(rows, 8), 256, 0, s>>>(row_ptr, col_idx, H, N, blk, nb, rows,
                                                            kept);
    if (check_launch()) return BSA_ERR_CUDA;
  }
  bsa::csr_sparsity_final_kernel<<<ceil_div(H, 128), 128, 0, s>>>(kept, B, H, N, sparsity);
  return check_launch();
}

int pattern_search_select(const double* mse, const double* sparsity, const int32_t* candidates,
                          int P, int H, double lambda, double eps, double* loss, int32_t* choice) {
  if (!mse || !sparsity || !candidates || !choice || P <= 0 || H <= 0) return BSA_ERR_INVALID_ARG;
  if (std::isnan(lambda) || std::isnan(eps)) return BSA_ERR_INVALID_ARG;
  for (int h = 0; h < H; ++h) {
    bool all_above = true;
    int best = 0;
    double best_l = 0.0;
    for (int i = 0; i < P; ++i) {
      const double l = mse[(size_t)i * H + h] + lambda * (1.0 - sparsity[(size_t)i * H + h]);
      if (loss) loss[(size_t)i * H + h] = l;
      if (!(l > eps)) all_above = false;
      if (i == 0 || l < best_l) {
        best = i;
        best_l = l;
      }
    }
    choice[h] = all_above ? BSA_PATTERN_FULL : candidates[best];
  }
  return BSA_OK;
}

int bsa_validate_csr_host(const int32_t* row_ptr_host, const int32_t* col_idx_host, int64_t rows,
                          int nb, int64_t col_len, int64_t* bad_row_host) {
  if (!row_ptr_host || rows < 0 || nb <= 0 || col_len < 0 || (!col_idx_host && col_len > 0))
    return BSA_ERR_INVALID_ARG;
  auto fail = [&](int64_t r) {
    if (bad_row_host) *bad_row_host = r;
    return BSA_ERR_CSR;
  };
  if (row_ptr_host[0] != 0) return fail(0);
  for (int64_t r = 0; r < rows; ++r) {
    const int64_t e0 = row_ptr_host[r], e1 = row_ptr_host[r + 1];
    if (e1 < e0 || e1 > col_len) return fail(r);
    for (int64_t e = e0; e < e1; ++e) {
      const int32_t c = col_idx_host[e];
      if (c < 0 || c >= nb) return fail(r);
      if (e > e0 && col_idx_host[e - 1] >= c) return fail(r);
    }
  }
  if (bad_row_host) *bad_row_host = -1;
  return BSA_OK;
}

int bsa_check_device_status(bsa_stream_t stream) {
  if (cudaStreamSynchronize(as_cuda(stream)) != cudaSuccess) return BSA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, bsa::g_status, sizeof(int)) != cudaSuccess) return BSA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(bsa::g_status, &zero, sizeof(int)) != cudaSuccess) return BSA_ERR_CUDA;
  }
  return v;
}

size_t asa_build_mask_workspace_size(int B, int H, int N, int d, int blk) {
  if (common_shape_checks(B, H, N, blk) != BSA_OK || (d != 64 && d != 128)) return 0;
  return asa_layout(B, H, N, d, blk).total;
}

int64_t asa_build_mask_max_nnz(int B, int H, int N, int blk, int mode, int topk,
                               float max_keep_ratio, int keep_diag, int n_sink_blocks) {
  if (common_shape_checks(B, H, N, blk) != BSA_OK) return -1;
  const long long nb = (N + blk - 1) / blk;
  long long per = select_cap(static_cast<int>(nb), max_keep_ratio);
  if (mode == BSA_MODE_TOPK) per = per < topk ? per : topk;
  if (per < 0) per = 0;
  per += (keep_diag ? 1 : 0) + (n_sink_blocks > 0 ? n_sink_blocks : 0);
  if (per > nb) per = nb;
  return (int64_t)B * H * nb * per;
}

// The argument checks shared by asa_build_mask and asa_build_mask_noalloc
// (everything but the workspace).
static int asa_mask_arg_checks(const void* q, const void* k, int B, int H, int N, int d, int blk,
                               int mode, int topk, float mass_tau, float max_keep_ratio,
                               int n_sink_blocks, float softmax_scale, const int32_t* row_ptr,
                               const int32_t* col_idx, int64_t col_capacity) {
  if (!q || !k || !row_ptr || (!col_idx && col_capacity > 0) || col_capacity < 0)
    return BSA_ERR_INVALID_ARG;
  int rc = common_shape_checks(B, H, N, blk);
  if (rc != BSA_OK) return rc;
  if (d != 64 && d != 128) return BSA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16)) return BSA_ERR_UNSUPPORTED;
  if (mode != BSA_MODE_TOPK && mode != BSA_MODE_MASS) return BSA_ERR_INVALID_ARG;
  if (mode == BSA_MODE_TOPK && topk < 1) return BSA_ERR_INVALID_ARG;
  if (mode == BSA_MODE_MASS && !(mass_tau > 0.f && mass_tau <= 1.f)) return BSA_ERR_INVALID_ARG;
  if (!(max_keep_ratio <= 1.0f) || std::isnan(softmax_scale)) return BSA_ERR_INVALID_ARG;
  if (n_sink_blocks < 0) return BSA_ERR_INVALID_ARG;
  if ((N + blk - 1) / blk > 65536) return BSA_ERR_UNSUPPORTED;
  return BSA_OK;
}

int asa_build_mask(const void* q, const void* k, int B, int H, int N, int d, int blk, int mode,
                   int topk, float mass_tau, float max_keep_ratio, int keep_diag,
                   int n_sink_blocks, float softmax_scale, int32_t* row_ptr, int32_t* col_idx,
                   int64_t col_capacity, void* workspace, size_t ws_bytes, bsa_stream_t stream) {
  const int rc = asa_mask_arg_checks(q, k, B, H, N, d, blk, mode, topk, mass_tau, max_keep_ratio,
                                     n_sink_blocks, softmax_scale, row_ptr, col_idx, col_capacity);
  if (rc != BSA_OK) return rc;
  const AsaLayout L = asa_layout(B, H, N, d, blk);
  if (!workspace || ws_bytes < L.total || !aligned(workspace, 256)) return BSA_ERR_WORKSPACE;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(d));
  cudaStream_t s = as_cuda(stream);
  if (d == 64)
    return launch_asa<64>(q, k, B, H, N, blk, mode, topk, mass_tau, max_keep_ratio, keep_diag,
                          n_sink_blocks, scale, row_ptr, col_idx, col_capacity, workspace, s);
  return launch_asa<128>(q, k, B, H, N, blk, mode, topk, mass_tau, max_keep_ratio, keep_diag,
                         n_sink_blocks, scale, row_ptr, col_idx, col_capacity, workspace, s);
}

int pattern_mask(const int32_t* head_pattern_host, int B, int H, int N, int blk, int band_w,
                 int frame_tokens, int f_lo, int f_hi, int stripe_blocks, int tile_global_frames,
                 int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                 int64_t* nnz_out_host, bsa_stream_t stream) {
  if (!head_pattern_host || !row_ptr || col_capacity < 0 || (!col_idx && col_capacity > 0))
    return BSA_ERR_INVALID_ARG;
  int rc = common_shape_checks(B, H, N, blk);
  if (rc != BSA_OK) return rc;
  if (H > bsa::kMaxPatternHeads) return BSA_ERR_UNSUPPORTED;
  if (band_w < 0 || frame_tokens <= 0 || f_lo > f_hi || stripe_blocks < 0 ||
      tile_global_frames < 0)
    return BSA_ERR_INVALID_ARG;
  bsa::PatternParams p;
  std::memset(&p, 0, sizeof(p));
  for (int h = 0; h < H; ++h) {
    const int v = head_pattern_host[h];
    if (v < BSA_PATTERN_FULL || v > BSA_PATTERN_TILE3D) return BSA_ERR_INVALID_ARG;
    p.head_pattern[h] = static_cast<int8_t>(v);
  }
  p.B = B;
  p.H = H;
  p.N = N;
  p.blk = blk;
  p.lblk = blk == 16 ? 4 : blk == 32 ? 5 : blk == 64 ? 6 : 7;   // blk checked above
  p.nb = (N + blk - 1) / blk;
  // The kernels compute in 32 bits: band widths above 2^24 tokens and frames
  // above 2^28 tokens are not supported, and two clamps that change no mask
  // keep the rest in range (a stripe of nb blocks covers a whole frame; there
  // are at most N / frame_tokens + 1 frames).
  if ((long long)band_w * blk > (1LL << 24) || frame_tokens > (1 << 28))
    return BSA_ERR_UNSUPPORTED;
  const int frames = N / frame_tokens + 1;
  p.band_w = band_w;
  p.frame_tokens = frame_tokens;
  p.f_lo = f_lo;
  p.f_hi = f_hi;
  p.stripe_blocks = stripe_blocks < p.nb ? stripe_blocks : p.nb;
  p.tile_global_frames = tile_global_frames < frames ? tile_global_frames : frames;
  p.row_ptr = row_ptr;
  p.col_idx = col_idx;
  p.capacity = col_capacity;
  cudaStream_t s = as_cuda(stream);
  const long long rows = (long long)B * H * p.nb;
  bsa::pattern_rowptr_kernel<<<H, bsa::kPatternScanThreads, 0, s>>>(p);
  if (check_launch()) return BSA_ERR_CUDA;
  if (nnz_out_host) {
    int32_t nnz = 0;
    if (cudaMemcpyAsync(&nnz, row_ptr + rows, sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return BSA_ERR_CUDA;
    *nnz_out_host = nnz;
    if (nnz > col_capacity) return BSA_ERR_CAPACITY;
  }
  const dim3 wgrid(static_cast<unsigned>(ceil_div(p.nb, bsa::kPatternWriteWarps * bsa::kPatternRowsPerWarp)),
                   static_cast<unsigned>(H));
  bsa::pattern_write_kernel<<<wgrid, bsa::kPatternWriteWarps * 32, 0, s>>>(p);
  return check_launch();
}

size_t bsa_forward_workspace_size(int B, int H, int N, int d, int blk) {
  if (common_shape_checks(B, H, N, blk) != BSA_OK || (d != 64 && d != 128)) return 0;
  return 256;   // the item counter of the persistent grid
}

int bsa_forward(const void* q, const void* k, const void* v, int B, int H, int N, int d, int blk,
                const int32_t* row_ptr, const int32_t* col_idx, float softmax_scale, void* o,
                float* lse, void* workspace, size_t ws_bytes, bsa_stream_t stream) {
  return bsa_forward_residual(q, k, v, B, H, N, d, blk, row_ptr, col_idx, softmax_scale, o, lse,
                              nullptr, workspace, ws_bytes, stream);
}

int bsa_forward_residual(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                         int blk, const int32_t* row_ptr, const int32_t* col_idx,
                         float softmax_scale, void* o, float* lse, void* o_residual,
                         void* workspace, size_t ws_bytes, bsa_stream_t stream) {
  if (!q || !k || !v || !o || !row_ptr || !col_idx) return BSA_ERR_INVALID_ARG;
  if (o_residual != nullptr && !aligned(o_residual, 16)) return BSA_ERR_UNSUPPORTED;
  if (workspace != nullptr && (ws_bytes < 4 || !aligned(workspace, 4))) return BSA_ERR_WORKSPACE;
  int rc = common_shape_checks(B, H, N, blk);
  if (rc != BSA_OK) return rc;
  if (d != 64 && d != 128) return BSA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16))
    return BSA_ERR_UNSUPPORTED;
  if (std::isnan(softmax_scale)) return BSA_ERR_INVALID_ARG;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(d));
  cudaStream_t s = as_cuda(stream);
  int* counter = static_cast<int*>(workspace);
  if (counter != nullptr && cudaMemsetAsync(counter, 0, sizeof(int), s) != cudaSuccess)
    return BSA_ERR_CUDA;
  if (d == 64)
    return launch_fwd_blk<64>(blk, q, k, v, B, H, N, row_ptr, col_idx, scale, o, lse, o_residual,
                              counter, s);
  return launch_fwd_blk<128>(blk, q, k, v, B, H, N, row_ptr, col_idx, scale, o, lse, o_residual,
                             counter, s);
}

size_t bsa_backward_workspace_size(int B, int H, int N, int d, int blk) {
  if (common_shape_checks(B, H, N, blk) != BSA_OK || (d != 64 && d != 128)) return 0;
  return ((size_t)B * H * N * sizeof(float) + 255) & ~static_cast<size_t>(255);
}

int bsa_backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, int B, int H, int N, int d, int blk, const int32_t* row_ptr,
                 const int32_t* col_idx, float softmax_scale, void* dq, void* dk, void* dv,
                 void* workspace, size_t ws_bytes, bsa_stream_t stream) {
  return bsa_backward_residual(q, k, v, o, nullptr, dout, lse, B, H, N, d, blk, row_ptr, col_idx,
                               softmax_scale, dq, dk, dv, workspace, ws_bytes, stream);
}

int bsa_backward_residual(const void* q, const void* k, const void* v, const void* o,
                          const void* o_residual, const void* dout, const float* lse, int B,
                          int H, int N, int d, int blk, const int32_t* row_ptr,
                          const int32_t* col_idx, float softmax_scale, void* dq, void* dk,
                          void* dv, void* workspace, size_t ws_bytes, bsa_stream_t stream) {
  if (!q || !k || !v || !o || !dout || !lse || !row_ptr || !col_idx || !dq || !dk || !dv)
    return BSA_ERR_INVALID_ARG;
  if (o_residual != nullptr && !aligned(o_residual, 16)) return BSA_ERR_UNSUPPORTED;
  int rc = common_shape_checks(B, H, N, blk);
  if (rc != BSA_OK) return rc;
  if (d != 64 && d != 128) return BSA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
      !aligned(lse, 4))
    return BSA_ERR_UNSUPPORTED;
  if ((N + blk - 1) / blk > bsa::kBwdMaxNb) return BSA_ERR_UNSUPPORTED;
  // the D pass runs d/8 threads per token in a 1D grid of 256-thread blocks
  if ((long long)B * H * N * (d / 8) > 0x7fffffffLL) return BSA_ERR_UNSUPPORTED;
  if (std::isnan(softmax_scale)) return BSA_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < bsa_backward_workspace_size(B, H, N, d, blk) ||
      !aligned(workspace, 256))
    return BSA_ERR_WORKSPACE;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(d));
  cudaStream_t s = as_cuda(stream);
  float* delta = static_cast<float*>(workspace);
  const long long tokens = (long long)B * H * N;
  const auto* ob = static_cast<const __nv_bfloat16*>(o);
  const auto* rb = static_cast<const __nv_bfloat16*>(o_residual);
  const auto* db = static_cast<const __nv_bfloat16*>(dout);
  if (d == 64) {
    bsa::bwd_delta_kernel<64><<<ceil_div(tokens * 8, 256), 256, 0, s>>>(ob, rb, db, tokens, delta);
    if (check_launch()) return BSA_ERR_CUDA;
    return launch_bwd_blk<64>(blk, q, k, v, dout, B, H, N, row_ptr, col_idx, lse, delta, scale,
                              dq, dk, dv, s);
  }
  bsa::bwd_delta_kernel<128><<<ceil_div(tokens * 16, 256), 256, 0, s>>>(ob, rb, db, tokens, delta);
  if (check_launch()) return BSA_ERR_CUDA;
  return launch_bwd_blk<128>(blk, q, k, v, dout, B, H, N, row_ptr, col_idx, lse, delta, scale,
                             dq, dk, dv, s);
}

}  // extern "C"

namespace {
__global__ void exp2_poly_kernel(const float* x, float* y, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = bsa::exp2_poly(x[i]);
}
}  // namespace

namespace {
// One thread waits, with the bounded wait every kernel of this library uses,
// on an mbarrier phase that completes only if the thread arrives first.
// Without the arrive the wait gives up after limit_ns, the kernel records
// BSA_ERR_TIMEOUT and returns.
__global__ void wait_timeout_kernel(unsigned long long limit_ns, int arrive_first,
                                    unsigned long long* waited_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  bsa::mbar_init(&bar, 1);
  bsa::fence_mbar_init();
  if (arrive_first) bsa::mbar_arrive(&bar);
  const uint64_t t0 = bsa::global_ns();
  const bool ok = bsa::mbar_wait(&bar, 0, limit_ns);
  if (waited_ns) *waited_ns = bsa::global_ns() - t0;
  if (!ok) bsa::record_error(BSA_ERR_TIMEOUT);
}
}  // namespace

extern "C" int bsa_debug_wait_timeout(unsigned long long limit_ns, int arrive_first,
                                      unsigned long long* waited_ns, bsa_stream_t stream) {
  if (limit_ns > 10000000000ull) return BSA_ERR_INVALID_ARG;   // at most 10 s
  if (waited_ns && !aligned(waited_ns, 8)) return BSA_ERR_UNSUPPORTED;
  wait_timeout_kernel<<<1, 32, 0, as_cuda(stream)>>>(limit_ns, arrive_first, waited_ns);
  return check_launch();
}

extern "C" int bsa_debug_exp2_poly(const float* x, float* y, int n, bsa_stream_t stream) {
  if (!x || !y || n < 0) return BSA_ERR_INVALID_ARG;
  if (n == 0) return BSA_OK;
  exp2_poly_kernel<<<ceil_div(n, 256), 256, 0, as_cuda(stream)>>>(x, y, n);
  return check_launch();
}

// ============================================================================
// asa_build_mask_noalloc: the ASA mask with its scratch in a fixed-size device
// array that belongs to the library, for callers that cannot allocate device
// memory (see include/bsa.h).  The array is file-scope and static; host code
// must not hand its name to a kernel (on the host that name is only a stand-in
// for the device object), so the device address is looked up with
// cudaGetSymbolAddress, once per device, on the first call made while that
// device is current, and that address is what the kernels receive.
// ============================================================================
static __device__ __align__(256) unsigned char bsa_asa_noalloc_scratch[BSA_ASA_NOALLOC_MAX_WORKSPACE];

namespace {

constexpr int kNoallocMaxDevices = 64;
void* g_noalloc_addr[kNoallocMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of this device's copy of the scratch array (nullptr on error).
void* noalloc_scratch_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, bsa_asa_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_addr[dev] = p;
  }
  return g_noalloc_addr[dev];
}

}  // namespace

extern "C" int asa_build_mask_noalloc(const void* q, const void* k, int B, int H, int N, int d,
                                      int blk, int mode, int topk, float mass_tau,
                                      float max_keep_ratio, int keep_diag, int n_sink_blocks,
                                      float softmax_scale, int32_t* row_ptr, int32_t* col_idx,
                                      int64_t col_capacity, bsa_stream_t stream) {
  // the same argument checks as asa_build_mask, minus the caller's workspace
  const int rc = asa_mask_arg_checks(q, k, B, H, N, d, blk, mode, topk, mass_tau, max_keep_ratio,
                                     n_sink_blocks, softmax_scale, row_ptr, col_idx, col_capacity);
  if (rc != BSA_OK) return rc;
  // the scratch this shape needs must fit the fixed array
  if (asa_layout(B, H, N, d, blk).total > static_cast<size_t>(BSA_ASA_NOALLOC_MAX_WORKSPACE))
    return BSA_ERR_WORKSPACE;
  void* ws = noalloc_scratch_for_current_device();
  if (ws == nullptr) return BSA_ERR_CUDA;
  // The scratch keeps the previous call's contents.  What must start at zero
  // (the selection kernel's ticket and look-back flags) is zeroed by this
  // call's pooling kernel; everything else (pooled rows, bitmap words) is
  // written by this call before anything reads it.
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(d));
  cudaStream_t s = as_cuda(stream);
  if (d == 64)
    return launch_asa<64>(q, k, B, H, N, blk, mode, topk, mass_tau, max_keep_ratio, keep_diag,
                          n_sink_blocks, scale, row_ptr, col_idx, col_capacity, ws, s);
  return launch_asa<128>(q, k, B, H, N, blk, mode, topk, mass_tau, max_keep_ratio, keep_diag,
                         n_sink_blocks, scale, row_ptr, col_idx, col_capacity, ws, s);
}
