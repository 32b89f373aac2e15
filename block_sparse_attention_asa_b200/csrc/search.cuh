// search.cuh -- the device side of Sparse-vDiT's offline pattern search, sm_100a.
//
// Sparse-vDiT blog, "核心公式 / 离线搜索损失函数" and Algorithm 1: for each head
// and candidate pattern i, L_i = MSE(O_i - O_0) + lambda (1 - S_i), with O_0 the
// output of full attention and S_i the pattern's sparsity.  The two per-head
// reductions run here; the loss and the selection rule over H x P numbers are
// plain host code in bsa_api.cu.
//
// Readings (documented in include/bsa.h): the MSE averages over every element
// the head outputs (B * N * d terms); S is the fraction of (query, key) token
// pairs the mask does not compute, 1 - kept pairs / (B * N * N).
//
// Both reductions are deterministic: fixed-order fp32 sums inside a CTA, fp64
// partials summed in index order, integer pair counts.
#pragma once
#include "common.cuh"
#include <cuda_bf16.h>

namespace bsa {

constexpr int kMseTokens = 64;   // query tokens per CTA of head_mse_partial_kernel

// partial[bh * chunks + c] = sum over tokens [c*64, c*64+64) of head bh and all
// d of (o - o_ref)^2.  256 threads, 16-byte loads.
__global__ void __launch_bounds__(256) head_mse_partial_kernel(const __nv_bfloat16* __restrict__ o_ref,
                                                               const __nv_bfloat16* __restrict__ o,
                                                               int N, int d, int chunks,
                                                               double* __restrict__ partial) {
  __shared__ float wsum[8];
  const long long bh = blockIdx.y;
  const int c = blockIdx.x;
  const int t0 = c * kMseTokens, t1 = min(N, t0 + kMseTokens);
  const long long base = (bh * N + t0) * d;
  const int nvec = (t1 - t0) * d / 8;   // d is a multiple of 8
  const uint4* a = reinterpret_cast<const uint4*>(o_ref + base);
  const uint4* b = reinterpret_cast<const uint4*>(o + base);
  float acc = 0.f;
  for (int e = threadIdx.x; e < nvec; e += 256) {
    const uint4 ra = __ldg(a + e), rb = __ldg(b + e);
    const __nv_bfloat162* ha = reinterpret_cast<const __nv_bfloat162*>(&ra);
    const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&rb);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 fa = __bfloat1622float2(ha[k]), fb = __bfloat1622float2(hb[k]);
      const float dx = fb.x - fa.x, dy = fb.y - fa.y;
      acc = fmaf(dx, dx, acc);
      acc = fmaf(dy, dy, acc);
    }
  }
  acc = warp_sum_f(acc);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < 8; ++w) s += wsum[w];
    partial[bh * chunks + c] = s;
  }
}

// mse[h] = (sum over b and chunks, in index order) / (B * N * d)
__global__ void head_mse_final_kernel(const double* __restrict__ partial, int B, int H, int N, int d,
                                      int chunks, double* __restrict__ mse) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= H) return;
  double s = 0.0;
  for (int b = 0; b < B; ++b) {
    const double* p = partial + ((long long)b * H + h) * chunks;
    for (int c = 0; c < chunks; ++c) s += p[c];
  }
  mse[h] = s / ((double)B * N * d);
}

// kept[h] += n_q(i) * (valid keys of the row's blocks), one warp per row.
__global__ void __launch_bounds__(256) csr_pairs_kernel(const int32_t* __restrict__ row_ptr,
                                                        const int32_t* __restrict__ col_idx, int H,
                                                        int N, int blk, int nb, long long rows,
                                                        unsigned long long* __restrict__ kept) {
  const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= rows || (threadIdx.x & 31) != 0) return;
  const int i = static_cast<int>(r % nb);
  const int h = static_cast<int>((r / nb) % H);
  const int e0 = row_ptr[r], e1 = row_ptr[r + 1];
  if (e1 <= e0) return;
  const long long nq = min(blk, N - i * blk);
  long long keys = (long long)(e1 - e0) * blk;
  const int last_len = N - (nb - 1) * blk;
  if (col_idx[e1 - 1] == nb - 1) keys -= blk - last_len;   // ascending: the last entry
  atomicAdd(&kept[h], static_cast<unsigned long long>(nq * keys));
}

__global__ void csr_sparsity_final_kernel(const unsigned long long* __restrict__ kept, int B, int H,
                                          int N, double* __restrict__ sparsity) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h < H) sparsity[h] = 1.0 - (double)kept[h] / ((double)B * N * (double)N);
}

}  // namespace bsa
