// common.cuh -- status word, warp helpers and the CSR scan shared by the mask
// builders.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include "../../include/bsa.h"

namespace bsa {

// First error recorded by any kernel of this library on this device since the
// last bsa_check_device_status().  0 = none.
__device__ int g_status;

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_status, 0, code); }

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Butterfly sum: every lane ends with the same value, the order is fixed.
__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

__device__ __forceinline__ float warp_incl_scan_f(float v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    float t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// In-place inclusive scan of row_ptr[1..rows] (the per-row counts), one CTA of
// 1024 threads: row_ptr[r+1] becomes the end of row r; row_ptr[0] = 0.
// A total past INT32_MAX is recorded as BSA_ERR_CAPACITY.
__global__ void __launch_bounds__(1024) csr_scan_kernel(int32_t* row_ptr, int rows) {
  __shared__ long long warp_tot[32];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int per = (rows + 1023) / 1024;
  const int lo = min(rows, t * per), hi = min(rows, lo + per);
  long long s = 0;
  for (int r = lo; r < hi; ++r) s += row_ptr[r + 1];
  // block exclusive scan of the per-thread sums
  long long incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    long long v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    long long w = warp_tot[lane];
    long long wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      long long v = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += v;
    }
    warp_tot[lane] = wi - w;
  }
  __syncthreads();
  long long run = warp_tot[warp] + incl - s;
  for (int r = lo; r < hi; ++r) {
    run += row_ptr[r + 1];
    if (run > 0x7fffffffLL) {
      record_error(BSA_ERR_CAPACITY);
      run = 0x7fffffffLL;
    }
    row_ptr[r + 1] = static_cast<int32_t>(run);
  }
  if (t == 0) row_ptr[0] = 0;
}

}  // namespace bsa
