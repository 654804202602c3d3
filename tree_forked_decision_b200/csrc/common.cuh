// common.cuh -- small device helpers shared by the flide kernels.
#pragma once

#include <atomic>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "flide.h"

namespace flide {

// Past K/V rows read in place from a block-paged history pool: history row i
// of request r is pool row block_table[req_slot[r] * max_blocks + i /
// block_rows] * block_rows + i % block_rows.
struct PagedPast {
  const int32_t *block_table, *req_slot;
  int max_blocks, block_rows, n_blocks, n_slots;
};

// Records the first device-detected error; later ones are dropped.
__device__ __forceinline__ void set_status(int32_t *status, int32_t code) {
  atomicCAS(status, 0, code);
}

__device__ __forceinline__ bool failed(const int32_t *status) {
  return *(volatile const int32_t *)status != 0;
}

#ifdef FLIDE_DEBUG_BOUNDS
constexpr bool kBoundsChecks = true;
#else
constexpr bool kBoundsChecks = false;
#endif

// Bounds check of an index taken from device data, compiled in only by the
// debug build (FLIDE_DEBUG_BOUNDS).  Returns whether 0 <= i < n; on a failure
// it records the site and the value in the index's check slots (first failure
// wins) and FLIDE_ERR_BOUNDS in the status word, so the caller can skip the
// access.  The release build folds every call to `true`.
__device__ __forceinline__ bool in_bounds(int32_t *status, int32_t *counts, long long i,
                                          long long n, int site) {
  if (!kBoundsChecks || (i >= 0 && i < n)) return true;
  if (atomicCAS(&counts[FLIDE_CNT_CHECK_SITE], 0, site) == 0)
    counts[FLIDE_CNT_CHECK_VALUE] = (int32_t)i;
  set_status(status, FLIDE_ERR_BOUNDS);
  return false;
}
// i if it passes the check, else 0 (for reads that must still happen)
__device__ __forceinline__ long long checked(int32_t *status, int32_t *counts, long long i,
                                             long long n, int site) {
  return in_bounds(status, counts, i, n, site) ? i : 0;
}

template <typename T>
__device__ __forceinline__ float load_f(const T *p);
template <>
__device__ __forceinline__ float load_f<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float load_f<__nv_bfloat16>(const __nv_bfloat16 *p) {
  return __bfloat162float(*p);
}

template <typename T>
__device__ __forceinline__ void store_f(T *p, float x);
template <>
__device__ __forceinline__ void store_f<float>(float *p, float x) { *p = x; }
template <>
__device__ __forceinline__ void store_f<__nv_bfloat16>(__nv_bfloat16 *p, float x) {
  *p = __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

__device__ __forceinline__ int warp_incl_scan(int x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// Exclusive scan of one value per thread across a block of blockDim.x
// (multiple of 32, <= 1024) threads; returns the exclusive prefix and writes
// the block total to *total.  `scratch` holds >= 33 ints of shared memory.
__device__ __forceinline__ int block_excl_scan(int x, int *scratch, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  int incl = warp_incl_scan(x);
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nwarps ? scratch[lane] : 0;
    int wi = warp_incl_scan(w);
    if (lane < nwarps) scratch[lane] = wi - w;
    if (lane == 31) scratch[32] = wi;
  }
  __syncthreads();
  int res = incl - x + scratch[warp];
  *total = scratch[32];
  __syncthreads();
  return res;
}

}  // namespace flide

#define FLIDE_LAUNCH_CHECK()                                   \
  do {                                                         \
    cudaError_t e_ = cudaGetLastError();                       \
    if (e_ != cudaSuccess) return FLIDE_ERR_CUDA;              \
  } while (0)
