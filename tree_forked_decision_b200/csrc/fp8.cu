// fp8.cu -- per-tensor e4m3 quantisation for the fp8 attention path.
//
// The pages run Flide in FP8 where the hardware has it (techfi24.com, "Exact
// State Forking"; "Performances": a 35B model quantised to FP8) without naming
// the encoding.  Used here: the e4m3 format (bias 7, 3 mantissa bits, largest
// finite value 448) with one scale per tensor, its absolute maximum mapped to
// 448.  Two HBM-bound passes:
//   flide_amax            amax = max |x| over one or more tensors (atomic max
//                         on the float's bit pattern, which orders like the
//                         value for non-negative floats; NaN entries are
//                         ignored)
//   flide_quantize_e4m3   inv = 448 / amax, code = e4m3_rn_sat(x * inv) (both
//                         fp32 operations rounded to nearest), and
//                         descale = amax / 448; amax 0 gives inv = descale = 1
// Each thread handles 8 elements per step: one 16-byte load (bf16) or two
// (fp32), one 8-byte store of codes.
#include "common.cuh"
#include "sm100.cuh"

namespace flide {
namespace {

using namespace sm100;

constexpr int kThreads = 256;
constexpr float kE4m3Max = 448.0f;

__device__ __forceinline__ void load8(const float *x, int64_t v, float (&f)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4 *>(x) + 2 * v);
  const float4 b = __ldg(reinterpret_cast<const float4 *>(x) + 2 * v + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16 *x, int64_t v, float (&f)[8]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4 *>(x) + v);
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ float load1(const float *x, int64_t i) { return x[i]; }
__device__ __forceinline__ float load1(const __nv_bfloat16 *x, int64_t i) {
  return __bfloat162float(x[i]);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) amax_kernel(const T *__restrict__ x, int64_t n,
                                                        float *amax) {
  __shared__ uint32_t red[kThreads / 32];
  const int64_t nv = n / 8;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  float m = 0.f;
#pragma unroll 4
  for (int64_t v = (int64_t)blockIdx.x * kThreads + threadIdx.x; v < nv; v += stride) {
    float f[8];
    load8(x, v, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
  }
  if (blockIdx.x == 0 && threadIdx.x < n - 8 * nv) m = fmaxf(m, fabsf(load1(x, 8 * nv + threadIdx.x)));
  uint32_t b = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = b;
  __syncthreads();
  if (threadIdx.x < 32) {
    b = threadIdx.x < kThreads / 32 ? red[threadIdx.x] : 0u;
    b = __reduce_max_sync(0xffffffffu, b);
    if (threadIdx.x == 0) atomicMax(reinterpret_cast<unsigned int *>(amax), b);
  }
}

__device__ __forceinline__ float inv_scale(float a) { return a > 0.f ? kE4m3Max / a : 1.f; }

template <typename T>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const T *__restrict__ x, int64_t n,
                                                            const float *__restrict__ amax,
                                                            uint8_t *__restrict__ out,
                                                            float *descale) {
  const float a = *amax;
  const float inv = inv_scale(a);
  if (descale && blockIdx.x == 0 && threadIdx.x == 0) *descale = a > 0.f ? a / kE4m3Max : 1.f;
  const int64_t nv = n / 8;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
#pragma unroll 4
  for (int64_t v = (int64_t)blockIdx.x * kThreads + threadIdx.x; v < nv; v += stride) {
    float f[8];
    load8(x, v, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = __fmul_rn(f[i], inv);
    uint2 w;
    w.x = pack_e4m3x4(f[0], f[1], f[2], f[3]);
    w.y = pack_e4m3x4(f[4], f[5], f[6], f[7]);
    reinterpret_cast<uint2 *>(out)[v] = w;
  }
  if (blockIdx.x == 0 && threadIdx.x < n - 8 * nv) {
    const int64_t i = 8 * nv + threadIdx.x;
    out[i] = (uint8_t)(pack_e4m3x4(__fmul_rn(load1(x, i), inv), 0.f, 0.f, 0.f) & 0xffu);
  }
}

int grid_for(int64_t n) {
  const int64_t nv = (n / 8 + kThreads - 1) / kThreads;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t cap = (int64_t)sms * 8;  // 8 resident 256-thread blocks per SM
  return (int)(nv < 1 ? 1 : (nv < cap ? nv : cap));
}

}  // namespace
}  // namespace flide

using namespace flide;

extern "C" {

int flide_amax(const void *x, int64_t n, int32_t dtype, float *amax, int32_t accumulate,
               flide_stream stream) {
  if (!amax || n < 0 || (n > 0 && !x)) return FLIDE_ERR_SHAPE;
  if (dtype != FLIDE_F32 && dtype != FLIDE_BF16) return FLIDE_ERR_SHAPE;
  if ((uintptr_t)x % 16 != 0 || (uintptr_t)amax % 4 != 0) return FLIDE_ERR_SHAPE;
  cudaStream_t s = (cudaStream_t)stream;
  if (!accumulate && cudaMemsetAsync(amax, 0, sizeof(float), s) != cudaSuccess) return FLIDE_ERR_CUDA;
  if (n == 0) return FLIDE_OK;
  const int grid = grid_for(n);
  if (dtype == FLIDE_F32)
    amax_kernel<float><<<grid, kThreads, 0, s>>>((const float *)x, n, amax);
  else
    amax_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>((const __nv_bfloat16 *)x, n, amax);
  FLIDE_LAUNCH_CHECK();
  return FLIDE_OK;
}

int flide_quantize_e4m3(const void *x, int64_t n, int32_t dtype, const float *amax,
                        uint8_t *out, float *descale, flide_stream stream) {
  if (!amax || n < 0 || (n > 0 && (!x || !out))) return FLIDE_ERR_SHAPE;
  if (dtype != FLIDE_F32 && dtype != FLIDE_BF16) return FLIDE_ERR_SHAPE;
  if ((uintptr_t)x % 16 != 0 || (uintptr_t)out % 8 != 0) return FLIDE_ERR_SHAPE;
  cudaStream_t s = (cudaStream_t)stream;
  const int grid = grid_for(n);
  if (dtype == FLIDE_F32)
    quantize_kernel<float><<<grid, kThreads, 0, s>>>((const float *)x, n, amax, out, descale);
  else
    quantize_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>((const __nv_bfloat16 *)x, n, amax,
                                                             out, descale);
  FLIDE_LAUNCH_CHECK();
  return FLIDE_OK;
}

}  // extern "C"
