// selftest.cu -- diagnostic entry point: the library's bounded mbarrier wait
// run against a barrier that nothing arrives at, so a test can check that an
// expired wait reports FLIDE_ERR_TIMEOUT through the status word and leaves the
// CUDA context usable (no fault, trap or unbounded spin is involved).
#include "common.cuh"
#include "sm100.cuh"

namespace flide {
namespace {

using namespace sm100;

__global__ void selftest_wait_kernel(int32_t *status, uint64_t timeout_ns, int arrive) {
  __shared__ __align__(8) uint64_t bar_mem;
  __shared__ int abort_flag;
  const uint32_t bar = static_cast<uint32_t>(__cvta_generic_to_shared(&bar_mem));
  mbar_init(bar, 1);
  abort_flag = 0;
  fence_mbar_init();
  if (arrive) mbar_arrive(bar);
  if (!mbar_wait(bar, 0, &abort_flag, timeout_ns)) set_status(status, FLIDE_ERR_TIMEOUT);
}

}  // namespace
}  // namespace flide

extern "C" int flide_selftest_wait_timeout(int32_t *status, int32_t timeout_us, int32_t arrive,
                                           flide_stream stream) {
  using namespace flide;
  if (!status || timeout_us < 1 || timeout_us > 10000000) return FLIDE_ERR_SHAPE;
  selftest_wait_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(status, (uint64_t)timeout_us * 1000ull,
                                                          arrive ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? FLIDE_OK : FLIDE_ERR_CUDA;
}
