// Self-test of the bounded in-kernel waits: a barrier that nothing completes
// must make the waiting kernel give up, flag DSA_DEV_TIMEOUT and return.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);                 // one arrival expected; none will come
    fence_mbar_init();
    mbar_wait_limit(&bar, 0, status, nullptr, limit_ns);
  }
}

}  // namespace
}  // namespace dsa

extern "C" dsa_status dsa_selftest_wait_timeout(void* ws, size_t ws_bytes, uint32_t limit_us, void* stream) {
  if (!ws || ws_bytes < dsa::kWsHeader) return DSA_ERR_INVALID_ARGUMENT;
  if (limit_us < 1 || limit_us > 2000000) return DSA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), st) != cudaSuccess) return DSA_ERR_CUDA;
  dsa::wait_timeout_kernel<<<1, 32, 0, st>>>(static_cast<uint32_t*>(ws), static_cast<uint64_t>(limit_us) * 1000ull);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  dsa::count_launches(1);
  return DSA_OK;
}
