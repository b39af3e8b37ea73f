// ckda_selftest.cu -- failure-detection self-test: the library's bounded
// mbarrier wait, run against a barrier that nothing arrives at, gives up,
// records the time-out in the workspace status word and lets the kernel
// return.  The GPU context stays usable; nothing faults, traps or hangs.
#include <cstdint>

#include "ckda_internal.cuh"
#include "ckda_tc.cuh"

namespace ckda {
namespace {
using namespace tc;

constexpr uint32_t kSiteSelftest = 900;  // the status word's detail for this wait

__global__ void bounded_wait_selftest_kernel(DevStatus *st, uint32_t polls) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  // phase 0 never completes: no thread arrives and no copy is tracked by it
  if (threadIdx.x == 0) mbar_wait(&bar, 0, st, kSiteSelftest, polls);
}

}  // namespace
}  // namespace ckda

using namespace ckda;

extern "C" int ckda_selftest_bounded_wait(void *ws, size_t ws_bytes, uint32_t polls, cudaStream_t stream) {
  if (!ws || ws_bytes < sizeof(DevStatus)) return ws ? CKDA_ERR_WORKSPACE : CKDA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return CKDA_ERR_ALIGNMENT;
  DevStatus *st = static_cast<DevStatus *>(ws);
  if (cudaMemsetAsync(st, 0, sizeof(DevStatus), stream) != cudaSuccess) return CKDA_ERR_CUDA;
  bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(st, polls);
  return cudaGetLastError() == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}
