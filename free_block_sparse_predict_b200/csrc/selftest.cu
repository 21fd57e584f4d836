// Failure-detection self-test: proves on a live GPU that a device-side wait
// which can never be satisfied ends by itself and reports through the
// workspace status word, leaving the context usable.  It runs the same
// time-bounded mbarrier wait the attention kernel uses, on a barrier that no
// thread ever arrives on.  No fault, trap or hang is involved.
#include <cstdint>

#include "sm100_ptx.cuh"
#include "sparge_internal.h"

namespace sparge {
namespace {

__global__ void unsatisfiable_wait_kernel(int32_t* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing arrives on `bar`: the bounded wait must give up on its own
    if (!mbar_wait(&bar, 0, &abort_flag, status)) atomicExch(status, int32_t(SPARGE_ETIMEOUT));
  }
}

}  // namespace
}  // namespace sparge

using namespace sparge;

extern "C" sparge_status_t sparge_selftest_wait_timeout(void* ws, cudaStream_t stream) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SPARGE_EINVAL;
  DeviceScope dev;
  const sparge_status_t st = dev.enter(ws);
  if (st != SPARGE_OK) return st;
  unsatisfiable_wait_kernel<<<1, 32, 0, stream>>>(static_cast<int32_t*>(ws));
  return cudaGetLastError() == cudaSuccess ? SPARGE_OK : SPARGE_ECUDA;
}
