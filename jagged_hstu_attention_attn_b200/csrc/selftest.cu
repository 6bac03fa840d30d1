// selftest.cu -- device-side check of the library's bounded waits.
//
// Every wait inside the attention kernels is an mbarrier wait with a time
// limit (mbar_wait_limit in common.cuh): when the phase it waits for never
// completes, the wait records HSTU_ERR_TIMEOUT in the caller's status word,
// raises the CTA's abort flag and returns, so the kernel can wind down and
// the context stays usable.  This kernel exercises exactly that path in the
// one way that is safe to provoke: it waits, with a short limit, on an
// mbarrier that nothing will ever arrive on.  No copy or tensor-core work is
// in flight, so returning after the limit leaves nothing behind.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace hstu {
namespace {

__global__ void wait_timeout_kernel(uint64_t limit_ns, int* status, int* result) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected; none will come
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const bool ok = mbar_wait_limit(&bar, 0, &abort_flag, status, limit_ns);
  const bool all_ok = __all_sync(0xffffffffu, ok);
  if (threadIdx.x == 0) *result = all_ok ? 1 : 0;
}

}  // namespace

cudaError_t wait_timeout_launch(int64_t limit_ns, int* status, int* result, cudaStream_t stream) {
  count_launch();
  wait_timeout_kernel<<<1, 32, 0, stream>>>((uint64_t)limit_ns, status, result);
  return cudaGetLastError();
}

}  // namespace hstu
