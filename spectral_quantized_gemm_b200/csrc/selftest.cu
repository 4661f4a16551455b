// Self-test of the bounded-wait path that every tensor-core kernel relies on: a CTA waits
// on an mbarrier that nothing arrives at, with a short cycle limit; the wait gives up,
// the kernel raises METIS_DEV_TIMEOUT in the context's status word and returns normally,
// leaving the context usable.  Nothing faults, traps or hangs.
#include <cuda_runtime.h>

#include "device_common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace metis {
namespace {

__global__ void wait_timeout_kernel(long long limit_cycles, uint32_t* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);   // expects one arrival that never comes
    tc::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !tc::mbar_wait(&bar, 0, nullptr, limit_cycles)) raise_status(status, METIS_DEV_TIMEOUT);
}

}  // namespace

metis_status launch_wait_timeout_selftest(metis_ctx* ctx, int64_t limit_cycles) {
  wait_timeout_kernel<<<1, 32, 0, ctx->stream>>>((long long)limit_cycles, ctx->status);
  count_launch();
  return check_cuda(ctx, cudaGetLastError(), "wait self-test launch");
}

}  // namespace metis
