// Self-test of the bounded mbarrier wait used by every kernel of libgqa_attn: one
// CTA waits on a barrier that no thread or copy ever completes.  The wait must give
// up after its budget, record GQA_ERR_DEVICE_TIMEOUT in the status word and let the
// kernel return normally, so a lost arrival never hangs the GPU.
#include "internal.h"

namespace gqa {
namespace {

__global__ void selftest_wait_kernel(int32_t* status, int64_t budget_ns) {
  __shared__ __align__(8) uint64_t bar_storage;
  const uint32_t bar = smem_u32(&bar_storage);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);  // expects one arrival that never comes
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_bounded(bar, 0, budget_ns, status);
}

}  // namespace

int launch_selftest_wait(int32_t* status, int64_t budget_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(status, budget_ns);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
}

}  // namespace gqa
