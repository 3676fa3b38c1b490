// Self-test of the bounded mbarrier wait used by every kernel of libgqa_attn: one
// CTA waits on a barrier that no thread or copy ever completes.  The wait must give
// up after its budget, record GQA_ERR_DEVICE_TIMEOUT in the status word and let the
// kernel return normally, so a lost arrival never hangs the GPU.  A second self-test
// covers the index checks of a build made with GQA_DEBUG_BOUNDS.
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

#if defined(GQA_DEBUG_BOUNDS)
// Self-test of the index checks of a checked build: every thread checks one shared
// address inside a 1 KiB region of the dynamic window and one global index inside a
// buffer; with `planted` set, thread 0 also checks an address one 16-byte step past the
// region's end and an index one past the buffer's end.  Only the checks run: no access
// is made at any of these addresses, so the planted ones fault nothing.  The flag must
// stay clear without `planted` and be set with it.
__global__ void selftest_bounds_kernel(int32_t* status, int planted) {
  extern __shared__ __align__(16) char smem[];
  if (threadIdx.x == 0) debug_flag_reset();
  __syncthreads();
  const uint32_t lo = smem_u32(smem);
  debug_region_ok(lo + 16 * threadIdx.x, 16, lo, 1024);
  debug_index_ok(int64_t(threadIdx.x), 64);
  if (planted && threadIdx.x == 0) {
    debug_region_ok(lo + 1024, 16, lo, 1024);
    debug_index_ok(64, 64);
  }
  __syncthreads();
  if (threadIdx.x == 0) debug_flag_report(status);
}
#endif

}  // namespace

int launch_selftest_wait(int32_t* status, int64_t budget_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(status, budget_ns);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
}

int launch_selftest_bounds(int32_t* status, int planted, cudaStream_t stream) {
#if defined(GQA_DEBUG_BOUNDS)
  // 1 KiB region + the 16-byte flag at the window's end
  selftest_bounds_kernel<<<1, 64, 1024 + 16, stream>>>(status, planted);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
#else
  (void)status, (void)planted, (void)stream;
  return GQA_ERR_UNSUPPORTED;  // the checks are compiled out of this build
#endif
}

}  // namespace gqa
