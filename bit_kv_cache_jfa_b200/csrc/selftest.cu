// selftest.cu — the bounded-wait error path, exercised without a fault.
#include "jfa_internal.cuh"

namespace jfa {

// One warp waits on an mbarrier whose phase cannot complete: it expects 16
// bytes that no copy delivers.  The bounded wait gives up after about a
// second and the kernel records JFA_DEVERR_TIMEOUT in the workspace flag, as
// the scan does when a record copy never lands; the context stays usable.
__global__ void bounded_wait_kernel(uint32_t* flag) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_expect_tx(&bar, 16);
  __syncwarp();
  const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&bar, 0));
  if (!ok && threadIdx.x == 0) set_flag(flag, JFA_DEVERR_TIMEOUT);
}

int launch_bounded_wait_selftest(uint32_t* flag, cudaStream_t st) {
  bounded_wait_kernel<<<1, 32, 0, st>>>(flag);
  return cudaGetLastError() == cudaSuccess ? JFA_OK : JFA_ERR_CUDA;
}

}  // namespace jfa
