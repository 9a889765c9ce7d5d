// ssta_selftest_bounded_wait: runs the library's bounded mbarrier wait (the one
// every pipeline wait of the attention kernel uses) on the device against a
// barrier phase that either completes (control) or never completes, so that a
// test can check that a stalled pipeline ends in SSTA_ERR_DEVICE_TIMEOUT in the
// status word and an exited kernel, never in a hang or a trap.
#include "ssta_internal.h"
#include "ssta_wait.cuh"

namespace ssta {
namespace {

using namespace wait;

// One warp, one barrier expecting one arrival.  With `complete`, thread 0 arrives
// first and the wait returns at once; otherwise nothing ever arrives and the wait
// gives up after timeout_ns.
__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel(int32_t* status, uint64_t timeout_ns,
                                                                   int complete) {
  __shared__ __align__(8) uint64_t barrier_word;
  __shared__ int abort_flag;
  const uint32_t bar = smem_u32(&barrier_word);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  if (complete && threadIdx.x == 0) mbar_arrive(bar);
  __syncwarp();
  const Ctl ctl{&abort_flag, status, timeout_ns};
  wait_warp(bar, 0, ctl);
}

}  // namespace
}  // namespace ssta

using namespace ssta;

extern "C" ssta_status ssta_selftest_bounded_wait(int32_t timeout_us, int32_t complete, void* workspace,
                                                  size_t workspace_bytes, void* stream) {
  if (timeout_us < 1 || timeout_us > 2000000) return SSTA_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < 256) return SSTA_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) % 256) != 0) return SSTA_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* status = static_cast<int32_t*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(int32_t), s) != cudaSuccess) return SSTA_ERR_LAUNCH;
  bounded_wait_selftest_kernel<<<1, 32, 0, s>>>(status, (uint64_t)timeout_us * 1000ull, complete ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? SSTA_OK : SSTA_ERR_LAUNCH;
}
