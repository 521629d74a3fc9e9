// debug.cu -- test hooks that exercise device-side failure handling without
// faulting the GPU (declared in rans_b200_debug.h).
#include "rans_b200_debug.h"
#include "rans_common.cuh"

namespace rb {
namespace {

// An mbarrier expecting 16 bytes that no copy delivers: the same bounded
// try-wait as the table staging gives up after `limit` tries and records
// RANS_ERR_TIMEOUT.  Nothing is in flight when the kernel returns.
__global__ void wait_timeout_kernel(uint32_t limit, int32_t *status) {
  __shared__ uint64_t bar_storage;
  const uint32_t bar = smem_addr(&bar_storage);
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0)
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(16u)
                 : "memory");
  bool done = false;
  for (uint32_t it = 0; it < limit; ++it) {
    if (mbar_try_wait(bar, 0)) {
      done = true;
      break;
    }
  }
  if (!__syncthreads_or(done ? 1 : 0) && threadIdx.x == 0) report(status, RANS_ERR_TIMEOUT, -1);
}

}  // namespace
}  // namespace rb

extern "C" __attribute__((visibility("default"))) int rans_debug_wait_timeout(
    void *workspace, uint32_t limit, void *stream) {
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) != 0 || limit < 1 ||
      limit > (1u << 21))
    return RANS_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, 256, s) != cudaSuccess) return RANS_ERR_CUDA;
  rb::wait_timeout_kernel<<<1, 32, 0, s>>>(limit, reinterpret_cast<int32_t *>(workspace));
  return cudaGetLastError() == cudaSuccess ? RANS_OK : RANS_ERR_CUDA;
}
