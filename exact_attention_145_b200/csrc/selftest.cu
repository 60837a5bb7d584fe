// selftest.cu - failure-detection self-test of the bounded pipeline wait.
//
// One warp waits, with the same bounded mbarrier wait the attention kernels
// use, on a barrier that nothing ever arrives on. The wait gives up after its
// cycle limit (about a second), raises the CTA's abort flag and the kernel
// reports ATTN_DEV_TIMEOUT in the caller's status word, then exits normally,
// leaving the CUDA context usable. No fault, trap or endless loop is involved.
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/attn.h"
#include "sm100.cuh"

namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    attn_sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    attn_sm100::fence_barrier_init();
  }
  __syncwarp();
  // Phase 0 never completes: nothing arrives on the barrier.
  const bool got = attn_sm100::mbar_wait(&bar, 0, &abort_flag);
  if (threadIdx.x == 0 && !got && abort_flag) atomicOr(status, ATTN_DEV_TIMEOUT);
}

}  // namespace

extern "C" attn_status attn_selftest_wait_timeout(int* status, void* stream) {
  if (status == nullptr) return ATTN_ERR_INVALID_ARG;
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
