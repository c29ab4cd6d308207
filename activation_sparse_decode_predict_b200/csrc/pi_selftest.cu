// pi_selftest.cu -- makes the persistent kernel's bounded waits run out on
// purpose, so that tests can check the timeout path without faulting a GPU.
//
// Kind 0: one CTA waits on an mbarrier that nothing arrives on.
// Kind 1: one CTA waits on a grid-barrier count that nothing reaches.
// Both waits give up after the same limit the decode kernel uses, record
// PI_ERR_TIMEOUT in the workspace status word, raise the abort flag and return.
#include <cuda_runtime.h>

#include "pi.h"
#include "pi_args.h"
#include "pi_common.cuh"
#include "pi_sync.cuh"

namespace pi {

namespace {

__global__ void k_wait_never(Ctrl* ctrl, int kind) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  if (kind == 0) {
    mbar_wait(&bar, 0, ctrl);  // phase 0 never completes
  } else {
    const unsigned base = ld_relaxed_u32(&ctrl->bar_count);
    grid_wait(ctrl, base, 1000000u, 1u);  // a count nobody adds up to
  }
}

}  // namespace
}  // namespace pi

extern "C" pi_status pi_selftest_bounded_wait(void* ws, int32_t kind, void* stream) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) {
    pi::set_last_error("ws is NULL or not 256-byte aligned");
    return PI_ERR_INVALID_ARG;
  }
  if (kind != 0 && kind != 1) {
    pi::set_last_error("kind must be 0 (mbarrier) or 1 (grid barrier)");
    return PI_ERR_INVALID_ARG;
  }
  pi::k_wait_never<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<pi::Ctrl*>(ws), kind);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    pi::set_last_error(cudaGetErrorString(e));
    return PI_ERR_CUDA;
  }
  return PI_OK;
}
