// pi_launch.h -- host-side launch with programmatic dependent launch allowed:
// the kernel may be scheduled while the previous kernel on the stream is
// still running, and it orders itself after that kernel with pdl_wait()
// (pi_common.cuh).  Also captured into CUDA graphs as programmatic edges.
#pragma once
#include <cuda_runtime.h>

#include <utility>

namespace pi {

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace pi
