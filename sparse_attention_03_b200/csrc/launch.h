// Kernel launch with programmatic dependent launch (PDL): the grid may be
// scheduled while the previous kernel on the stream is still finishing, so its
// launch latency hides behind that kernel's tail. Every kernel launched this way
// calls pdl_wait() (griddepcontrol.wait) before it reads anything a previous
// kernel may have written; the wait returns once that kernel has completed and
// its memory is visible. Without the attribute the wait is a no-op.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace lsa {

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

}  // namespace lsa
