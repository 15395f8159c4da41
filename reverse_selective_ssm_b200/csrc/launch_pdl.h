// Kernel launch with programmatic stream serialization: the grid may be
// scheduled while the previous kernel of the stream is still running, and
// waits for it in grid_dep_wait (common.cuh) before touching what it writes.
// Its launch and its CTAs' set-up then overlap the previous grid's tail.
// Inside a CUDA graph capture the dependency becomes a programmatic edge.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace r2l {

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace r2l
