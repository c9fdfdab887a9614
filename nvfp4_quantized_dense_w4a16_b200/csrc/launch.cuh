// Kernel launch with programmatic dependent launch, shared by the kernels
// that chain within one FFN call.
#pragma once

#include <cuda_runtime.h>

#include <utility>

#include "profile.h"

namespace ffn {

// Launch with programmatic stream serialisation: the kernel may begin while
// the previous kernel in the stream finishes (the kernels wait for its
// results with griddepcontrol.wait).  Not while per-kernel timing is
// recorded: an event between two kernels must not let the second start early.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = profiling() ? 0 : 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace ffn
