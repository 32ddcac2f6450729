// Host-side kernel launch with programmatic dependent launch (PDL).
//
// Kernels of one call (and of consecutive calls on a stream) form a chain:
// with the programmatic-serialisation attribute the next kernel's CTAs are
// scheduled as soon as the current kernel's CTAs have all started and called
// pdl_trigger(), and they block in pdl_wait() until it has completed.  This
// hides the launch latency between the short kernels of a decode step.  Set
// PBSA_PDL=0 in the environment to launch with plain stream order.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace pbsa {

bool pdl_enabled();
int sm_count();   // SMs of the current device

template <typename... KArgs, typename... Args>
inline cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace pbsa
