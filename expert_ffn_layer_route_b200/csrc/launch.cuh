// Kernel launch with programmatic dependent launch (PDL) enabled, so a kernel
// can be scheduled while its predecessor in the stream drains; the kernels
// synchronise with pdl_wait_and_trigger() before touching global memory.
// MOE_PDL=0 in the environment launches without the attribute.
#pragma once

#include <cstdlib>
#include <cuda_runtime.h>

namespace moe {

inline bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("MOE_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
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
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace moe
