// Kernel launch with programmatic dependent launch (PDL) enabled, so a kernel
// can be scheduled while its predecessor in the stream drains; the kernels
// synchronise with pdl_wait_and_trigger() before touching global memory.
// MOE_PDL=0 in the environment launches without the attribute.
#pragma once

#include <cstdint>
#include <cstdlib>
#include <mutex>

#include <cuda_runtime.h>

namespace moe {

// Handle of the CUDA context current on this thread (0 if none yet), read
// through the driver entry point.  State that lives inside a context -- a
// kernel's function attributes, the device address of a module variable -- is
// cached under (device, context), so that a new context on the same device
// (after cudaDeviceReset, or one the caller made current) is set up again.
uintptr_t current_ctx();

// The dynamic shared-memory limit of kernel `Kern` is a per-device (per
// context) attribute: raise it once per device and context, not per launch.
template <auto Kern>
inline cudaError_t set_dyn_smem_once(size_t smem) {
  struct Slot {
    uintptr_t ctx = 0;
    size_t smem = 0;
  };
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static Slot slots[kMaxDev];
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDev) return cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  std::lock_guard<std::mutex> lk(mu);
  Slot& s = slots[dev];
  const uintptr_t ctx = current_ctx();
  if (ctx != 0 && s.ctx == ctx && s.smem >= smem) return cudaSuccess;
  err = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const uintptr_t now = current_ctx();  // the call above creates the context if there was none
  s.smem = (now == s.ctx && s.smem > smem) ? s.smem : smem;
  s.ctx = now;
  return cudaSuccess;
}

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
