// Launch helpers.  Raising a kernel's dynamic shared-memory limit: the attribute is
// per device, so a launcher records, per device, that it has been set (one bit per
// device ordinal).  Programmatic dependent launch: the hot kernels of a forward are
// launched so that each may start (its CTAs scheduled as SMs free up, running the
// set-up that touches only shared memory and TMEM) before the kernel ahead of it in
// the stream has finished; every such kernel executes griddepcontrol.wait before it
// reads or writes global memory that kernels ahead of it touch.  LENS_PDL=0 in the
// environment turns it off (plain stream order), for measurement.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include <atomic>

namespace lens {

template <class F>
inline cudaError_t ensure_smem_limit(F* func, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

inline bool pdl_enabled() {
  static const bool on = [] {
    const char* e = getenv("LENS_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

// Set while a launch is bracketed by profiling events (this thread only).
inline bool& pdl_suspended() {
  static thread_local bool s = false;
  return s;
}

// kernel<<<grid, block, smem, st>>>(args...), with programmatic dependent launch
// when enabled.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
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
  cfg.numAttrs = pdl_enabled() && !pdl_suspended() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace lens
