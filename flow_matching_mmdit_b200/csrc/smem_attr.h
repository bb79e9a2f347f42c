// Raising a kernel's dynamic shared-memory limit: the attribute is per device, so a
// launcher records, per device, that it has been set (one bit per device ordinal).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

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

}  // namespace lens
