// Timestep embedding that allocates nothing: the same kernels as the handle's
// timestep path (sinusoid -> linear_1 -> SiLU -> linear_2), with the two
// intermediate activations kept in a fixed device array defined in this file
// instead of a handle's workspace.
//
// Who needs it: code that may not call cudaMalloc or any allocating routine, for
// example a plugin inside a host application that owns and budgets all device
// memory itself, or a latency-critical loop where cudaMalloc's implicit device
// synchronisation (and its possible failure) is not acceptable.  Such a caller only
// supplies the weights, the timesteps and the output buffer.
#include <math.h>

#include <mutex>

#include "kernels.cuh"
#include "lens_dit.h"

using namespace lens;

namespace {

constexpr int kNoAllocMaxT = 64;   // timesteps per call
// the timesteps travel to the feature kernel in a TimestepList by value
static_assert(kNoAllocMaxT <= kMaxTimesteps, "TimestepList cannot hold kNoAllocMaxT timesteps");
// sinusoid features [T, 256] followed by the hidden layer [T, 1536], fp32: 448 KiB.
// Every GPU that loads the library holds this array until the process exits.
constexpr size_t kScratchFloats = (size_t)kNoAllocMaxT * (kFreqDim + kHidden);
static __device__ __align__(256) float g_noalloc_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device.  In host code the array's
// name is only a host-side stand-in, so the address is looked up once per device
// (with that device current) and cached.  With lazy module loading (the CUDA
// default) this lookup is also what loads the module on that device and reserves
// the array, so it can fail for lack of device memory: that case is reported as
// LENS_ERR_OOM, any other failure as LENS_ERR_CUDA.
lens_status scratch_on_current_device(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LENS_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LENS_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    float* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_noalloc_scratch);
    if (e == cudaErrorMemoryAllocation) {
      cudaGetLastError();
      return LENS_ERR_OOM;
    }
    if (e != cudaSuccess || !p) return LENS_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return LENS_OK;
}

}  // namespace

extern "C" lens_status lens_op_timestep_embed_noalloc(const float* t, int T, const uint16_t* w1, const float* b1,
                                                      const uint16_t* w2, const float* b2, float* temb,
                                                      void* stream) {
  if (!t || !w1 || !w2 || !temb) return LENS_ERR_INVALID_ARG;
  // the weight rows are read 16 bytes at a time
  if ((reinterpret_cast<uintptr_t>(w1) | reinterpret_cast<uintptr_t>(w2)) & 15) return LENS_ERR_INVALID_ARG;
  if (T < 1 || T > kNoAllocMaxT) return LENS_ERR_SHAPE;
  for (int i = 0; i < T; ++i)
    if (!isfinite(t[i])) return LENS_ERR_INVALID_ARG;
  float* scratch = nullptr;
  lens_status s = scratch_on_current_device(&scratch);
  if (s != LENS_OK) return s;
  float* feat = scratch;                                  // [T, 256]
  float* hid = scratch + (size_t)kNoAllocMaxT * kFreqDim;  // [T, 1536]
  // Both scratch regions are fully written before they are read, so nothing left
  // over from an earlier call is ever used.
  TimestepList tl;
  tl.T = T;
  for (int i = 0; i < T; ++i) tl.t[i] = t[i];
  cudaStream_t st = (cudaStream_t)stream;
  if (launch_timestep_features(tl, feat, st) != cudaSuccess) return LENS_ERR_CUDA;
  if (launch_small_linear(feat, T, kFreqDim, reinterpret_cast<const __nv_bfloat16*>(w1), b1, kHidden, false, hid,
                          nullptr, 0, st) != cudaSuccess)
    return LENS_ERR_CUDA;
  if (launch_small_linear(hid, T, kHidden, reinterpret_cast<const __nv_bfloat16*>(w2), b2, kHidden, true, temb,
                          nullptr, 0, st) != cudaSuccess)
    return LENS_ERR_CUDA;
  return LENS_OK;
}
