// Declarations shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ptx.cuh"

namespace lens {

constexpr int kHidden = 1536;
constexpr int kHeads = 24;
constexpr int kHeadDim = 64;
constexpr int kMlp = 4096;
constexpr int kInCh = 128;
constexpr int kLatCh = 32;
constexpr int kTxtLayers = 4;
constexpr int kTxtDim = 2880;
constexpr int kFreqDim = 256;
constexpr int kModPerStream = 6 * kHidden;    // 9216
constexpr int kModPerBlock = 2 * kModPerStream;
constexpr int kMaxTimesteps = 64;             // per modulation launch (GEMM N <= 64)

struct TimestepList {
  float t[kMaxTimesteps];
  int T;
};

// Valid text lengths per batch row (text keys at and past n[b] are padding).
constexpr int kMaxRows = 64;
struct TextLengths {
  int n[kMaxRows];
};

// attention.cu (txt_len == nullptr: every text key is valid)
cudaError_t launch_joint_attention(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, int B,
                                   int heads, int n_txt, int n_img, __nv_bfloat16* out_txt, __nv_bfloat16* out_img,
                                   const TextLengths* txt_len, int* err, cudaStream_t st);

// elementwise.cu
cudaError_t launch_noise_tokens(uint64_t seed, int B, int gh, int gw, float* tokens, cudaStream_t st);
cudaError_t launch_patchify(const float* latent, int B, int gh, int gw, float* tokens, cudaStream_t st);
cudaError_t launch_unpatchify(const float* tokens, int B, int gh, int gw, float* latent, cudaStream_t st);
cudaError_t launch_tokens_to_operand(const float* tokens, int64_t rows, int copies, int64_t copy_rows,
                                     __nv_bfloat16* xin, cudaStream_t st);
cudaError_t launch_rope_table(int gh, int gw, int n_txt, float2* table, cudaStream_t st);
// One RMSNorm + modulate segment: rows of x [M, 1536] fp32 -> y bf16; sample b =
// row / rows_per_batch reads shift / scale at b * mod_stride.
struct RmsSeg {
  const float* x;
  const float* shift;
  const float* scale;
  __nv_bfloat16* y;
  int M;
  int rows_per_batch;
  int64_t mod_stride;
};
cudaError_t launch_rmsnorm_modulate(const RmsSeg& s0, const RmsSeg& s1, float eps, cudaStream_t st);
cudaError_t launch_rmsnorm_modulate(const float* x, int M, int rows_per_batch, const float* shift,
                                    const float* scale, int64_t mod_stride, float eps, __nv_bfloat16* y,
                                    cudaStream_t st);
cudaError_t launch_text_norm(const __nv_bfloat16* E, int rows, const float* gains, float eps, __nv_bfloat16* out,
                             cudaStream_t st);
cudaError_t launch_timestep_features(const TimestepList& tl, float* out, cudaStream_t st);
cudaError_t launch_small_linear(const float* x, int T, int K, const __nv_bfloat16* W, const float* bias, int N,
                                bool silu_in, float* out, __nv_bfloat16* silu_out_bf16, int silu_rows,
                                cudaStream_t st);
cudaError_t launch_euler_cfg(float* x, const float* v, int64_t per_sample, int B, bool cfg, float dt,
                             float guidance, __nv_bfloat16* xin, cudaStream_t st);
cudaError_t launch_euler_plain(float* x, const float* vc, const float* vu, int64_t n, float dt, float guidance,
                               cudaStream_t st);
// norm-rescaled CFG: pass 1 writes kCfgNormParts x 2 fp64 partial norms per sample to
// `part` ([B][kCfgNormParts][2]); pass 2 reduces them and applies
// x -= dt (phi |c| / |p| + 1 - phi) p, p = u + g (c - u), refreshing xin when given
constexpr int kCfgNormParts = 128;
cudaError_t launch_cfg_norm_partials(const float* vc, const float* vu, int64_t per_sample, int B, float guidance,
                                     double* part, cudaStream_t st);
cudaError_t launch_euler_cfg_rescaled(float* x, const float* vc, const float* vu, int64_t per_sample, int B,
                                      float dt, float guidance, float phi, const double* part, __nv_bfloat16* xin,
                                      int xin_copies, cudaStream_t st);
// x -= dt (u + g (c - u)) (or dt c for vu == NULL) on n = rows x 128 values, with one
// img_in operand row refreshed per token
cudaError_t launch_euler_step(float* x, const float* vc, const float* vu, int64_t n, float dt, float guidance,
                              __nv_bfloat16* xin, cudaStream_t st);

}  // namespace lens
