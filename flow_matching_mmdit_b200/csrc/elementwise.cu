// Memory-bound kernels of the denoiser path: seeded noise, patchify / unpatchify,
// the RoPE table, RMSNorm + AdaLN modulation, the text-layer norm, the timestep
// embedding MLP and the Euler / CFG update.  All accesses are coalesced (warp-per-row
// or element-per-thread over the contiguous output), 128-bit where the row allows.
#include <math.h>

#include "kernels.cuh"
#include "smem_attr.h"

namespace lens {

namespace {

constexpr int kThreads = 256;

inline int grid_for(int64_t n, int threads = kThreads) {
  int64_t g = (n + threads - 1) / threads;
  return (int)(g > (1 << 30) ? (1 << 30) : (g < 1 ? 1 : g));
}

// ---------------------------------------------------------------- noise
// SplitMix64 output function at state v (Steele, Lea and Flood 2014; Vigna's
// splitmix64.c): add the golden gamma, two xor-shift-multiply rounds, final shift.
__device__ __forceinline__ uint64_t splitmix64(uint64_t v) {
  uint64_t z = v + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Standard normal for latent element n: Box-Muller on two SplitMix64 words,
// u1 in (0, 1], u2 in [0, 1), evaluated in double and rounded to float.
__device__ __forceinline__ float normal_at(uint64_t seed, uint64_t n) {
  const uint64_t w1 = splitmix64(seed ^ splitmix64(2 * n));
  const uint64_t w2 = splitmix64(seed ^ splitmix64(2 * n + 1));
  const double u1 = (double)((w1 >> 11) + 1) * 0x1.0p-53;
  const double u2 = (double)(w2 >> 11) * 0x1.0p-53;
  return (float)(sqrt(-2.0 * log(u1)) * cos(2.0 * M_PI * u2));
}

// Token element e of [B, gh*gw, 128] <-> latent element of [B, 32, 2gh, 2gw]:
// token (i, j) in row-major order, feature c*4 + 2r + s = latent[c, 2i + r, 2j + s].
__device__ __forceinline__ int64_t latent_index_of_token(int64_t e, int gh, int gw) {
  const int f = (int)(e & 127);
  const int64_t tokb = e >> 7;
  const int64_t ntok = (int64_t)gh * gw;
  const int64_t b = tokb / ntok;
  const int tok = (int)(tokb - b * ntok);
  const int i = tok / gw, j = tok - (tok / gw) * gw;
  const int c = f >> 2, r = (f >> 1) & 1, s = f & 1;
  return (((b * kLatCh + c) * (2 * gh) + 2 * i + r) * (int64_t)(2 * gw)) + 2 * j + s;
}

__global__ void noise_tokens_kernel(uint64_t seed, int64_t n, int gh, int gw, float* __restrict__ tokens) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x)
    tokens[e] = normal_at(seed, (uint64_t)latent_index_of_token(e, gh, gw));
}

__global__ void patchify_kernel(const float* __restrict__ latent, int64_t n, int gh, int gw,
                                float* __restrict__ tokens) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x)
    tokens[e] = latent[latent_index_of_token(e, gh, gw)];
}

__global__ void unpatchify_kernel(const float* __restrict__ tokens, int64_t n, int gh, int gw,
                                  float* __restrict__ latent) {
  const int W2 = 2 * gw, H2 = 2 * gh;
  for (int64_t l = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; l < n; l += (int64_t)gridDim.x * blockDim.x) {
    const int x = (int)(l % W2);
    const int64_t r1 = l / W2;
    const int y = (int)(r1 % H2);
    const int64_t r2 = r1 / H2;
    const int c = (int)(r2 % kLatCh);
    const int64_t b = r2 / kLatCh;
    const int64_t tok = b * gh * gw + (int64_t)(y >> 1) * gw + (x >> 1);
    latent[l] = tokens[tok * kInCh + c * 4 + (y & 1) * 2 + (x & 1)];
  }
}

// fp32 tokens -> bf16 GEMM operand [rows, 256] = [hi | lo], hi = bf16(x),
// lo = bf16(x - hi), so the 128 -> 1536 projection sees x to ~16 bits.
__global__ void tokens_to_operand_kernel(const float* __restrict__ tokens, int64_t n, int copies, int64_t copy_rows,
                                         __nv_bfloat16* __restrict__ xin) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const float x = tokens[e];
    const __nv_bfloat16 hi = __float2bfloat16_rn(x);
    const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
    const int64_t row = e >> 7;
    const int f = (int)(e & 127);
    for (int c = 0; c < copies; ++c) {
      __nv_bfloat16* dst = xin + (row + c * copy_rows) * 256;
      dst[f] = hi;
      dst[128 + f] = lo;
    }
  }
}

// ---------------------------------------------------------------- RoPE table
// Pair p of the 64-dim head: p < 4 -> axis 0 (8 dims), p < 18 -> axis 1 (28 dims,
// image row i), else axis 2 (28 dims, image column j).  Pair m of an axis of d_a
// dims turns by pos * 10000^(-2m / d_a).  Text tokens (ids 0) get cos 1, sin 0.
__global__ void rope_table_kernel(int gh, int gw, int n_txt, int ntok, float2* __restrict__ table) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= ntok * 32) return;
  const int tok = e >> 5, p = e & 31;
  int pos = 0, m, da;
  if (p < 4) {
    m = p;
    da = 8;
  } else if (p < 18) {
    m = p - 4;
    da = 28;
    if (tok >= n_txt) pos = (tok - n_txt) / gw;
  } else {
    m = p - 18;
    da = 28;
    if (tok >= n_txt) pos = (tok - n_txt) % gw;
  }
  const double ang = (double)pos * pow(10000.0, -2.0 * m / (double)da);
  table[e] = make_float2((float)cos(ang), (float)sin(ang));
}

// ---------------------------------------------------------------- RMSNorm + modulate
// One warp per row of 1536 fp32: y = (1 + scale) * x * rsqrt(mean(x^2) + eps) + shift.
// Up to two independent segments (the image and the text stream of a block) share
// one launch: rows [0, s0.M) belong to segment 0, the next s1.M rows to segment 1.
// Every warp issues its row's twelve 16-byte loads first; meanwhile the CTA stages
// the shift and 1 + scale of its first row's sample in shared memory once (12 KB),
// so the eight warps of a CTA read them from there instead of each pulling them
// through L1.  A warp whose row belongs to another sample or segment (a CTA that
// straddles a boundary) reads its own from global memory.
// 64 registers (4 blocks of 256 per SM): the 4352 rows of a 1024^2 block fit one wave.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// The row's segment, picked field by field: taking the address of a by-value kernel
// parameter would make the compiler copy both segments to local memory.
struct RmsRow {
  const float* x;
  const float* shift;
  const float* scale;
  __nv_bfloat16* y;
  bool ok;
};
__device__ __forceinline__ RmsRow rms_row(const RmsSeg& s0, const RmsSeg& s1, int row) {
  const bool second = row >= s0.M;
  const int r = second ? row - s0.M : row;
  const int b = r / (second ? s1.rows_per_batch : s0.rows_per_batch);
  const int64_t mod = b * (second ? s1.mod_stride : s0.mod_stride);
  RmsRow o;
  o.ok = !second || r < s1.M;
  o.x = (second ? s1.x : s0.x) + (int64_t)r * kHidden;
  o.y = (second ? s1.y : s0.y) + (int64_t)r * kHidden;
  o.shift = (second ? s1.shift : s0.shift) + mod;
  o.scale = (second ? s1.scale : s0.scale) + mod;
  return o;
}

__global__ void __launch_bounds__(256, 4) rmsnorm_modulate_kernel(RmsSeg s0, RmsSeg s1, float eps) {
  __shared__ float4 sm_shift[kHidden / 4], sm_scale[kHidden / 4];
  grid_dependency_sync();
  // the CTA's first row decides which sample's modulation is staged; the copies are
  // asynchronous (global -> shared, no registers) and overlap the row loads below
  const RmsRow first = rms_row(s0, s1, blockIdx.x * (blockDim.x >> 5));   // ok: the grid covers M rows
  for (int i = threadIdx.x; i < kHidden / 4; i += blockDim.x) {
    cp_async16(&sm_shift[i], first.shift + 4 * i);
    cp_async16(&sm_scale[i], first.scale + 4 * i);
  }
  cp_async_commit();
  const RmsRow rw = rms_row(s0, s1, blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5));
  const int lane = threadIdx.x & 31;
  float4 v[12];
  if (rw.ok) {
    const float4* xr = reinterpret_cast<const float4*>(rw.x);
#pragma unroll
    for (int i = 0; i < 12; ++i) v[i] = xr[lane + 32 * i];
  }
  cp_async_wait_all();
  __syncthreads();
  if (!rw.ok) return;
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < 12; ++i) ss += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss * (1.0f / kHidden) + eps);
  const bool staged = rw.shift == first.shift;
  const float4* sh = staged ? sm_shift : reinterpret_cast<const float4*>(rw.shift);
  const float4* sc = staged ? sm_scale : reinterpret_cast<const float4*>(rw.scale);
  uint2* yr = reinterpret_cast<uint2*>(rw.y);
#pragma unroll
  for (int i = 0; i < 12; ++i) {
    const float4 a = sh[lane + 32 * i], c = sc[lane + 32 * i];
    uint2 w;
    w.x = pack_bf16x2((1.f + c.x) * v[i].x * r + a.x, (1.f + c.y) * v[i].y * r + a.y);
    w.y = pack_bf16x2((1.f + c.z) * v[i].z * r + a.z, (1.f + c.w) * v[i].w * r + a.w);
    yr[lane + 32 * i] = w;
  }
}

// ---------------------------------------------------------------- text layers
// One warp per (token, layer): RMSNorm of the 2880-wide slice times txt_norm.l,
// written at column l * 2880 of the concatenated 11520-wide row.
__global__ void text_norm_kernel(const __nv_bfloat16* __restrict__ E, int rows, const float* __restrict__ gains,
                                 float eps, __nv_bfloat16* __restrict__ out) {
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= rows * kTxtLayers) return;
  const int layer = w % kTxtLayers;
  const uint4* src = reinterpret_cast<const uint4*>(E + (int64_t)w * kTxtDim);
  constexpr int kVec = kTxtDim / 8;   // 360
  float ss = 0.f;
  for (int i = lane; i < kVec; i += 32) {
    const uint4 u = src[i];
    const uint32_t p[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = bf16lo(p[j]), c = bf16hi(p[j]);
      ss += a * a + c * c;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss * (1.0f / kTxtDim) + eps);
  const float* gl = gains + layer * kTxtDim;
  uint4* dst = reinterpret_cast<uint4*>(out + (int64_t)(w / kTxtLayers) * (kTxtLayers * kTxtDim) + layer * kTxtDim);
  for (int i = lane; i < kVec; i += 32) {
    const uint4 u = src[i];
    const uint32_t p[4] = {u.x, u.y, u.z, u.w};
    uint32_t q[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      q[j] = pack_bf16x2(bf16lo(p[j]) * r * __ldg(gl + 8 * i + 2 * j), bf16hi(p[j]) * r * __ldg(gl + 8 * i + 2 * j + 1));
    dst[i] = make_uint4(q[0], q[1], q[2], q[3]);
  }
}

// ---------------------------------------------------------------- timestep embedding
// [cos(1000 t f_k) | sin(1000 t f_k)], f_k = exp(-ln(10000) k / 128), in double.
__global__ void timestep_features_kernel(TimestepList tl, float* __restrict__ out) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= tl.T * kFreqDim) return;
  const int ti = e / kFreqDim, k = e % kFreqDim;
  const int half = kFreqDim / 2;
  const int kk = k < half ? k : k - half;
  const double f = exp(-log(10000.0) * (double)kk / (double)half);
  const double a = 1000.0 * (double)tl.t[ti] * f;
  out[e] = (float)(k < half ? cos(a) : sin(a));
}

// out[t][n] = sum_k W[n][k] * act(x[t][k]) + bias[n] for T <= 64 rows; act = SiLU or
// identity.  One warp per output feature n, 8 rows of x staged in shared memory at a
// time.  Optionally also writes bf16(SiLU(out)) and zero rows up to silu_rows (the
// B operand of the modulation GEMM).
__global__ void small_linear_kernel(const float* __restrict__ x, int T, int K, const __nv_bfloat16* __restrict__ W,
                                    const float* __restrict__ bias, int N, int silu_in, float* __restrict__ out,
                                    __nv_bfloat16* __restrict__ silu_out, int silu_rows) {
  extern __shared__ float xs[];   // [8][K]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * (blockDim.x >> 5) + warp;
  const __nv_bfloat16* wr = W + (int64_t)(n < N ? n : 0) * K;
  for (int t0 = 0; t0 < T; t0 += 8) {
    const int tc = min(8, T - t0);
    __syncthreads();
    for (int i = threadIdx.x; i < tc * K; i += blockDim.x) {
      float v = x[(int64_t)t0 * K + i];
      if (silu_in) v = v / (1.f + expf(-v));
      xs[i] = v;
    }
    __syncthreads();
    float acc[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) acc[r] = 0.f;
    for (int k = lane * 8; k < K; k += 256) {
      const uint4 u = *reinterpret_cast<const uint4*>(wr + k);
      const uint32_t p[4] = {u.x, u.y, u.z, u.w};
      float wv[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        wv[2 * j] = bf16lo(p[j]);
        wv[2 * j + 1] = bf16hi(p[j]);
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (r < tc) {
          const float* xr = xs + r * K + k;
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[r] += wv[j] * xr[j];
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      float a = acc[r];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0 && n < N && r < tc) {
        const float y = a + (bias ? bias[n] : 0.f);
        out[(int64_t)(t0 + r) * N + n] = y;
        if (silu_out) silu_out[(int64_t)(t0 + r) * N + n] = __float2bfloat16_rn(y / (1.f + expf(-y)));
      }
    }
  }
  if (silu_out && lane == 0 && n < N)
    for (int r = T; r < silu_rows; ++r) silu_out[(int64_t)r * N + n] = __float2bfloat16_rn(0.f);
}

// ---------------------------------------------------------------- Euler / CFG
// x -= dt * v, v = vu + g (vc - vu) under CFG (v rows: B cond then B uncond) or vc.
// Also refreshes the bf16 [hi | lo] operand of img_in for the next step (both the
// cond and the uncond copy under CFG).
__global__ void euler_cfg_kernel(float* __restrict__ x, const float* __restrict__ v, int64_t n, int64_t total_cond,
                                 int cfg, float dt, float g, __nv_bfloat16* __restrict__ xin) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const float vc = v[e];
    float vv = vc;
    if (cfg) {
      const float vu = v[total_cond + e];
      vv = vu + g * (vc - vu);
    }
    const float xn = x[e] - dt * vv;
    x[e] = xn;
    if (xin) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(xn);
      const __nv_bfloat16 lo = __float2bfloat16_rn(xn - __bfloat162float(hi));
      const int64_t row = e >> 7;
      const int f = (int)(e & 127);
      xin[row * 256 + f] = hi;
      xin[row * 256 + 128 + f] = lo;
      if (cfg) {
        xin[(row + (total_cond >> 7)) * 256 + f] = hi;
        xin[(row + (total_cond >> 7)) * 256 + 128 + f] = lo;
      }
    }
  }
}

__global__ void euler_plain_kernel(float* __restrict__ x, const float* __restrict__ vc,
                                   const float* __restrict__ vu, int64_t n, float dt, float g) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    float vv = vc[e];
    if (vu) vv = vu[e] + g * (vv - vu[e]);
    x[e] = x[e] - dt * vv;
  }
}

}  // namespace

cudaError_t launch_noise_tokens(uint64_t seed, int B, int gh, int gw, float* tokens, cudaStream_t st) {
  const int64_t n = (int64_t)B * gh * gw * kInCh;
  noise_tokens_kernel<<<grid_for(n), kThreads, 0, st>>>(seed, n, gh, gw, tokens);
  return cudaGetLastError();
}
cudaError_t launch_patchify(const float* latent, int B, int gh, int gw, float* tokens, cudaStream_t st) {
  const int64_t n = (int64_t)B * gh * gw * kInCh;
  patchify_kernel<<<grid_for(n), kThreads, 0, st>>>(latent, n, gh, gw, tokens);
  return cudaGetLastError();
}
cudaError_t launch_unpatchify(const float* tokens, int B, int gh, int gw, float* latent, cudaStream_t st) {
  const int64_t n = (int64_t)B * gh * gw * kInCh;
  unpatchify_kernel<<<grid_for(n), kThreads, 0, st>>>(tokens, n, gh, gw, latent);
  return cudaGetLastError();
}
cudaError_t launch_tokens_to_operand(const float* tokens, int64_t rows, int copies, int64_t copy_rows,
                                     __nv_bfloat16* xin, cudaStream_t st) {
  const int64_t n = rows * kInCh;
  tokens_to_operand_kernel<<<grid_for(n), kThreads, 0, st>>>(tokens, n, copies, copy_rows, xin);
  return cudaGetLastError();
}
cudaError_t launch_rope_table(int gh, int gw, int n_txt, float2* table, cudaStream_t st) {
  const int ntok = n_txt + gh * gw;
  rope_table_kernel<<<grid_for((int64_t)ntok * 32), kThreads, 0, st>>>(gh, gw, n_txt, ntok, table);
  return cudaGetLastError();
}
cudaError_t launch_rmsnorm_modulate(const RmsSeg& s0, const RmsSeg& s1, float eps, cudaStream_t st) {
  const int M = s0.M + s1.M;
  if (M <= 0) return cudaSuccess;
  return launch_pdl(rmsnorm_modulate_kernel, dim3((M + 7) / 8), dim3(256), 0, st, s0, s1, eps);
}
cudaError_t launch_rmsnorm_modulate(const float* x, int M, int rows_per_batch, const float* shift,
                                    const float* scale, int64_t mod_stride, float eps, __nv_bfloat16* y,
                                    cudaStream_t st) {
  RmsSeg a{x, shift, scale, y, M, rows_per_batch, mod_stride};
  RmsSeg none{x, shift, scale, y, 0, 1, 0};
  return launch_rmsnorm_modulate(a, none, eps, st);
}
cudaError_t launch_text_norm(const __nv_bfloat16* E, int rows, const float* gains, float eps, __nv_bfloat16* out,
                             cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const int warps = rows * kTxtLayers;
  text_norm_kernel<<<(warps + 7) / 8, 256, 0, st>>>(E, rows, gains, eps, out);
  return cudaGetLastError();
}
cudaError_t launch_timestep_features(const TimestepList& tl, float* out, cudaStream_t st) {
  timestep_features_kernel<<<grid_for((int64_t)tl.T * kFreqDim), kThreads, 0, st>>>(tl, out);
  return cudaGetLastError();
}
cudaError_t launch_small_linear(const float* x, int T, int K, const __nv_bfloat16* W, const float* bias, int N,
                                bool silu_in, float* out, __nv_bfloat16* silu_out_bf16, int silu_rows,
                                cudaStream_t st) {
  const size_t smem = (size_t)8 * K * sizeof(float);
  static std::atomic<uint64_t> attr{0};
  {
    const cudaError_t e = ensure_smem_limit(small_linear_kernel, 65536, attr);
    if (e != cudaSuccess) return e;
  }
  small_linear_kernel<<<(N + 7) / 8, 256, smem, st>>>(x, T, K, W, bias, N, silu_in ? 1 : 0, out, silu_out_bf16,
                                                       silu_rows);
  return cudaGetLastError();
}
// ------------------------------------------------------------------ norm-rescaled CFG (a14 variant)
// v = f * p with p = u + g (c - u) and f = phi |c| / |p| + (1 - phi), both norms over
// one sample's whole velocity.  Pass 1 writes per-block partial sums of c^2 and p^2
// (fp64) to fixed slots; pass 2 reduces a sample's slots in a fixed order (so the
// result never depends on scheduling) and applies the Euler update.
__global__ void cfg_norm_partials_kernel(const float* __restrict__ vc, const float* __restrict__ vu,
                                         int64_t per_sample, float g, double* __restrict__ part) {
  const int b = blockIdx.y;
  const float* c = vc + (int64_t)b * per_sample;
  const float* u = vu + (int64_t)b * per_sample;
  float sc = 0.f, sp = 0.f;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < per_sample;
       e += (int64_t)gridDim.x * blockDim.x) {
    const float cv = c[e], uv = u[e];
    const float pv = fmaf(g, cv - uv, uv);
    sc = fmaf(cv, cv, sc);
    sp = fmaf(pv, pv, sp);
  }
  double dc = sc, dp = sp;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    dc += __shfl_xor_sync(0xffffffffu, dc, o);
    dp += __shfl_xor_sync(0xffffffffu, dp, o);
  }
  __shared__ double red[2][32];
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    red[0][w] = dc;
    red[1][w] = dp;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double a = 0.0, q = 0.0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
      a += red[0][i];
      q += red[1][i];
    }
    double* dst = part + ((int64_t)b * gridDim.x + blockIdx.x) * 2;
    dst[0] = a;
    dst[1] = q;
  }
}

__global__ void euler_cfg_rescaled_kernel(float* __restrict__ x, const float* __restrict__ vc,
                                          const float* __restrict__ vu, int64_t per_sample, int64_t total,
                                          float dt, float g, float phi, const double* __restrict__ part,
                                          int nparts, __nv_bfloat16* __restrict__ xin, int xin_copies) {
  const int b = blockIdx.y;
  __shared__ float s_f;
  if (threadIdx.x < 32) {
    // lane l sums slots l, l + 32, ...; then a fixed xor tree
    double a = 0.0, q = 0.0;
    for (int i = threadIdx.x; i < nparts; i += 32) {
      a += part[((int64_t)b * nparts + i) * 2];
      q += part[((int64_t)b * nparts + i) * 2 + 1];
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, o);
      q += __shfl_xor_sync(0xffffffffu, q, o);
    }
    if (threadIdx.x == 0) s_f = (float)((double)phi * (q > 0.0 ? sqrt(a / q) : 1.0) + (1.0 - (double)phi));
  }
  __syncthreads();
  const float f = s_f;
  const int64_t base = (int64_t)b * per_sample;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < per_sample;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = base + i;
    const float cv = vc[e], uv = vu[e];
    const float xn = x[e] - dt * (f * fmaf(g, cv - uv, uv));
    x[e] = xn;
    if (xin) {      // refresh the [hi | lo] img_in operand of the cond (and the uncond) row
      const __nv_bfloat16 hi = __float2bfloat16_rn(xn);
      const __nv_bfloat16 lo = __float2bfloat16_rn(xn - __bfloat162float(hi));
      const int64_t row = e >> 7;
      const int ft = (int)(e & 127);
      xin[row * 256 + ft] = hi;
      xin[row * 256 + 128 + ft] = lo;
      if (xin_copies == 2) {
        xin[(row + (total >> 7)) * 256 + ft] = hi;
        xin[(row + (total >> 7)) * 256 + 128 + ft] = lo;
      }
    }
  }
}

cudaError_t launch_cfg_norm_partials(const float* vc, const float* vu, int64_t per_sample, int B, float guidance,
                                     double* part, cudaStream_t st) {
  if (per_sample <= 0 || B <= 0) return cudaSuccess;
  cfg_norm_partials_kernel<<<dim3(kCfgNormParts, B), 256, 0, st>>>(vc, vu, per_sample, guidance, part);
  return cudaGetLastError();
}

cudaError_t launch_euler_cfg_rescaled(float* x, const float* vc, const float* vu, int64_t per_sample, int B,
                                      float dt, float guidance, float phi, const double* part, __nv_bfloat16* xin,
                                      int xin_copies, cudaStream_t st) {
  if (per_sample <= 0 || B <= 0) return cudaSuccess;
  if (xin && (per_sample & 127)) return cudaErrorInvalidValue;
  int64_t blocks = (per_sample + 256 * 8 - 1) / (256 * 8);
  if (blocks > 1024) blocks = 1024;
  euler_cfg_rescaled_kernel<<<dim3((unsigned)blocks, B), 256, 0, st>>>(x, vc, vu, per_sample, per_sample * B, dt,
                                                                       guidance, phi, part, kCfgNormParts, xin,
                                                                       xin_copies);
  return cudaGetLastError();
}

// One Euler step of the step-wise sampler: x -= dt (u + g (c - u)), or dt c when vu is
// NULL, refreshing one [hi | lo] img_in operand row per token.
__global__ void euler_step_kernel(float* __restrict__ x, const float* __restrict__ vc,
                                  const float* __restrict__ vu, int64_t n, float dt, float g,
                                  __nv_bfloat16* __restrict__ xin) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const float cv = vc[e];
    const float vv = vu ? vu[e] + g * (cv - vu[e]) : cv;
    const float xn = x[e] - dt * vv;
    x[e] = xn;
    const __nv_bfloat16 hi = __float2bfloat16_rn(xn);
    const __nv_bfloat16 lo = __float2bfloat16_rn(xn - __bfloat162float(hi));
    xin[(e >> 7) * 256 + (e & 127)] = hi;
    xin[(e >> 7) * 256 + 128 + (e & 127)] = lo;
  }
}

cudaError_t launch_euler_step(float* x, const float* vc, const float* vu, int64_t n, float dt, float guidance,
                              __nv_bfloat16* xin, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  if (n & 127) return cudaErrorInvalidValue;
  euler_step_kernel<<<grid_for(n), kThreads, 0, st>>>(x, vc, vu, n, dt, guidance, xin);
  return cudaGetLastError();
}

cudaError_t launch_euler_cfg(float* x, const float* v, int64_t per_sample, int B, bool cfg, float dt,
                             float guidance, __nv_bfloat16* xin, cudaStream_t st) {
  const int64_t n = per_sample * B;
  euler_cfg_kernel<<<grid_for(n), kThreads, 0, st>>>(x, v, n, n, cfg ? 1 : 0, dt, guidance, xin);
  return cudaGetLastError();
}
cudaError_t launch_euler_plain(float* x, const float* vc, const float* vu, int64_t n, float dt, float guidance,
                               cudaStream_t st) {
  euler_plain_kernel<<<grid_for(n), kThreads, 0, st>>>(x, vc, vu, n, dt, guidance);
  return cudaGetLastError();
}

}  // namespace lens
