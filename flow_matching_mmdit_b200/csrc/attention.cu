// Joint attention over the concatenated [text; image] sequence of one MMDiT block
// (MLX port article, "双流注意力机制": the two streams attend jointly; survey page,
// "交叉注意力与条件注入": one concatenated sequence).  Per (batch, head):
//   O = softmax(Q K^T / sqrt(64)) V, no mask, N = n_txt + n_img tokens.
//
// Flash-style single pass: a CTA owns 128 query rows (8 warps x 16 rows) and streams
// 64-key K/V tiles through a double-buffered, XOR-swizzled shared-memory ring filled
// by cp.async.  Scores and the running output live in registers; the row max and
// sum use base-2 exponentials with the 1/8 scale folded in.  Keys past N are masked;
// rows past N are computed on zero-filled queries and never stored.
#include "kernels.cuh"

namespace lens {

namespace {

constexpr int kBQ = 128;
constexpr int kBK = 64;
constexpr int kWarps = 8;

__device__ __forceinline__ uint32_t swz(int row, int chunk) {   // byte offset inside a [rows][128 B] tile
  return uint32_t(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Load a [rows][64] bf16 tile (rows from `row0`, clipped at `n_rows`) into swizzled smem.
template <int ROWS>
__device__ __forceinline__ void load_tile(uint32_t sbase, const __nv_bfloat16* g, int row0, int n_rows) {
  constexpr int kChunks = ROWS * 8;
#pragma unroll
  for (int i = threadIdx.x; i < kChunks; i += kWarps * 32) {
    const int r = i >> 3, c = i & 7;
    const int gr = row0 + r;
    const bool ok = gr < n_rows;
    const __nv_bfloat16* src = g + (int64_t)(ok ? gr : 0) * 64 + c * 8;
    cp_async16(sbase + swz(r, c), src, ok);
  }
}

__global__ void __launch_bounds__(kWarps * 32) joint_attention_mma_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    int N, int n_txt, int heads, __nv_bfloat16* __restrict__ out_txt, __nv_bfloat16* __restrict__ out_img,
    float scale_log2) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK = sQ + kBQ * 128;              // 2 buffers of kBK x 128 B
  const uint32_t sV = sK + 2 * kBK * 128;

  const int b = blockIdx.z, h = blockIdx.y;
  const int q0 = blockIdx.x * kBQ;
  const int64_t head_off = ((int64_t)b * heads + h) * N * 64;
  const __nv_bfloat16* Qg = q + head_off;
  const __nv_bfloat16* Kg = k + head_off;
  const __nv_bfloat16* Vg = v + head_off;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;

  const int nkt = (N + kBK - 1) / kBK;
  load_tile<kBQ>(sQ, Qg, q0, N);
  load_tile<kBK>(sK, Kg, 0, N);
  load_tile<kBK>(sV, Vg, 0, N);
  cp_async_commit();

  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  uint32_t qa[4][4];

  for (int j = 0; j < nkt; ++j) {
    const int buf = j & 1;
    if (j + 1 < nkt) {
      load_tile<kBK>(sK + (buf ^ 1) * kBK * 128, Kg, (j + 1) * kBK, N);
      load_tile<kBK>(sV + (buf ^ 1) * kBK * 128, Vg, (j + 1) * kBK, N);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (j == 0) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = 2 * kk + (lane >> 4);
        ldsm_x4(sQ + swz(r, c), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
      }
    }
    const uint32_t kb = sK + buf * kBK * 128, vb = sV + buf * kBK * 128;

    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        uint32_t r0, r1, r2, r3;
        const int r = 16 * p + (lane & 7) + ((lane >> 4) << 3);
        const int c = 2 * kk + ((lane >> 3) & 1);
        ldsm_x4(kb + swz(r, c), r0, r1, r2, r3);
        mma_bf16_16816(s[2 * p], qa[kk], r0, r1);
        mma_bf16_16816(s[2 * p + 1], qa[kk], r2, r3);
      }
    }
    if ((j + 1) * kBK > N) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int key = j * kBK + nt * 8 + 2 * t4;
        if (key >= N) s[nt][0] = s[nt][2] = -INFINITY;
        if (key + 1 >= N) s[nt][1] = s[nt][3] = -INFINITY;
      }
    }
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
      mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0 * scale_log2), mn1 = fmaxf(m1, mx1 * scale_log2);
    const float c0 = ex2(m0 - mn0), c1 = ex2(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      s[nt][0] = ex2(s[nt][0] * scale_log2 - mn0);
      s[nt][1] = ex2(s[nt][1] * scale_log2 - mn0);
      s[nt][2] = ex2(s[nt][2] * scale_log2 - mn1);
      s[nt][3] = ex2(s[nt][3] * scale_log2 - mn1);
      rs0 += s[nt][0] + s[nt][1];
      rs1 += s[nt][2] + s[nt][3];
      o[nt][0] *= c0;
      o[nt][1] *= c0;
      o[nt][2] *= c1;
      o[nt][3] *= c1;
    }
    l0 = l0 * c0 + rs0;
    l1 = l1 * c1 + rs1;

#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int qd = 0; qd < 4; ++qd) {
        uint32_t r0, r1, r2, r3;
        const int r = 16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int c = 2 * qd + (lane >> 4);
        ldsm_x4_t(vb + swz(r, c), r0, r1, r2, r3);
        mma_bf16_16816(o[2 * qd], pa, r0, r1);
        mma_bf16_16816(o[2 * qd + 1], pa, r2, r3);
      }
    }
    __syncthreads();
  }

  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float i0 = 1.f / l0, i1 = 1.f / l1;
  const int n_img = N - n_txt;
  const int hid = heads * 64;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int tok = q0 + warp * 16 + g + half * 8;
    if (tok >= N) continue;
    __nv_bfloat16* dst = tok < n_txt ? out_txt + ((int64_t)b * n_txt + tok) * hid
                                     : out_img + ((int64_t)b * n_img + (tok - n_txt)) * hid;
    dst += h * 64 + 2 * t4;
    const float inv = half ? i1 : i0;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const uint32_t w = pack_bf16x2(o[nt][2 * half] * inv, o[nt][2 * half + 1] * inv);
      *reinterpret_cast<uint32_t*>(dst + nt * 8) = w;
    }
  }
}

}  // namespace

cudaError_t launch_joint_attention(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, int B,
                                   int heads, int n_txt, int n_img, __nv_bfloat16* out_txt, __nv_bfloat16* out_img,
                                   cudaStream_t st) {
  const int N = n_txt + n_img;
  if (N <= 0 || B <= 0) return cudaSuccess;
  const size_t smem = kBQ * 128 + 4 * kBK * 128;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(joint_attention_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dim3 grid((N + kBQ - 1) / kBQ, heads, B);
  const float scale_log2 = 0.125f * 1.4426950408889634f;
  joint_attention_mma_kernel<<<grid, kWarps * 32, smem, st>>>(q, k, v, N, n_txt, heads, out_txt, out_img,
                                                              scale_log2);
  return cudaGetLastError();
}

}  // namespace lens
