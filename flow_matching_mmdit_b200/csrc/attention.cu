// Joint attention over the concatenated [text; image] sequence of one MMDiT block
// (MLX port article, "双流注意力机制": the two streams attend jointly; survey page,
// "交叉注意力与条件注入": one concatenated sequence).  Per (batch, head):
//   O = softmax(Q K^T / sqrt(64)) V, no mask, N = n_txt + n_img tokens.
//
// Flash-style single pass on the tcgen05 tensor cores (layout below): scores and the
// output accumulate in TMEM, the running row max and sum live in registers of the
// softmax warps, base-2 exponentials carry the 1/8 scale.  Keys past N are masked;
// rows past N are computed on zero-filled queries and never stored.
#include "gemm.h"
#include "kernels.cuh"

namespace lens {

namespace {

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ============================================================ tcgen05 version
// One CTA per (128 query rows, head, batch row); warp roles (192 threads):
//   warp 0      TMA: Q tile once, then K and V tiles of 128 keys into a 3-stage ring
//   warp 1      UMMA issuer: S_j = Q K_j^T (M=128, N=128, K=64) into one of two TMEM
//               S buffers, and O += P_{j-1} V_{j-1} (M=128, N=64, K=128) into TMEM
//   warps 2..5  softmax: one query row per thread; reads S_j from TMEM, keeps the
//               running max m and sum l in registers, writes P_j (bf16) to shared
//               memory as the K-major A operand, and rescales the O row in TMEM
//               when m grows by more than 2^8 (otherwise the stale max is kept:
//               softmax is invariant to the subtracted constant)
// TMEM columns: S buffers [0,128) and [128,256); O [256,320).
namespace tc {

constexpr int BQ = 128, BKV = 128, STAGES = 3;
constexpr uint32_t Q_BYTES = BQ * 64 * 2;          // 16 KB
constexpr uint32_t KV_BYTES = BKV * 64 * 2;        // 16 KB each for K and V
constexpr uint32_t P_BYTES = BQ * BKV * 2;         // 32 KB: two 64-key swizzle atoms
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_KV = OFF_Q + Q_BYTES;
constexpr uint32_t OFF_P = OFF_KV + STAGES * 2 * KV_BYTES;
constexpr uint32_t OFF_BAR = OFF_P + P_BYTES;
constexpr size_t SMEM = 1024 + OFF_BAR + 256;
constexpr float kRescaleThreshold = 8.0f;          // log2 units

__global__ void __launch_bounds__(192, 1)
    joint_attention_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                              const __grid_constant__ CUtensorMap tmV, int N, int n_txt, int heads,
                              __nv_bfloat16* __restrict__ out_txt, __nv_bfloat16* __restrict__ out_img,
                              float scale_log2, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = sm + OFF_Q;
  uint8_t* sKV = sm + OFF_KV;
  uint8_t* sP = sm + OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + STAGES;
  uint64_t* s_full = kv_empty + STAGES;   // [2]
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pv_done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, h = blockIdx.y;
  const int bh = b * heads + h;
  const int q0 = blockIdx.x * BQ;
  const int nkv = (N + BKV - 1) / BKV;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t last_parity[STAGES];
      bool issued[STAGES] = {false, false, false};
      bool ok = true;
      mbar_expect_tx(q_full, Q_BYTES);
      tma_load_3d(sQ, &tmQ, q_full, 0, q0, bh);
      for (int j = 0; j < nkv; ++j) {
        const int s = j % STAGES;
        const uint32_t ph = (j / STAGES) & 1;
        if (!mbar_wait(&kv_empty[s], ph ^ 1, err)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&kv_full[s], 2 * KV_BYTES);
        tma_load_3d(sKV + s * 2 * KV_BYTES, &tmK, &kv_full[s], 0, j * BKV, bh);
        tma_load_3d(sKV + s * 2 * KV_BYTES + KV_BYTES, &tmV, &kv_full[s], 0, j * BKV, bh);
        issued[s] = true;
        last_parity[s] = ph;
      }
      mbar_wait_drain(q_full, 0);
      if (!ok)
        for (int s = 0; s < STAGES; ++s)
          if (issued[s]) mbar_wait_drain(&kv_full[s], last_parity[s]);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(128, BKV);
      constexpr uint32_t idesc_pv = umma_idesc_bf16_bmn(128, 64);
      bool ok = mbar_wait(q_full, 0, err);
      tc_fence_after();
      const uint64_t qdesc = umma_desc_sw128(smem_u32(sQ));
      for (int j = 0; ok && j <= nkv; ++j) {
        if (j < nkv) {
          const int s = j % STAGES;
          if (!mbar_wait(&kv_full[s], (j / STAGES) & 1, err)) break;
          tc_fence_after();
          const uint64_t kdesc = umma_desc_sw128(smem_u32(sKV + s * 2 * KV_BYTES));
          const uint32_t d = tmem + (j & 1) * 128;
#pragma unroll
          for (int k = 0; k < 4; ++k) umma_bf16(d, qdesc + 2 * k, kdesc + 2 * k, idesc_s, k > 0 ? 1u : 0u);
          umma_commit(&s_full[j & 1]);
        }
        if (j >= 1) {
          const int jj = j - 1;
          if (!mbar_wait(p_full, jj & 1, err)) break;
          tc_fence_after();
          const int s = jj % STAGES;
          const uint32_t pbase = smem_u32(sP);
          const uint32_t vbase = smem_u32(sKV + s * 2 * KV_BYTES + KV_BYTES);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t pdesc = umma_desc_sw128(pbase + (k >> 2) * (BQ * 128) + (k & 3) * 32);
            const uint64_t vdesc = umma_desc_sw128_mn(vbase + k * 2048);
            umma_bf16(tmem + 256, pdesc, vdesc, idesc_pv, (jj > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&kv_empty[s]);
          umma_commit(pv_done);
        }
      }
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + (uint32_t(quarter * 32) << 16);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!mbar_wait(&s_full[j & 1], (j >> 1) & 1, err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sc[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(lane_addr + (j & 1) * 128 + c * 32, *reinterpret_cast<float(*)[32]>(&sc[32 * c]));
      tmem_ld_wait();
      if ((j + 1) * BKV > N) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (j * BKV + i >= N) sc[i] = -INFINITY;
      }
      float mx = sc[0];
#pragma unroll
      for (int i = 1; i < 128; ++i) mx = fmaxf(mx, sc[i]);
      mx *= scale_log2;
      float corr = 1.f;
      if (mx > m + kRescaleThreshold) {
        corr = ex2(m - mx);
        m = mx;
      }
      float rs = 0.f;
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        sc[i] = ex2(fmaf(sc[i], scale_log2, -m));
        rs += sc[i];
      }
      l = l * corr + rs;
      if (j > 0) {
        if (!mbar_wait(pv_done, (j - 1) & 1, err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, corr != 1.f)) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            float o[32];
            tmem_ld32(lane_addr + 256 + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= corr;
            tmem_st32(lane_addr + 256 + c * 32, o);
          }
          tmem_st_wait();
        }
      }
      // P row r -> two 64-key atoms, 128-byte swizzle (16-byte chunk c of the row
      // goes to position c ^ (r & 7))
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint32_t addr = smem_u32(sP) + (c >> 3) * (BQ * 128) + r * 128 + ((((c & 7) ^ (r & 7))) << 4);
        const uint32_t w0 = pack_bf16x2(sc[8 * c + 0], sc[8 * c + 1]);
        const uint32_t w1 = pack_bf16x2(sc[8 * c + 2], sc[8 * c + 3]);
        const uint32_t w2 = pack_bf16x2(sc[8 * c + 4], sc[8 * c + 5]);
        const uint32_t w3 = pack_bf16x2(sc[8 * c + 6], sc[8 * c + 7]);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w0), "r"(w1), "r"(w2), "r"(w3)
                     : "memory");
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok && mbar_wait(pv_done, (nkv - 1) & 1, err)) {
      tc_fence_after();
      float o0[32], o1[32];
      tmem_ld32(lane_addr + 256, o0);
      tmem_ld32(lane_addr + 256 + 32, o1);
      tmem_ld_wait();
      const int tok = q0 + r;
      if (tok < N) {
        const float inv = 1.f / l;
        const int hid = heads * 64;
        __nv_bfloat16* dst = tok < n_txt ? out_txt + ((int64_t)b * n_txt + tok) * hid
                                         : out_img + ((int64_t)b * (N - n_txt) + (tok - n_txt)) * hid;
        uint4* d4 = reinterpret_cast<uint4*>(dst + h * 64);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          d4[j] = make_uint4(pack_bf16x2(o0[8 * j] * inv, o0[8 * j + 1] * inv),
                             pack_bf16x2(o0[8 * j + 2] * inv, o0[8 * j + 3] * inv),
                             pack_bf16x2(o0[8 * j + 4] * inv, o0[8 * j + 5] * inv),
                             pack_bf16x2(o0[8 * j + 6] * inv, o0[8 * j + 7] * inv));
#pragma unroll
        for (int j = 0; j < 4; ++j)
          d4[4 + j] = make_uint4(pack_bf16x2(o1[8 * j] * inv, o1[8 * j + 1] * inv),
                                 pack_bf16x2(o1[8 * j + 2] * inv, o1[8 * j + 3] * inv),
                                 pack_bf16x2(o1[8 * j + 4] * inv, o1[8 * j + 5] * inv),
                                 pack_bf16x2(o1[8 * j + 6] * inv, o1[8 * j + 7] * inv));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc
}  // namespace

cudaError_t launch_joint_attention(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, int B,
                                   int heads, int n_txt, int n_img, __nv_bfloat16* out_txt, __nv_bfloat16* out_img,
                                   int* err, cudaStream_t st) {
  const int N = n_txt + n_img;
  if (N <= 0 || B <= 0) return cudaSuccess;
  // [B*heads, N, 64] views: tiles of 128 rows never cross into the next head, and
  // rows past N read as zeros
  CUtensorMap tq, tk, tv;
  if (!encode_tmap_bf16_3d(&tq, q, 64, N, (uint64_t)B * heads, 128) ||
      !encode_tmap_bf16_3d(&tk, k, 64, N, (uint64_t)B * heads, 128) ||
      !encode_tmap_bf16_3d(&tv, v, 64, N, (uint64_t)B * heads, 128))
    return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(tc::joint_attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tc::SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dim3 grid((N + tc::BQ - 1) / tc::BQ, heads, B);
  const float scale_log2 = 0.125f * 1.4426950408889634f;
  tc::joint_attention_tc_kernel<<<grid, 192, tc::SMEM, st>>>(tq, tk, tv, N, n_txt, heads, out_txt, out_img,
                                                            scale_log2, err);
  return cudaGetLastError();
}

}  // namespace lens
