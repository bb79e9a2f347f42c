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
#include "smem_attr.h"

namespace lens {

namespace {

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


// Packed fp32 pairs (Blackwell f32x2 arithmetic): one instruction for two lanes
// of the softmax's scale-and-shift and running sums.
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// three-input maximum (one instruction on sm_100)
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// ============================================================ tcgen05 version
// One CTA per (256 query rows = two 128-row tiles X = 0, 1; head; batch row).
// Warp roles (320 threads):
//   warps 0..3  softmax of tile 0, warps 4..7 softmax of tile 1: one query row per
//               thread; S_X is read from TMEM into registers and released at once,
//               so the tensor cores compute S_X for the next keys while this tile's
//               exponentials run, and the two tiles ping-pong on the tensor cores
//   warp 8      TMA: both Q tiles once, then K and V tiles of 128 keys (3 stages)
//   warp 9      UMMA issuer: S_X = Q_X K_j^T (M=128, N=128, K=64) and
//               O_X += P_X V_j (M=128, N=64, K=128) with P_X read from TMEM.
//               A wait in this thread stalls until its queued UMMAs are accepted,
//               so the waits S_0 and S_1 need (K/V stage, both S slots released)
//               are taken back to back: the queue drains once for them.
// The running max m and sum l of each row live in registers; O_X is rescaled in
// TMEM only when m grows by more than 2^8 (softmax is invariant to the subtracted
// constant, so a stale max is exact up to rounding).
// P_X goes from the softmax registers into TMEM (two bf16 per column) and is the A
// operand of P V there, so neither P nor its operand reads touch shared memory.
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,320), O_1 [320,384),
// P_0 [384,448), P_1 [448,512).
namespace tc {

constexpr int BQ = 128, BKV = 128, STAGES = 3, TILES = 2;
constexpr int THREADS = 320;
constexpr uint32_t Q_BYTES = BQ * 64 * 2;          // 16 KB per query tile
constexpr uint32_t KV_BYTES = BKV * 64 * 2;        // 16 KB each for K and V
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_KV = OFF_Q + TILES * Q_BYTES;
constexpr uint32_t OFF_BAR = OFF_KV + STAGES * 2 * KV_BYTES;
constexpr size_t SMEM = 1024 + OFF_BAR + 256;
constexpr float kRescaleThreshold = 8.0f;          // log2 units

struct Bars {
  uint64_t q_full;
  uint64_t kv_full[STAGES];
  uint64_t kv_empty[STAGES];
  uint64_t s_full[TILES];    // MMA -> softmax: S_X ready
  uint64_t s_free[TILES];    // softmax -> MMA: S_X read into registers
  uint64_t p_full[TILES];    // softmax -> MMA: P_X written, O_X rescaled
  uint64_t pv_done[TILES];   // MMA -> softmax: O_X += P_X V finished
  uint32_t tmem_slot;
};

__global__ void __launch_bounds__(THREADS, 1)
    joint_attention_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                              const __grid_constant__ CUtensorMap tmV, int N, int n_txt, int heads,
                              __nv_bfloat16* __restrict__ out_txt, __nv_bfloat16* __restrict__ out_img,
                              float scale_log2, const TextLengths txt_len, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = sm + OFF_Q;
  uint8_t* sKV = sm + OFF_KV;
  Bars& bar = *reinterpret_cast<Bars*>(sm + OFF_BAR);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, h = blockIdx.y;
  const int bh = b * heads + h;
  const int q0 = blockIdx.x * (TILES * BQ);
  const int nkv = (N + BKV - 1) / BKV;
  // text keys [txt_valid, n_txt) of this batch row are padding and never attended
  const int txt_valid = txt_len.n[b] < n_txt ? txt_len.n[b] : n_txt;
  const int txt_pad_end = n_txt;

  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bar.kv_full[s], 1);
      mbar_init(&bar.kv_empty[s], 1);
    }
    for (int x = 0; x < TILES; ++x) {
      mbar_init(&bar.s_full[x], 1);
      mbar_init(&bar.s_free[x], 4);
      mbar_init(&bar.p_full[x], 4);
      mbar_init(&bar.pv_done[x], 1);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 9) {
    tmem_alloc(&bar.tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_slot;

  if (warp == 8) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      uint32_t last_parity[STAGES] = {0, 0, 0};
      bool issued[STAGES] = {false, false, false};
      bool ok = true;
      mbar_expect_tx(&bar.q_full, TILES * Q_BYTES);
      for (int x = 0; x < TILES; ++x) tma_load_3d(sQ + x * Q_BYTES, &tmQ, &bar.q_full, 0, q0 + x * BQ, bh);
      for (int j = 0; j < nkv; ++j) {
        const int s = j % STAGES;
        const uint32_t ph = (j / STAGES) & 1;
        if (!mbar_wait(&bar.kv_empty[s], ph ^ 1, err)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&bar.kv_full[s], 2 * KV_BYTES);
        tma_load_3d(sKV + s * 2 * KV_BYTES, &tmK, &bar.kv_full[s], 0, j * BKV, bh);
        tma_load_3d(sKV + s * 2 * KV_BYTES + KV_BYTES, &tmV, &bar.kv_full[s], 0, j * BKV, bh);
        issued[s] = true;
        last_parity[s] = ph;
      }
      mbar_wait_drain(&bar.q_full, 0);
      if (!ok)
        for (int s = 0; s < STAGES; ++s)
          if (issued[s]) mbar_wait_drain(&bar.kv_full[s], last_parity[s]);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---------------------------------------------------------------- UMMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(128, BKV);
      constexpr uint32_t idesc_pv = umma_idesc_bf16_bmn(128, 64);
      bool ok = mbar_wait(&bar.q_full, 0, err);
      tc_fence_after();
      for (int j = 0; ok && j <= nkv; ++j) {
        if (j < nkv) {
          const int s = j % STAGES;
          // every wait S_0[j] and S_1[j] need, back to back: only the first drains the queue
          ok = mbar_wait(&bar.kv_full[s], (j / STAGES) & 1, err) &&
               (j == 0 || (mbar_wait(&bar.s_free[0], (j - 1) & 1, err) && mbar_wait(&bar.s_free[1], (j - 1) & 1, err)));
          if (!ok) break;
          tc_fence_after();
          const uint64_t kdesc = umma_desc_sw128(smem_u32(sKV + s * 2 * KV_BYTES));
#pragma unroll
          for (int x = 0; x < TILES; ++x) {
            const uint64_t qdesc = umma_desc_sw128(smem_u32(sQ + x * Q_BYTES));
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_bf16(tmem + x * 128, qdesc + 2 * k, kdesc + 2 * k, idesc_s, k > 0 ? 1u : 0u);
            umma_commit(&bar.s_full[x]);
          }
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int s = jj % STAGES;
          const uint32_t vbase = smem_u32(sKV + s * 2 * KV_BYTES + KV_BYTES);
#pragma unroll
          for (int x = 0; x < TILES; ++x) {
            if (!mbar_wait(&bar.p_full[x], jj & 1, err)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k) {              // 16 keys = 8 TMEM columns of P per step
              const uint64_t vdesc = umma_desc_sw128_mn(vbase + k * 2048);
              umma_bf16_ts(tmem + 256 + x * 64, tmem + 384 + x * 64 + 8 * k, vdesc, idesc_pv,
                           (jj > 0 || k > 0) ? 1u : 0u);
            }
            umma_commit(&bar.pv_done[x]);
          }
          if (!ok) break;
          umma_commit(&bar.kv_empty[s]);
        }
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax
    const int x = warp >> 2;                // query tile
    const int quarter = warp & 3;           // TMEM lane quarter
    const int r = quarter * 32 + lane;      // row inside the tile
    const uint32_t lane_addr = tmem + (uint32_t(quarter * 32) << 16);
    const uint32_t s_col = x * 128, o_col = 256 + x * 64, p_col = 384 + x * 64;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!mbar_wait(&bar.s_full[x], j & 1, err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sc[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(lane_addr + s_col + c * 32, *reinterpret_cast<float(*)[32]>(&sc[32 * c]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.s_free[x]);     // S_X may be overwritten now
      if ((j + 1) * BKV > N) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (j * BKV + i >= N) sc[i] = -INFINITY;
      }
      if (j * BKV < txt_pad_end && (j + 1) * BKV > txt_valid) {   // padded text keys of this sample
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (j * BKV + i >= txt_valid && j * BKV + i < txt_pad_end) sc[i] = -INFINITY;
      }
      // 8 independent partial maxima (three-input max) keep the dependency chains short
      float pm[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        pm[q] = max3f(sc[q], sc[q + 8], sc[q + 16]);
#pragma unroll
        for (int t = 3; t < 15; t += 2) pm[q] = max3f(pm[q], sc[q + 8 * t], sc[q + 8 * t + 8]);
        pm[q] = fmaxf(pm[q], sc[q + 120]);
      }
      float mx = max3f(max3f(pm[0], pm[1], pm[2]), max3f(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
      mx *= scale_log2;
      float corr = 1.f;
      if (mx > m + kRescaleThreshold) {
        corr = ex2(m - mx);
        m = mx;
      }
      // every key seen so far masked: m is still -inf and so is every score here
      const float m_base = m == -INFINITY ? 0.f : m;
      uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
      // x = s log2(e) / 8 - m for two keys per instruction
      const uint64_t sl2 = f2_pack(scale_log2, scale_log2), mb2 = f2_pack(-m_base, -m_base);
      uint32_t pk[64];
#pragma unroll
      for (int i = 0; i < 128; i += 2) {
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(sc[i], sc[i + 1]), sl2, mb2), x0, x1);
        const float e0 = ex2(x0), e1 = ex2(x1);
        acc2[(i >> 1) & 3] = f2_add(acc2[(i >> 1) & 3], f2_pack(e0, e1));
        pk[i >> 1] = pack_bf16x2(e0, e1);
      }
      float ps[8];
      f2_unpack(acc2[0], ps[0], ps[1]);
      f2_unpack(acc2[1], ps[2], ps[3]);
      f2_unpack(acc2[2], ps[4], ps[5]);
      f2_unpack(acc2[3], ps[6], ps[7]);
      const float rs = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      l = l * corr + rs;
      if (j > 0) {
        if (!mbar_wait(&bar.pv_done[x], (j - 1) & 1, err)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      // P row r -> TMEM, column c = keys (2c, 2c + 1)
      tmem_st32_u(lane_addr + p_col, pk);
      tmem_st32_u(lane_addr + p_col + 32, pk + 32);
      if (j > 0 && __any_sync(0xffffffffu, corr != 1.f)) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float o[32];
          tmem_ld32(lane_addr + o_col + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= corr;
          tmem_st32(lane_addr + o_col + c * 32, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.p_full[x]);
    }
    if (ok && mbar_wait(&bar.pv_done[x], (nkv - 1) & 1, err)) {
      tc_fence_after();
      float o0[32], o1[32];
      tmem_ld32(lane_addr + o_col, o0);
      tmem_ld32(lane_addr + o_col + 32, o1);
      tmem_ld_wait();
      const int tok = q0 + x * BQ + r;
      if (tok < N) {
        const float inv = 1.f / l;
        const int hid = heads * 64;
        __nv_bfloat16* dst = tok < n_txt ? out_txt + ((int64_t)b * n_txt + tok) * hid
                                         : out_img + ((int64_t)b * (N - n_txt) + (tok - n_txt)) * hid;
        uint4* d4 = reinterpret_cast<uint4*>(dst + h * 64);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          d4[q] = make_uint4(pack_bf16x2(o0[8 * q] * inv, o0[8 * q + 1] * inv),
                             pack_bf16x2(o0[8 * q + 2] * inv, o0[8 * q + 3] * inv),
                             pack_bf16x2(o0[8 * q + 4] * inv, o0[8 * q + 5] * inv),
                             pack_bf16x2(o0[8 * q + 6] * inv, o0[8 * q + 7] * inv));
#pragma unroll
        for (int q = 0; q < 4; ++q)
          d4[4 + q] = make_uint4(pack_bf16x2(o1[8 * q] * inv, o1[8 * q + 1] * inv),
                                 pack_bf16x2(o1[8 * q + 2] * inv, o1[8 * q + 3] * inv),
                                 pack_bf16x2(o1[8 * q + 4] * inv, o1[8 * q + 5] * inv),
                                 pack_bf16x2(o1[8 * q + 6] * inv, o1[8 * q + 7] * inv));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc

}  // namespace

cudaError_t launch_joint_attention(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, int B,
                                   int heads, int n_txt, int n_img, __nv_bfloat16* out_txt, __nv_bfloat16* out_img,
                                   const TextLengths* txt_len, int* err, cudaStream_t st) {
  const int N = n_txt + n_img;
  if (N <= 0 || B <= 0) return cudaSuccess;
  if (B > kMaxRows) return cudaErrorInvalidValue;
  TextLengths lens;
  for (int b = 0; b < kMaxRows; ++b) lens.n[b] = (txt_len && b < B) ? txt_len->n[b] : n_txt;
  // [B*heads, N, 64] views: tiles of 128 rows never cross into the next head, and
  // rows past N read as zeros
  CUtensorMap tq, tk, tv;
  if (!encode_tmap_bf16_3d(&tq, q, 64, N, (uint64_t)B * heads, 128) ||
      !encode_tmap_bf16_3d(&tk, k, 64, N, (uint64_t)B * heads, 128) ||
      !encode_tmap_bf16_3d(&tv, v, 64, N, (uint64_t)B * heads, 128))
    return cudaErrorInvalidValue;
  static std::atomic<uint64_t> attr{0};
  {
    const cudaError_t e = ensure_smem_limit(tc::joint_attention_tc_kernel, (int)tc::SMEM, attr);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((N + tc::TILES * tc::BQ - 1) / (tc::TILES * tc::BQ), heads, B);
  const float scale_log2 = 0.125f * 1.4426950408889634f;
  tc::joint_attention_tc_kernel<<<grid, tc::THREADS, tc::SMEM, st>>>(tq, tk, tv, N, n_txt, heads, out_txt, out_img,
                                                                        scale_log2, lens, err);
  return cudaGetLastError();
}

}  // namespace lens
