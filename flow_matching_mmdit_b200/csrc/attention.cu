// Joint attention over the concatenated [text; image] sequence of one MMDiT block
// (MLX port article, "双流注意力机制": the two streams attend jointly; survey page,
// "交叉注意力与条件注入": one concatenated sequence).  Per (batch, head):
//   O = softmax(Q K^T / sqrt(64)) V, no mask, N = n_txt + n_img tokens.
//
// Flash-style single pass on the tcgen05 tensor cores (layout below): scores and the
// output accumulate in TMEM, the running row max and sum live in registers of the
// softmax warps, base-2 exponentials carry the 1/8 scale.  Keys past N are masked;
// rows past N are computed on zero-filled queries and never stored.
#include "exp2_poly.h"
#include "gemm.h"
#include "kernels.cuh"
#include "smem_attr.h"

// Which of each thread's 16 groups of four scores per key tile take their
// exponentials on the FMA pipe (bit g set) instead of the exponential unit.
#ifndef LENS_ATTN_EMU_MASK
#define LENS_ATTN_EMU_MASK 0x0000u
#endif

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
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x0, 2^x1 of a packed pair on the FMA pipe: exp2_poly (exp2_poly.h) step by step
// on fp32 pairs, with the clamp and the exponent add on the integer side.
__device__ __forceinline__ void exp2_fma_pair(uint64_t x, float& a, float& b) {
  float x0, x1;
  f2_unpack(x, x0, x1);
  const uint64_t xc = f2_pack(fmaxf(x0, kExp2Floor), fmaxf(x1, kExp2Floor));
  const uint64_t t = f2_add(xc, f2_pack(kExp2Round, kExp2Round));
  const uint64_t f = f2_sub(xc, f2_sub(t, f2_pack(kExp2Round, kExp2Round)));
  uint64_t p = f2_fma(f, f2_pack(kExp2C3, kExp2C3), f2_pack(kExp2C2, kExp2C2));
  p = f2_fma(p, f, f2_pack(kExp2C1, kExp2C1));
  p = f2_fma(p, f, f2_pack(kExp2C0, kExp2C0));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  a = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  b = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

// three-input maximum (one instruction on sm_100)
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}


// ============================================================ tcgen05 version
// One CTA per (256 query rows = two 128-row tiles X = 0, 1; head; batch row).
// Warp roles (608 threads):
//   warps 0..15 softmax, eight warps per tile (X = warp / 8): warp (quarter q, half
//               h) owns TMEM lanes 32q + 16h + [0, 16) and reads S_X with the
//               16-lane shape, so each thread holds two query rows (r and r + 8) and
//               32 of the 128 keys of each, and the four threads of a row combine
//               their maxima with two shuffles.  Four softmax warps per SMSP and 64
//               scores per thread (not 128) leave room to hide the exponential and
//               TMEM latencies.  S_X is released as soon as it is in registers, so
//               the tensor cores compute S_X for the next keys meanwhile.
//   warp 16     TMA: both Q tiles once, then K and V tiles of 128 keys (3 stages)
//   warp 17     S issuer: S_X = Q_X K_j^T (M=128, N=128, K=64), each tile as soon
//               as its S slot is released
//   warp 18     P V issuer: O_X += P_X V_j (M=128, N=64, K=128) with P_X in TMEM.
//               A wait in an issuing thread stalls until that thread's queued UMMAs
//               are accepted, so the two kinds of MMA come from two threads: a P V
//               wait does not hold back the next S, nor the reverse.
// Tile 1 starts its first exponentials only when tile 0 has finished its own: the
// two tiles then keep alternating on the exponential unit instead of contending
// for it in phase.
// The running max m and sum l of each row live in registers; O_X is rescaled in
// TMEM only when m grows by more than 2^8 (softmax is invariant to the subtracted
// constant, so a stale max is exact up to rounding).
// P_X goes from the softmax registers into TMEM (two bf16 per column) and is the A
// operand of P V there, so neither P nor its operand reads touch shared memory.
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,320), O_1 [320,384),
// P_0 [384,448), P_1 [448,512).
namespace tc {

constexpr int BQ = 128, BKV = 128, STAGES = 3, TILES = 2;
constexpr int THREADS = 608;
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
  uint64_t stagger;          // tile 0 -> tile 1: tile 0 finished its first exponentials
  uint64_t drain[2];         // each MMA issuer's own completion after an abort
  uint32_t tmem_slot;
};

static_assert(sizeof(Bars) <= 256, "barriers overflow their shared-memory reserve");

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
      mbar_init(&bar.kv_empty[s], 2);
    }
    for (int x = 0; x < TILES; ++x) {
      mbar_init(&bar.s_full[x], 1);
      mbar_init(&bar.s_free[x], 8);
      mbar_init(&bar.p_full[x], 8);
      mbar_init(&bar.pv_done[x], 1);
    }
    mbar_init(&bar.stagger, 8);
    mbar_init(&bar.drain[0], 1);
    mbar_init(&bar.drain[1], 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 17) {
    tmem_alloc(&bar.tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_slot;
  grid_dependency_sync();    // set-up above touched only shared memory and TMEM

  if (warp == 16) {
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
      // after an abort the consumers may not have waited for every stage filled here
      if (!ok || err_raised(err))
        for (int s = 0; s < STAGES; ++s)
          if (issued[s]) mbar_wait_drain(&bar.kv_full[s], last_parity[s]);
    }
    __syncwarp();
  } else if (warp == 17) {
    // ---------------------------------------------------------------- S issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(128, BKV);
      bool ok = mbar_wait(&bar.q_full, 0, err);
      tc_fence_after();
      for (int j = 0; ok && j < nkv; ++j) {
        const int s = j % STAGES;
        ok = mbar_wait(&bar.kv_full[s], (j / STAGES) & 1, err);
        if (!ok) break;
        const uint64_t kdesc = umma_desc_sw128(smem_u32(sKV + s * 2 * KV_BYTES));
#pragma unroll
        for (int x = 0; x < TILES; ++x) {
          if (j > 0 && !mbar_wait(&bar.s_free[x], (j - 1) & 1, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t qdesc = umma_desc_sw128(smem_u32(sQ + x * Q_BYTES));
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tmem + x * 128, qdesc + 2 * k, kdesc + 2 * k, idesc_s, k > 0 ? 1u : 0u);
          umma_commit(&bar.s_full[x]);
        }
        if (!ok) break;
        umma_commit(&bar.kv_empty[s]);
      }
      if (!ok) umma_drain(&bar.drain[0]);   // no S MMA still runs when TMEM is freed
    }
    __syncwarp();
  } else if (warp == 18) {
    // ---------------------------------------------------------------- P V issuer
    if (lane == 0) {
      constexpr uint32_t idesc_pv = umma_idesc_bf16_bmn(128, 64);
      bool ok = true;
      for (int jj = 0; ok && jj < nkv; ++jj) {
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
          for (int k = 0; k < 8; ++k) {
            const uint64_t vdesc = umma_desc_sw128_mn(vbase + k * 2048);
            umma_bf16_ts(tmem + 256 + x * 64, tmem + 384 + x * 64 + 8 * k, vdesc, idesc_pv,
                         (jj > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&bar.pv_done[x]);
        }
        if (!ok) break;
        umma_commit(&bar.kv_empty[s]);
      }
      if (!ok) umma_drain(&bar.drain[1]);   // no P V MMA still runs when TMEM is freed
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax
    // Eight warps per tile: warp (quarter, half) reads TMEM lanes quarter*32 + half*16
    // + [0, 16); each thread holds rows rlo and rlo + 8, 32 of the 128 keys of each
    // (columns 8g + cq + {0, 1}); the four threads of a row combine maxima by shuffles.
    const int x = warp >> 3;
    const int half = (warp >> 2) & 1;
    const int quarter = warp & 3;
    const int rlo = quarter * 32 + half * 16 + (lane >> 2);
    const uint32_t lane_addr = tmem + (uint32_t(quarter * 32 + half * 16) << 16);
    const uint32_t s_col = x * 128, o_col = 256 + x * 64, p_col = 384 + x * 64;
    const int cq = 2 * (lane & 3);
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    bool ok = true;
    // two key tiles per loop body (the barrier parities become constants): 1 % faster
#pragma unroll 2
    for (int j = 0; j < nkv; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.s_full[x], j & 1, err))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sc[64];
      tmem_ld_16x256b_x16(lane_addr + s_col, sc);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.s_free[x]);
      if ((j + 1) * BKV > N) {
#pragma unroll
        for (int g = 0; g < 16; ++g)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            if (j * BKV + 8 * g + cq + e >= N) sc[4 * g + e] = sc[4 * g + 2 + e] = -INFINITY;
      }
      if (j * BKV < txt_pad_end && (j + 1) * BKV > txt_valid) {
#pragma unroll
        for (int g = 0; g < 16; ++g)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int key = j * BKV + 8 * g + cq + e;
            if (key >= txt_valid && key < txt_pad_end) sc[4 * g + e] = sc[4 * g + 2 + e] = -INFINITY;
          }
      }
      float p0[4], p1[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        p0[q] = fmaxf(sc[4 * q], sc[4 * q + 1]);
        p1[q] = fmaxf(sc[4 * q + 2], sc[4 * q + 3]);
      }
#pragma unroll
      for (int g = 4; g < 16; ++g) {
        p0[g & 3] = max3f(p0[g & 3], sc[4 * g], sc[4 * g + 1]);
        p1[g & 3] = max3f(p1[g & 3], sc[4 * g + 2], sc[4 * g + 3]);
      }
      float mx0 = max3f(p0[0], p0[1], fmaxf(p0[2], p0[3]));
      float mx1 = max3f(p1[0], p1[1], fmaxf(p1[2], p1[3]));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2)) * scale_log2;
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2)) * scale_log2;
      float c0 = 1.f, c1 = 1.f;
      if (mx0 > m0 + kRescaleThreshold) {
        c0 = ex2(m0 - mx0);
        m0 = mx0;
      }
      if (mx1 > m1 + kRescaleThreshold) {
        c1 = ex2(m1 - mx1);
        m1 = mx1;
      }
      const uint64_t sl2 = f2_pack(scale_log2, scale_log2);
      const uint64_t nb0 = f2_pack(m0 == -INFINITY ? 0.f : -m0, m0 == -INFINITY ? 0.f : -m0);
      const uint64_t nb1 = f2_pack(m1 == -INFINITY ? 0.f : -m1, m1 == -INFINITY ? 0.f : -m1);
      if (x == 1 && j == 0 && !__all_sync(0xffffffffu, mbar_wait(&bar.stagger, 0, err))) {
        ok = false;
        break;
      }
      uint64_t a0[2] = {0ull, 0ull}, a1[2] = {0ull, 0ull};
      uint32_t pk[32];
#pragma unroll
      for (int g = 0; g < 16; ++g) {
        const uint64_t x01 = f2_fma(f2_pack(sc[4 * g], sc[4 * g + 1]), sl2, nb0);
        const uint64_t x23 = f2_fma(f2_pack(sc[4 * g + 2], sc[4 * g + 3]), sl2, nb1);
        float e0, e1, e2, e3;
        if ((LENS_ATTN_EMU_MASK >> g) & 1u) {
          exp2_fma_pair(x01, e0, e1);
          exp2_fma_pair(x23, e2, e3);
        } else {
          float x0, x1, x2, x3;
          f2_unpack(x01, x0, x1);
          f2_unpack(x23, x2, x3);
          e0 = ex2(x0);
          e1 = ex2(x1);
          e2 = ex2(x2);
          e3 = ex2(x3);
        }
        a0[g & 1] = f2_add(a0[g & 1], f2_pack(e0, e1));
        a1[g & 1] = f2_add(a1[g & 1], f2_pack(e2, e3));
        pk[2 * g] = pack_bf16x2(e0, e1);
        pk[2 * g + 1] = pack_bf16x2(e2, e3);
      }
      if (x == 0 && j == 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.stagger);
      }
      float s0, s1, s2, s3;
      f2_unpack(f2_add(a0[0], a0[1]), s0, s1);
      f2_unpack(f2_add(a1[0], a1[1]), s2, s3);
      l0 = l0 * c0 + (s0 + s1);
      l1 = l1 * c1 + (s2 + s3);
      if (j > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bar.pv_done[x], (j - 1) & 1, err))) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      tmem_st_16x128b_x16(lane_addr + p_col, pk);
      if (j > 0 && __any_sync(0xffffffffu, c0 != 1.f || c1 != 1.f)) {
        float o[32];
        tmem_ld_16x256b_x8(lane_addr + o_col, o);
        tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          o[4 * g] *= c0;
          o[4 * g + 1] *= c0;
          o[4 * g + 2] *= c1;
          o[4 * g + 3] *= c1;
        }
        tmem_st_16x256b_x8(lane_addr + o_col, o);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.p_full[x]);
    }
    // row sums: the four threads of a row hold disjoint keys
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (__all_sync(0xffffffffu, ok && mbar_wait(&bar.pv_done[x], (nkv - 1) & 1, err))) {
      tc_fence_after();
      float o[32];
      tmem_ld_16x256b_x8(lane_addr + o_col, o);
      tmem_ld_wait();
      const int hid = heads * 64;
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int tok = q0 + x * BQ + rlo + 8 * rr;
        if (tok < N) {
          // a row with no attended key (l = 0) writes zeros rather than 0 * inf
          const float lr = rr ? l1 : l0;
          const float inv = lr > 0.f ? 1.f / lr : 0.f;
          __nv_bfloat16* dst = tok < n_txt ? out_txt + ((int64_t)b * n_txt + tok) * hid
                                           : out_img + ((int64_t)b * (N - n_txt) + (tok - n_txt)) * hid;
          uint32_t* d32 = reinterpret_cast<uint32_t*>(dst + h * 64 + cq);
#pragma unroll
          for (int g = 0; g < 8; ++g)
            d32[4 * g] = pack_bf16x2(o[4 * g + 2 * rr] * inv, o[4 * g + 2 * rr + 1] * inv);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 17) {
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
  return launch_pdl(tc::joint_attention_tc_kernel, grid, dim3(tc::THREADS), tc::SMEM, st, tq, tk, tv, N, n_txt, heads,
                    out_txt, out_img, scale_log2, lens, err);
}

}  // namespace lens
