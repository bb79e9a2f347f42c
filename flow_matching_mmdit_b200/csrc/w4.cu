// int4 weight-only path: 4-bit codes with a bf16 scale and bias per 64 weights
// ("从提示词到成图：Lens-3.8B-4bit完整管线解析", section 4: 4-bit weights, group size
// 64, img_in / txt_in / proj_out / time_text_embed / norm_out kept in bf16).
//
// The tensor cores take bf16 operands (kind::f16 needs both operands of one type),
// so the 4-bit operand is widened to bf16 in shared memory: TMA brings the codes and
// scales of a 64-wide k block, four dequantizing warps write the bf16 tile in the
// 128-byte-swizzled K-major layout UMMA reads, and only then does the MMA warp issue.
// Everything else (persistent tile walk, two TMEM accumulators, fused epilogues) is
// the bf16 GEMM's (gemm_tc.cuh).
#include "gemm.h"
#include "gemm_tc.cuh"
#include "smem_attr.h"

namespace lens {

void finalize_problems(GemmArgs& a, int bn, int bm);   // gemm.cu

namespace {

// ------------------------------------------------------------------ quantization
// One thread per (row, group of 64).  fp32 arithmetic with explicit round-to-nearest
// operations, so the codes are those of the plain definition bit for bit.
__global__ void quantize_w4_kernel(const __nv_bfloat16* __restrict__ w, int64_t rows, int64_t k,
                                   uint32_t* __restrict__ codes, uint32_t* __restrict__ scales, int64_t scale_ld) {
  const int64_t groups = k / 64;
  const int64_t gi = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (gi >= rows * groups) return;
  const int64_t r = gi / groups, g = gi % groups;
  const __nv_bfloat16* src = w + r * k + g * 64;
  float v[64];
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __bfloat162float(src[i]);
  float mn = v[0], mx = v[0];
#pragma unroll
  for (int i = 1; i < 64; ++i) {
    mn = fminf(mn, v[i]);
    mx = fmaxf(mx, v[i]);
  }
  const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
  const __nv_bfloat16 bb = __float2bfloat16_rn(mn);
  const float s = __bfloat162float(sb), b = __bfloat162float(bb);
  uint32_t word[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) word[i] = 0u;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    float q = s > 0.f ? rintf(__fdiv_rn(__fsub_rn(v[i], b), s)) : 0.f;
    q = fminf(fmaxf(q, 0.f), 15.f);
    const int within = i & 7, j = within >> 1;
    word[i >> 3] |= uint32_t(q) << ((within & 1) ? 16 + 4 * j : 4 * j);
  }
  uint32_t* dst = codes + r * (k / 8) + g * 8;
#pragma unroll
  for (int i = 0; i < 8; ++i) dst[i] = word[i];
  scales[g * scale_ld + r] = uint32_t(__bfloat16_as_ushort(sb)) | (uint32_t(__bfloat16_as_ushort(bb)) << 16);
}

// ------------------------------------------------------------------ GEMM configuration
// MH = 128-row halves of the M tile (2: one widened B tile feeds two M = 128 MMAs,
// halving the widening per MMA flop; B side only).
template <int BN, int EPI, bool QA, int MH = 1>
struct GemmW4Cfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int QROWS = QA ? BM : BN;                       // rows of the 4-bit operand tile
  static constexpr uint32_t A_BYTES = MH * BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  static constexpr uint32_t QC_BYTES = QROWS * 32;                 // codes of one k block
  static constexpr uint32_t QS_BYTES = ((QROWS * 4 + 127) / 128) * 128;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + QC_BYTES + QS_BYTES;
  static constexpr uint32_t TX_BYTES = (QA ? B_BYTES : A_BYTES) + QROWS * 32 + QROWS * 4;
  static constexpr uint32_t EPI_SLOT = 4096;
  static constexpr uint32_t EPI_BYTES = epi_uses_tma(EPI) ? 4 * 2 * EPI_SLOT : 0;
  static constexpr uint32_t AUX_BYTES = EPI == EPI_QKV ? 1024 : 0;
  static constexpr uint32_t BAR_BYTES = 512;
  static constexpr uint32_t BUDGET = 232448 - 1024 - BAR_BYTES - EPI_BYTES - AUX_BYTES;
  static constexpr int STAGES = (BUDGET / STAGE_BYTES) > 8 ? 8 : (BUDGET / STAGE_BYTES);
  static constexpr uint32_t TMEM_COLS = pow2_at_least(2 * MH * BN);
  static constexpr size_t SMEM = 1024 + size_t(STAGES) * STAGE_BYTES + EPI_BYTES + AUX_BYTES + BAR_BYTES;
  static_assert(STAGES >= 2, "shared memory too small for two stages");
  static_assert(MH == 1 || (MH == 2 && !QA), "two M halves only with a 4-bit B");
  static_assert(2 * MH * BN <= 512, "two accumulators must fit TMEM");
};

constexpr int kW4Threads = 320;

// Widen one k block of the 4-bit operand (QROWS rows) into the bf16 tile at dst
// (128-byte rows, 16-byte chunk c of row n stored at chunk c ^ (n & 7)).  tid in [0, 128).
// Work item = half a row (32 codes, 16 bytes): one 16-byte code load and one scale
// load feed four 16-byte stores; a quarter warp stores 8 distinct chunk positions.
// A thread's items are independent: all their loads are issued before any math.
template <int QROWS>
__device__ __forceinline__ void dequant_block(const uint32_t* __restrict__ qc, const uint32_t* __restrict__ qs,
                                              uint8_t* dst, int tid) {
  const uint32_t k128 = 0x43004300u;                   // bf16 pair (128, 128)
  constexpr int kItems = (QROWS * 2 + 127) / 128;      // half rows per thread (the last may be partial)
  // every item's loads first, so their latencies overlap
  uint4 x4[kItems];
  uint32_t sbw[kItems];
#pragma unroll
  for (int u = 0; u < kItems; ++u) {
    const int it = tid + 128 * u;
    if (it < QROWS * 2) {
      x4[u] = reinterpret_cast<const uint4*>(qc)[it];
      sbw[u] = qs[it >> 1];
    }
  }
#pragma unroll
  for (int u = 0; u < kItems; ++u) {
    const int it = tid + 128 * u;
    if (it >= QROWS * 2) break;
    const int n = it >> 1, half = it & 1;
    const uint32_t s2 = __byte_perm(sbw[u], 0, 0x1010), b2 = __byte_perm(sbw[u], 0, 0x3232);
    const uint32_t xs[4] = {x4[u].x, x4[u].y, x4[u].z, x4[u].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t v = ((xs[i] >> (4 * j)) & 0x000F000Fu) | k128;   // (128 + q_2j, 128 + q_2j+1), exact
        asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(v) : "r"(v), "r"(k128));
        asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(o[j]) : "r"(v), "r"(s2), "r"(b2));
      }
      const int wi = half * 4 + i;
      *reinterpret_cast<uint4*>(dst + n * 128 + ((wi ^ (n & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

template <int MH>
__device__ __forceinline__ void w4_decode(const GemmArgs& a, int t, int bn, int& pi, int& m0, int& n0) {
  if (MH == 2)
    decode_tile2(a, t, bn, pi, m0, n0);       // 256-row tiles
  else
    decode_tile(a, t, bn, pi, m0, n0);
}

// ------------------------------------------------------------------ kernel
// Warp roles (320 threads):
//   warp 0      TMA: the bf16 operand tile (A when QA is false, else B), the codes and
//               the scales of the 4-bit operand, one k block per stage
//   warp 1      UMMA issuer: waits until a stage is widened (bfull), 4 x K=16 MMAs
//   warps 2..5  epilogue (as the bf16 GEMM)
//   warps 6..9  widen the 4-bit operand of each stage into its bf16 slot, make the
//               stores visible to the tensor core (async proxy), arrive on bfull
// bfull is arrived only after full completed, so it also covers the TMA bytes.
template <int BN, int EPI, bool QA, int MH>
__global__ void __launch_bounds__(kW4Threads, 1)
    gemm_w4_kernel(const __grid_constant__ CUtensorMap tmX0, const __grid_constant__ CUtensorMap tmQ0,
                   const __grid_constant__ CUtensorMap tmS0, const __grid_constant__ CUtensorMap tmX1,
                   const __grid_constant__ CUtensorMap tmQ1, const __grid_constant__ CUtensorMap tmS1,
                   const __grid_constant__ CUtensorMap tmC0, const __grid_constant__ CUtensorMap tmC1,
                   const __grid_constant__ GemmArgs args) {
  using C = GemmW4Cfg<BN, EPI, QA, MH>;
  constexpr int STAGES = C::STAGES;
  constexpr uint32_t A_HALF = C::A_BYTES / MH;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * C::A_BYTES;
  uint8_t* sEpi = sB + STAGES * C::B_BYTES;
  float* sAux = reinterpret_cast<float*>(sEpi + C::EPI_BYTES);
  uint8_t* sQc = sEpi + C::EPI_BYTES + C::AUX_BYTES;
  uint8_t* sQs = sQc + STAGES * C::QC_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sQs + STAGES * C::QS_BYTES);
  uint64_t* bfull = full + STAGES;
  uint64_t* empty = bfull + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;          // MMA issuer's own completion after an abort
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&bfull[s], 4);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmX0);
    tma_prefetch_desc(&tmQ0);
    tma_prefetch_desc(&tmS0);
    if (args.num_problems > 1) {
      tma_prefetch_desc(&tmX1);
      tma_prefetch_desc(&tmQ1);
      tma_prefetch_desc(&tmS1);
    }
  }
  if constexpr (EPI == EPI_QKV) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) {
      const GemmProblem& P = args.p[(i >> 7) < args.num_problems ? (i >> 7) : 0];
      sAux[i] = (i & 64) ? P.gain_k[i & 63] : P.gain_q[i & 63];
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t last_parity[STAGES];
      bool issued[STAGES];
      for (int s = 0; s < STAGES; ++s) issued[s] = false, last_parity[s] = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < args.total_tiles && ok; t += gridDim.x) {
        int pi, m0, n0;
        w4_decode<MH>(args, t, BN, pi, m0, n0);
        const CUtensorMap* mX = pi ? &tmX1 : &tmX0;
        const CUtensorMap* mQ = pi ? &tmQ1 : &tmQ0;
        const CUtensorMap* mS = pi ? &tmS1 : &tmS0;
        const int q0 = QA ? m0 : n0;
        const int kblocks = args.p[pi].K / C::BK;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, args.err)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&full[stage], C::TX_BYTES);
          if (QA) {
            tma_load_2d(sB + stage * C::B_BYTES, mX, &full[stage], kb * C::BK, n0);
          } else {
#pragma unroll
            for (int h = 0; h < MH; ++h)
              tma_load_2d(sA + stage * C::A_BYTES + h * A_HALF, mX, &full[stage], kb * C::BK, m0 + 128 * h);
          }
          tma_load_2d(sQc + stage * C::QC_BYTES, mQ, &full[stage], kb * 32, q0);
          tma_load_2d(sQs + stage * C::QS_BYTES, mS, &full[stage], q0, kb);
          issued[stage] = true;
          last_parity[stage] = phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok || err_raised(args.err)) {
        // after an abort the consumers may not have waited for every stage filled here
        for (int s = 0; s < STAGES; ++s)
          if (issued[s]) mbar_wait_drain(&full[s], last_parity[s]);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(128, BN);
      uint32_t stage = 0, phase = 0;
      int li = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < args.total_tiles && ok; t += gridDim.x, ++li) {
        int pi, m0, n0;
        w4_decode<MH>(args, t, BN, pi, m0, n0);
        const int kblocks = args.p[pi].K / C::BK;
        const uint32_t acc = li & 1;
        const uint32_t use = li >> 1;
        if (!mbar_wait_sleep(&tempty[acc], (use & 1) ^ 1, args.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * MH * BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_sleep(&bfull[stage], phase, args.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bd = umma_desc_sw128(smem_u32(sB + stage * C::B_BYTES));
#pragma unroll
          for (int h = 0; h < MH; ++h) {
            const uint64_t ad = umma_desc_sw128(smem_u32(sA + stage * C::A_BYTES + h * A_HALF));
#pragma unroll
            for (int k = 0; k < C::BK / 16; ++k)
              umma_bf16(d_tmem + h * BN, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
      }
      if (!ok) umma_drain(drain);   // no UMMA still writes TMEM or reads a stage when the CTA leaves
    }
    __syncwarp();
  } else if (warp < 6) {
    const int quarter = warp & 3;
    uint8_t* slots = sEpi + quarter * 2 * C::EPI_SLOT;
    uint32_t slot = 0;
    int li = 0;
    for (int t = blockIdx.x; t < args.total_tiles; t += gridDim.x, ++li) {
      int pi, m0, n0;
      w4_decode<MH>(args, t, BN, pi, m0, n0);
      const uint32_t acc = li & 1;
      const uint32_t use = li >> 1;
      if (!mbar_wait(&tfull[acc], use & 1, args.err)) break;
      tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < MH; ++h) {
        const int row0 = m0 + 128 * h + quarter * 32;
        const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16) + acc * MH * BN + h * BN;
        const float4 none[16] = {};   // the epilogue loads its per-row operands itself here
        epilogue_tile<BN, EPI, 2, false>(args.p[pi], pi ? &tmC1 : &tmC0, row0 + lane, row0, n0, taddr, slots,
                                         slot, sAux + pi * 128, none);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
    if constexpr (epi_uses_tma(EPI)) {
      if (lane == 0) bulk_wait_read<0>();      // read out of shared memory; the grid covers the rest
      __syncwarp();
    }
  } else {
    const int tid = threadIdx.x - 192;
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < args.total_tiles && ok; t += gridDim.x) {
      int pi, m0, n0;
      w4_decode<MH>(args, t, BN, pi, m0, n0);
      const int kblocks = args.p[pi].K / C::BK;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!mbar_wait(&full[stage], phase, args.err)) {
          ok = false;
          break;
        }
        dequant_block<C::QROWS>(reinterpret_cast<const uint32_t*>(sQc + stage * C::QC_BYTES),
                                reinterpret_cast<const uint32_t*>(sQs + stage * C::QS_BYTES),
                                QA ? sA + stage * C::A_BYTES : sB + stage * C::B_BYTES, tid);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bfull[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int BN, int EPI, bool QA, int MH>
cudaError_t launch_w4_one(const CUtensorMap& X0, const CUtensorMap& Q0, const CUtensorMap& S0, const CUtensorMap& X1,
                          const CUtensorMap& Q1, const CUtensorMap& S1, const CUtensorMap& C0, const CUtensorMap& C1,
                          const GemmArgs& args, int sms, cudaStream_t st) {
  using C = GemmW4Cfg<BN, EPI, QA, MH>;
  static std::atomic<uint64_t> attr{0};
  {
    const cudaError_t e = ensure_smem_limit(gemm_w4_kernel<BN, EPI, QA, MH>, (int)C::SMEM, attr);
    if (e != cudaSuccess) return e;
  }
  const int grid = args.total_tiles < sms ? args.total_tiles : sms;
  gemm_w4_kernel<BN, EPI, QA, MH><<<grid, kW4Threads, C::SMEM, st>>>(X0, Q0, S0, X1, Q1, S1, C0, C1, args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_w4(const void* w_bf16, int64_t rows, int64_t k, uint8_t* codes, uint32_t* scales,
                               int64_t scale_ld, cudaStream_t st) {
  if (rows <= 0 || k <= 0 || k % 64 || scale_ld < rows || (reinterpret_cast<uintptr_t>(codes) & 15) ||
      (reinterpret_cast<uintptr_t>(w_bf16) & 1))
    return cudaErrorInvalidValue;
  const int64_t n = rows * (k / 64);
  quantize_w4_kernel<<<(unsigned)((n + 127) / 128), 128, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(w_bf16),
                                                                   rows, k, reinterpret_cast<uint32_t*>(codes),
                                                                   scales, scale_ld);
  return cudaGetLastError();
}

cudaError_t launch_gemm_w4(int bm, int bn, int epi, bool quant_a, const CUtensorMap* A0, const CUtensorMap* B0,
                           const CUtensorMap* Q0, const CUtensorMap* S0, const CUtensorMap* A1, const CUtensorMap* B1,
                           const CUtensorMap* Q1, const CUtensorMap* S1, const CUtensorMap* C0, const CUtensorMap* C1,
                           GemmArgs& args, int sms, cudaStream_t st) {
  if (bm != 128 && (bm != 256 || quant_a)) return cudaErrorInvalidValue;
  finalize_problems(args, bn, bm);
  if (args.total_tiles == 0) return cudaSuccess;
  const CUtensorMap* X0 = quant_a ? B0 : A0;
  const CUtensorMap* X1 = quant_a ? B1 : A1;
  if (!X0 || !Q0 || !S0) return cudaErrorInvalidValue;
  if (args.num_problems > 1 && (!X1 || !Q1 || !S1)) return cudaErrorInvalidValue;
  if (epi_uses_tma(epi) && (!C0 || (args.num_problems > 1 && !C1))) return cudaErrorInvalidValue;
  const CUtensorMap& x1 = X1 ? *X1 : *X0;
  const CUtensorMap& q1 = Q1 ? *Q1 : *Q0;
  const CUtensorMap& s1 = S1 ? *S1 : *S0;
  const CUtensorMap& c0 = C0 ? *C0 : *X0;
  const CUtensorMap& c1 = C1 ? *C1 : c0;
#define LENS_W4_CASE(BM_, BN_, EPI_, QA_)                                                                   \
  if (bm == BM_ && bn == BN_ && epi == EPI_ && quant_a == QA_)                                              \
    return launch_w4_one<BN_, EPI_, QA_, BM_ / 128>(*X0, *Q0, *S0, x1, q1, s1, c0, c1, args, sms, st);
  LENS_W4_CASE(128, 256, EPI_F32, false)
  LENS_W4_CASE(128, 128, EPI_F32, false)
  LENS_W4_CASE(256, 128, EPI_F32, false)
  LENS_W4_CASE(128, 192, EPI_QKV, false)
  LENS_W4_CASE(256, 128, EPI_QKV, false)
  LENS_W4_CASE(128, 192, EPI_RESID, false)
  LENS_W4_CASE(256, 96, EPI_RESID, false)
  LENS_W4_CASE(128, 256, EPI_SWIGLU, false)
  LENS_W4_CASE(256, 128, EPI_SWIGLU, false)
  LENS_W4_CASE(128, 16, EPI_F32_T, true)
  LENS_W4_CASE(128, 32, EPI_F32_T, true)
  LENS_W4_CASE(128, 64, EPI_F32_T, true)
#undef LENS_W4_CASE
  return cudaErrorInvalidValue;
}

}  // namespace lens
