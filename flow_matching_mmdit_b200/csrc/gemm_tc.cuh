// Persistent tcgen05/TMEM GEMM for sm_100a with the denoiser's fused epilogues.
//
//   D[m, n] = sum_k A[m, k] * B[n, k]       A, B bf16, K-contiguous, fp32 accumulate
//
// One CTA per SM walks a static round-robin list of 128 x BN output tiles drawn
// from up to two independent problems (the image and the text stream of a block
// run as one launch).  Warp roles (192 threads):
//   warp 0      TMA producer: 128x64 A and BNx64 B tiles, 128-byte swizzle,
//               STAGES-deep ring of shared-memory stages
//   warp 1      UMMA issuer (one thread): 4 x (M=128, N=BN, K=16) per stage into a
//               TMEM accumulator; two accumulators so the epilogue of tile i
//               overlaps the main loop of tile i+1
//   warps 2..5  epilogue: each warp reads its 32 TMEM lanes (= 32 output rows),
//               one row per thread, applies the fused epilogue, and (for the
//               store kinds) stages 32 x 128-byte boxes in a double-buffered
//               swizzled shared-memory slot that one lane ships with a TMA store
//               or a TMA reduce-add
// Epilogues:
//   EPI_F32     out = acc + bias                       (img_in, txt_in, proj_out)  TMA store
//   EPI_RESID   h  += gate[b] * (acc + bias)           (to_out / to_add_out, w2)   TMA reduce-add
//   EPI_SWIGLU  u   = silu(acc_g + b1) * (acc_u + b3)  (w1|w3 interleaved by 32)   TMA store
//   EPI_QKV     q, k: per-head RMSNorm * gain, RoPE; v as is; written head-major
//               into the joint [B, 24, N, 64] sequence
//   EPI_F32_T   out[n][m] = acc + bias[m]              (AdaLN modulation, A = weights)
#pragma once
#include "ptx.cuh"

namespace lens {

enum EpiKind { EPI_F32 = 0, EPI_RESID = 1, EPI_SWIGLU = 2, EPI_QKV = 3, EPI_F32_T = 4 };

struct GemmProblem {
  int M, N, K;
  int tiles_m, tiles_n, tile_begin;
  float* out_f32;
  int64_t ld_out;
  __nv_bfloat16* out_bf16;
  const float* bias;
  const float* gate;
  int64_t gate_stride;
  int rows_per_batch;
  int n_valid;
  __nv_bfloat16* q;
  __nv_bfloat16* k;
  __nv_bfloat16* v;
  const float* gain_q;
  const float* gain_k;
  const float2* rope;
  int n_tok;
  int tok_offset;
  int heads;
  float eps;
};

struct GemmArgs {
  GemmProblem p[2];
  int num_problems;
  int total_tiles;
  // CTA-pair kernel: tiles [tail_begin, total_tiles) (the last, partly filled round)
  // are each computed as tail_split narrower tiles of BN / tail_split columns, so that
  // they spread over the CTA pairs that would otherwise idle; total_items counts
  // the work items that result.  The other kernels leave them at (total_tiles, 1,
  // total_tiles).
  int tail_begin, tail_split, total_items;
  int* err;
};

constexpr bool epi_uses_tma(int epi) { return epi == EPI_F32 || epi == EPI_RESID || epi == EPI_SWIGLU; }
constexpr uint32_t pow2_at_least(uint32_t x) {
  uint32_t p = 32;
  while (p < x) p <<= 1;
  return p;
}

template <int BN, int EPI>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  // epilogue staging: 4 warps x 2 slots x (32 rows x 128 B)
  static constexpr uint32_t EPI_SLOT = 4096;
  static constexpr uint32_t EPI_BYTES = epi_uses_tma(EPI) ? 4 * 2 * EPI_SLOT : 0;
  static constexpr uint32_t AUX_BYTES = EPI == EPI_QKV ? 1024 : 0;
  static constexpr uint32_t BUDGET = 232448 - 1024 - 256 - EPI_BYTES - AUX_BYTES;
  static constexpr int STAGES = (BUDGET / STAGE_BYTES) > 12 ? 12 : (BUDGET / STAGE_BYTES);
  static constexpr uint32_t TMEM_COLS = pow2_at_least(2 * BN);
  static constexpr size_t SMEM = 1024 + size_t(STAGES) * STAGE_BYTES + EPI_BYTES + AUX_BYTES + 256;
};

__device__ __forceinline__ void decode_tile(const GemmArgs& a, int t, int bn, int& pi, int& m0, int& n0) {
  pi = (a.num_problems > 1 && t >= a.p[1].tile_begin) ? 1 : 0;
  const GemmProblem& P = a.p[pi];
  const int local = t - P.tile_begin;
  m0 = (local % P.tiles_m) * 128;
  n0 = (local / P.tiles_m) * bn;
}

// SiLU with the fast reciprocal division (the result is rounded to bf16): for very
// negative x the denominator overflows to inf and the quotient is 0, the limit.
__device__ __forceinline__ float silu_f(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

// ------------------------------------------------------------------ epilogues
// Stage one 32-row x 128-byte box (this thread's row = `lane`) in the warp's next
// shared-memory slot with the 128-byte swizzle, then let lane 0 ship it.
template <bool REDUCE, int NSLOTS>
__device__ __forceinline__ void stage_and_ship(uint8_t* slots, uint32_t& slot, const uint4 (&chunk)[8],
                                               const CUtensorMap* map, int x, int y, bool ship) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) bulk_wait_read<NSLOTS - 1>();   // the slot's previous box has been read out
  __syncwarp();
  uint8_t* buf = slots + slot * 4096;
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4*>(buf + lane * 128 + ((c ^ (lane & 7)) << 4)) = chunk[c];
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && ship) {
    if (REDUCE)
      tma_reduce_add_2d(map, buf, x, y);
    else
      tma_store_2d(map, buf, x, y);
  }
  if (lane == 0) bulk_commit();
  if (NSLOTS == 2) slot ^= 1;
}

// Per-row operands of a tile's epilogue that do not depend on the accumulator, loaded
// before the wait for it so that their latency hides behind that wait: the gates of the
// first 32-column chunk of this warp's part (residual epilogue, pre[0..7]), or this
// row's RoPE (cos, sin) pairs (QKV epilogue on a q or k tile, pre[0..15]).
template <int BN, int EPI>
__device__ __forceinline__ void epilogue_prefetch(const GemmProblem& P, int row, int n0, int part, int parts,
                                                  float4 (&pre)[16], int width = BN) {
  if (row >= P.M) return;
  const int b = row / P.rows_per_batch;
  if constexpr (EPI == EPI_RESID) {
    const float4* g4 = reinterpret_cast<const float4*>(P.gate + (int64_t)b * P.gate_stride + n0 +
                                                       part * (width / 32) / parts * 32);
#pragma unroll
    for (int j = 0; j < 8; ++j) pre[j] = __ldg(g4 + j);
  } else if constexpr (EPI == EPI_QKV) {
    if (n0 / (P.heads * 64) < 2) {
      const int tok = P.tok_offset + row - b * P.rows_per_batch;
      const float4* rope4 = reinterpret_cast<const float4*>(P.rope + (int64_t)tok * 32);
#pragma unroll
      for (int j = 0; j < 16; ++j) pre[j] = __ldg(rope4 + j);
    }
  }
}

// `part` of `parts` column ranges of the tile (32-column chunks, SwiGLU 128-column
// groups, QKV heads) is this warp's; the other parts go to warps reading the same
// TMEM lanes.  NSLOTS staging slots of 4 KB per warp.  With PRE, `pre` holds what
// epilogue_prefetch loaded for this tile (the residual and QKV epilogues use it);
// without, the epilogue loads those operands itself.
template <int BN, int EPI, int NSLOTS = 2, bool PRE = true>
__device__ __forceinline__ void epilogue_tile(const GemmProblem& P, const CUtensorMap* tmC, int row, int row0_warp,
                                              int n0, uint32_t taddr, uint8_t* slots, uint32_t& slot,
                                              const float* qk_gains, const float4 (&pre)[16], int part = 0,
                                              int parts = 1, int width = BN) {
  const bool live = row < P.M;
  const bool any_live = row0_warp < P.M;
  if constexpr (EPI == EPI_F32 || EPI == EPI_RESID) {
    const float* gate = nullptr;
    const int c_begin = part * (width / 32) / parts, c_end = (part + 1) * (width / 32) / parts;
    float4 gnext[8];                     // the gates of the next chunk, loaded one chunk ahead
    if constexpr (EPI == EPI_RESID) {
      const int b = live ? row / P.rows_per_batch : 0;
      gate = P.gate + (int64_t)b * P.gate_stride + n0;
      if (live) {
        const float4* g4 = reinterpret_cast<const float4*>(gate + c_begin * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j) gnext[j] = PRE ? pre[j] : __ldg(g4 + j);
      }
    }
#pragma unroll 1
    for (int c = c_begin; c < c_end; ++c) {
      float4 gcur[8];
      if constexpr (EPI == EPI_RESID) {
#pragma unroll
        for (int j = 0; j < 8; ++j) gcur[j] = gnext[j];
        if (live && c + 1 < c_end) {
          const float4* g4 = reinterpret_cast<const float4*>(gate + (c + 1) * 32);
#pragma unroll
          for (int j = 0; j < 8; ++j) gnext[j] = __ldg(g4 + j);
        }
      }
      float r[32];
      tmem_ld32(taddr + c * 32, r);
      tmem_ld_wait();
      const int col = c * 32;
      if (P.bias) {
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] += __ldg(P.bias + n0 + col + j);
      }
      if constexpr (EPI == EPI_RESID) {
        if (live) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            r[4 * j] *= gcur[j].x;
            r[4 * j + 1] *= gcur[j].y;
            r[4 * j + 2] *= gcur[j].z;
            r[4 * j + 3] *= gcur[j].w;
          }
        }
      }
      uint4 ch[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        ch[j] = make_uint4(__float_as_uint(r[4 * j]), __float_as_uint(r[4 * j + 1]), __float_as_uint(r[4 * j + 2]),
                           __float_as_uint(r[4 * j + 3]));
      stage_and_ship<EPI == EPI_RESID, NSLOTS>(slots, slot, ch, tmC, n0 + col, row0_warp, any_live);
    }
  } else if constexpr (EPI == EPI_SWIGLU) {
    // B rows were packed [w1 rows 32c..32c+31 | w3 rows 32c..32c+31] per 64 columns;
    // every 128 accumulator columns give 64 outputs = one 128-byte box row
#pragma unroll 1
    for (int c = part * (width / 128) / parts; c < (part + 1) * (width / 128) / parts; ++c) {
      uint4 ch[8];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float g[32], u[32];
        tmem_ld32(taddr + c * 128 + half * 64, g);
        tmem_ld32(taddr + c * 128 + half * 64 + 32, u);
        tmem_ld_wait();
        if (P.bias) {
          const float* b = P.bias + n0 + c * 128 + half * 64;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            g[j] += __ldg(b + j);
            u[j] += __ldg(b + 32 + j);
          }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
          ch[half * 4 + j] =
              make_uint4(pack_bf16x2(silu_f(g[8 * j + 0]) * u[8 * j + 0], silu_f(g[8 * j + 1]) * u[8 * j + 1]),
                         pack_bf16x2(silu_f(g[8 * j + 2]) * u[8 * j + 2], silu_f(g[8 * j + 3]) * u[8 * j + 3]),
                         pack_bf16x2(silu_f(g[8 * j + 4]) * u[8 * j + 4], silu_f(g[8 * j + 5]) * u[8 * j + 5]),
                         pack_bf16x2(silu_f(g[8 * j + 6]) * u[8 * j + 6], silu_f(g[8 * j + 7]) * u[8 * j + 7]));
      }
      stage_and_ship<false, NSLOTS>(slots, slot, ch, tmC, n0 / 2 + c * 64, row0_warp, any_live);
    }
  } else if constexpr (EPI == EPI_QKV) {
    // gains: the problem's q and k gains staged in shared memory at kernel start
    const int hidden = P.heads * 64;
    const int sec = n0 / hidden;                  // 0 = q, 1 = k, 2 = v
    const int head0 = (n0 - sec * hidden) / 64;
    const int b = live ? row / P.rows_per_batch : 0;
    const int tok = P.tok_offset + (live ? row - b * P.rows_per_batch : 0);
    __nv_bfloat16* base = sec == 0 ? P.q : (sec == 1 ? P.k : P.v);
    const float4* gain4 = reinterpret_cast<const float4*>(qk_gains + (sec == 0 ? 0 : 64));
    float4 rown[16];
    if constexpr (!PRE) {
      if (sec < 2 && live) {
        const float4* rope4 = reinterpret_cast<const float4*>(P.rope + (int64_t)tok * 32);
#pragma unroll
        for (int p = 0; p < 16; ++p) rown[p] = __ldg(rope4 + p);
      }
    }
    const float4 (&rp)[16] = *(PRE ? &pre : &rown);   // this row's (cos, sin) pairs (q and k tiles)
#pragma unroll 1
    for (int hh = part * (width / 64) / parts; hh < (part + 1) * (width / 64) / parts; ++hh) {
      float x[64];
      tmem_ld32(taddr + hh * 64, *reinterpret_cast<float(*)[32]>(&x[0]));
      tmem_ld32(taddr + hh * 64 + 32, *reinterpret_cast<float(*)[32]>(&x[32]));
      tmem_ld_wait();
      if (!live) continue;
      const int col = n0 + hh * 64;
      if (P.bias) {
#pragma unroll
        for (int j = 0; j < 64; ++j) x[j] += __ldg(P.bias + col + j);
      }
      if (sec < 2) {
        float ss0 = 0.f, ss1 = 0.f;
#pragma unroll
        for (int j = 0; j < 64; j += 2) {
          ss0 += x[j] * x[j];
          ss1 += x[j + 1] * x[j + 1];
        }
        const float rs = rsqrtf((ss0 + ss1) * (1.0f / 64.0f) + P.eps);
#pragma unroll
        for (int q4 = 0; q4 < 16; ++q4) {
          const float4 g = gain4[q4];
          x[4 * q4] *= rs * g.x;
          x[4 * q4 + 1] *= rs * g.y;
          x[4 * q4 + 2] *= rs * g.z;
          x[4 * q4 + 3] *= rs * g.w;
        }
#pragma unroll
        for (int p = 0; p < 16; ++p) {           // pairs 2p and 2p+1 of rp[p]
          const float a0 = x[4 * p], b0 = x[4 * p + 1], a1 = x[4 * p + 2], b1 = x[4 * p + 3];
          x[4 * p] = a0 * rp[p].x - b0 * rp[p].y;
          x[4 * p + 1] = a0 * rp[p].y + b0 * rp[p].x;
          x[4 * p + 2] = a1 * rp[p].z - b1 * rp[p].w;
          x[4 * p + 3] = a1 * rp[p].w + b1 * rp[p].z;
        }
      }
      const int head = head0 + hh;
      uint4* d4 = reinterpret_cast<uint4*>(base + (((int64_t)b * P.heads + head) * P.n_tok + tok) * 64);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        d4[j] = make_uint4(pack_bf16x2(x[8 * j], x[8 * j + 1]), pack_bf16x2(x[8 * j + 2], x[8 * j + 3]),
                           pack_bf16x2(x[8 * j + 4], x[8 * j + 5]), pack_bf16x2(x[8 * j + 6], x[8 * j + 7]));
    }
  } else if constexpr (EPI == EPI_F32_T) {
    const float bias = (live && P.bias) ? __ldg(P.bias + row) : 0.f;
    if constexpr (BN == 16) {
      float r[16];
      tmem_ld16(taddr, r);
      tmem_ld_wait();
      if (live) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (n0 + j < P.n_valid) P.out_f32[(int64_t)(n0 + j) * P.ld_out + row] = r[j] + bias;
      }
    } else {
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float r[32];
        tmem_ld32(taddr + c * 32, r);
        tmem_ld_wait();
        if (live) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int n = n0 + c * 32 + j;
            if (n < P.n_valid) P.out_f32[(int64_t)n * P.ld_out + row] = r[j] + bias;
          }
        }
      }
    }
  }
}

// ------------------------------------------------------------------ kernel
template <int BN, int EPI>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                   const __grid_constant__ CUtensorMap tmC0, const __grid_constant__ CUtensorMap tmC1,
                   const __grid_constant__ GemmArgs args) {
  using C = GemmCfg<BN, EPI>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * C::A_BYTES;
  uint8_t* sEpi = sB + STAGES * C::B_BYTES;
  float* sAux = reinterpret_cast<float*>(sEpi + C::EPI_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(sEpi + C::EPI_BYTES + C::AUX_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;          // MMA issuer's own completion after an abort
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmB0);
    if (args.num_problems > 1) {
      tma_prefetch_desc(&tmA1);
      tma_prefetch_desc(&tmB1);
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
  grid_dependency_sync();    // set-up above touched only shared memory, TMEM and weights

  if (warp == 0) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t last_parity[STAGES > 0 ? STAGES : 1];
      bool issued[STAGES > 0 ? STAGES : 1];
      for (int s = 0; s < STAGES; ++s) issued[s] = false, last_parity[s] = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < args.total_tiles && ok; t += gridDim.x) {
        int pi, m0, n0;
        decode_tile(args, t, BN, pi, m0, n0);
        const CUtensorMap* mA = pi ? &tmA1 : &tmA0;
        const CUtensorMap* mB = pi ? &tmB1 : &tmB0;
        const int kblocks = args.p[pi].K / C::BK;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, args.err)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&full[stage], C::STAGE_BYTES);
          tma_load_2d(sA + stage * C::A_BYTES, mA, &full[stage], kb * C::BK, m0);
          tma_load_2d(sB + stage * C::B_BYTES, mB, &full[stage], kb * C::BK, n0);
          issued[stage] = true;
          last_parity[stage] = phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok || err_raised(args.err)) {
        // leave no copy in flight into this CTA's shared memory (after an abort the
        // consumers may not have waited for every stage this thread filled)
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
        decode_tile(args, t, BN, pi, m0, n0);
        const int kblocks = args.p[pi].K / C::BK;
        const uint32_t acc = li & 1;
        const uint32_t use = li >> 1;
        if (!mbar_wait_sleep(&tempty[acc], (use & 1) ^ 1, args.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_sleep(&full[stage], phase, args.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = umma_desc_sw128(smem_u32(sA + stage * C::A_BYTES));
          const uint64_t bd = umma_desc_sw128(smem_u32(sB + stage * C::B_BYTES));
#pragma unroll
          for (int k = 0; k < C::BK / 16; ++k)
            umma_bf16(d_tmem, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
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
  } else {
    const int quarter = warp & 3;
    uint8_t* slots = sEpi + quarter * 2 * C::EPI_SLOT;
    uint32_t slot = 0;
    int li = 0;
    for (int t = blockIdx.x; t < args.total_tiles; t += gridDim.x, ++li) {
      int pi, m0, n0;
      decode_tile(args, t, BN, pi, m0, n0);
      const uint32_t acc = li & 1;
      const uint32_t use = li >> 1;
      const int row0 = m0 + quarter * 32;
      float4 pre[16];
      epilogue_prefetch<BN, EPI>(args.p[pi], row0 + lane, n0, 0, 1, pre);
      if (!mbar_wait(&tfull[acc], use & 1, args.err)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16) + acc * BN;
      epilogue_tile<BN, EPI>(args.p[pi], pi ? &tmC1 : &tmC0, row0 + lane, row0, n0, taddr, slots, slot,
                             sAux + pi * 128, pre);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
    if constexpr (epi_uses_tma(EPI)) {
      // every box has been read out of shared memory before the CTA leaves; the
      // grid's completion covers the writes to global memory
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ==================================================================== CTA-pair version
// The same problem list and epilogues on 256 x BN tiles computed by a cluster of two
// CTAs with cta_group::2 UMMA: CTA rank r stages A rows [m0 + 128 r, +128) and B
// rows [n0 + r BN/2, +BN/2); the leader (rank 0) issues M = 256 MMAs that read both
// CTAs' shared memory and write each CTA's 128-row half of D into its own TMEM.
// Per output element this halves the B operand traffic into shared memory.
//   full[s]    (leader)  TMA bytes of both CTAs; armed by the leader's producer
//   empty[s]   (both)    MMA commit multicast: stage s may be refilled
//   tfull[a]   (both)    MMA commit multicast: accumulator a holds a finished tile
//   tempty[a]  (leader)  2 x epilogue warps arrivals (both CTAs): accumulator a free
// The SwiGLU epilogue (a SiLU per output) runs on eight warps per CTA (320 threads),
// two per TMEM lane quarter, each taking half of a tile's 128-column groups: on four
// it took longer than the next tile's main loop (measured 23 % of the launch at the
// 1024^2 shape), and the MMA waited for a free accumulator.  One 4 KB staging slot
// each, the same 32 KB as four warps with two.  The other epilogues keep four warps:
// the residual ones are bound by the TMA reduce-add, and the QKV one measured slower
// on eight (three heads split 2 / 1, more warps beside the MMA issuer).
template <int BN, int EPI>
struct Gemm2Cfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = (BN / 2) * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_WARPS = EPI == EPI_SWIGLU ? 8 : 4;
  static constexpr int EPI_PARTS = EPI_WARPS / 4;            // column parts per TMEM lane quarter
  static constexpr int EPI_SLOTS = 2 / EPI_PARTS;            // 4 KB staging slots per epilogue warp
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr uint32_t EPI_SLOT = 4096;
  static constexpr uint32_t EPI_BYTES = epi_uses_tma(EPI) ? EPI_WARPS * EPI_SLOTS * EPI_SLOT : 0;
  static constexpr uint32_t AUX_BYTES = EPI == EPI_QKV ? 1024 : 0;
  static constexpr uint32_t BUDGET = 232448 - 1024 - 256 - EPI_BYTES - AUX_BYTES;
  static constexpr int STAGES = (BUDGET / STAGE_BYTES) > 8 ? 8 : (BUDGET / STAGE_BYTES);
  static constexpr uint32_t TMEM_COLS = pow2_at_least(2 * BN);
  static constexpr size_t SMEM = 1024 + size_t(STAGES) * STAGE_BYTES + EPI_BYTES + AUX_BYTES + 256;
};

__device__ __forceinline__ void decode_tile2(const GemmArgs& a, int t, int bn, int& pi, int& m0, int& n0) {
  pi = (a.num_problems > 1 && t >= a.p[1].tile_begin) ? 1 : 0;
  const GemmProblem& P = a.p[pi];
  const int local = t - P.tile_begin;
  m0 = (local % P.tiles_m) * 256;
  n0 = (local / P.tiles_m) * bn;
}

// Work item w: a whole tile, or one of the tail_split column slices of a tail tile.
// Each output element is still one MMA chain over the whole K, so its value does
// not depend on which kind of item computed it.
__device__ __forceinline__ void decode_item2(const GemmArgs& a, int w, int bn, int& pi, int& m0, int& n0,
                                             int& width) {
  int t = w, sub = 0;
  width = bn;
  if (w >= a.tail_begin) {
    const int q = w - a.tail_begin;
    t = a.tail_begin + q / a.tail_split;
    sub = q - (q / a.tail_split) * a.tail_split;
    width = bn / a.tail_split;
  }
  decode_tile2(a, t, bn, pi, m0, n0);
  n0 += sub * width;
}

// Abort path of the CTA-pair producer (leader, one thread): make every stage load
// either CTA issued land before the pair leaves.  L and R are the stage loads the
// leader and rank 1 issued, in the same (tile, k block) order; a use the leader
// armed but rank 1 never filled has its missing bytes counted as arrived, a use
// rank 1 filled but the leader never armed is armed for rank 1's bytes alone.  A
// CTA issues use i only once use i - STAGES has been consumed, so every use still
// outstanding lies in [max(L, R) - STAGES, max(L, R)) and is its stage's last.
template <int STAGES, class UseBytes>
__device__ __forceinline__ void drain_pair_stages(uint64_t* full, UseBytes use_bytes, uint32_t L, uint32_t R) {
  const uint32_t hi = L > R ? L : R;
  for (uint32_t i = hi > (uint32_t)STAGES ? hi - STAGES : 0; i < hi; ++i) {
    const uint32_t s = i % STAGES, par = (i / STAGES) & 1;
    if (i >= L)
      mbar_expect_tx(&full[s], use_bytes(i));
    else if (i >= R)
      mbar_complete_tx(&full[s], use_bytes(i));
    mbar_wait_drain(&full[s], par);
  }
}

// One CTA's bytes in stage use i of this pair (a column slice loads a narrower B box).
__device__ __forceinline__ uint32_t pair_use_bytes(const GemmArgs& a, int pair, int npairs, uint32_t i, int bn,
                                                   uint32_t a_bytes, uint32_t b_bytes, int bk) {
  for (int t = pair; t < a.total_items; t += npairs) {
    int pi, m0, n0, width;
    decode_item2(a, t, bn, pi, m0, n0, width);
    const uint32_t kb = (uint32_t)(a.p[pi].K / bk);
    if (i < kb) return a_bytes + (width == bn ? b_bytes : (uint32_t)(width / 2) * 128u);
    i -= kb;
  }
  return a_bytes + b_bytes;
}

template <int BN, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Gemm2Cfg<BN, EPI>::THREADS, 1)
    gemm2_tc_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                    const __grid_constant__ CUtensorMap tmC0, const __grid_constant__ CUtensorMap tmC1,
                    const __grid_constant__ CUtensorMap tmB0n, const __grid_constant__ CUtensorMap tmB1n,
                    const __grid_constant__ GemmArgs args) {
  using C = Gemm2Cfg<BN, EPI>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * C::A_BYTES;
  uint8_t* sEpi = sB + STAGES * C::B_BYTES;
  float* sAux = reinterpret_cast<float*>(sEpi + C::EPI_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(sEpi + C::EPI_BYTES + C::AUX_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;            // leader's MMA completion after an abort
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  uint32_t* peer_issued = tmem_slot + 1;   // leader: stage loads rank 1 issued

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * C::EPI_WARPS);
    }
    mbar_init(drain, 1);
    *peer_issued = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmB0);
    if (args.num_problems > 1) {
      tma_prefetch_desc(&tmA1);
      tma_prefetch_desc(&tmB1);
    }
    if (args.tail_split > 1) {
      tma_prefetch_desc(&tmB0n);
      if (args.num_problems > 1) tma_prefetch_desc(&tmB1n);
    }
  }
  if constexpr (EPI == EPI_QKV) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) {
      const GemmProblem& P = args.p[(i >> 7) < args.num_problems ? (i >> 7) : 0];
      sAux[i] = (i & 64) ? P.gain_k[i & 63] : P.gain_q[i & 63];
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();          // both CTAs' barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Programmatic dependent launch: only the producer and the epilogue warps touch memory
  // that kernels ahead in the stream write (the A operand; outputs, gates, biases), so
  // only they wait for those kernels; the producer first issues the weight (B) loads of
  // its first stages, which depend on no kernel.
  grid_launch_dependents();

  uint32_t prod_issued = 0;    // producer thread: stage loads issued
  bool prod_ok = true;
  if (warp == 0) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      // the first item's first stages (each stage's first use: nothing to wait for) get
      // their B tiles now, their A tiles once the kernels ahead have finished
      int npre = 0;
      if (pair < args.total_items) {
        int pi, m0, n0, width;
        decode_item2(args, pair, BN, pi, m0, n0, width);
        const bool slice = width < BN;
        const CUtensorMap* mB = slice ? (pi ? &tmB1n : &tmB0n) : (pi ? &tmB1 : &tmB0);
        const uint32_t bytes = C::A_BYTES + (slice ? (uint32_t)(width / 2) * 128u : C::B_BYTES);
        const int kblocks = args.p[pi].K / C::BK;
        npre = kblocks < STAGES ? kblocks : STAGES;
        for (int kb = 0; kb < npre; ++kb) {
          if (rank == 0) mbar_expect_tx(&full[kb], 2 * bytes);
          tma_load_2d_pair(sB + kb * C::B_BYTES, mB, &full[kb], kb * C::BK, n0 + (width / 2) * (int)rank);
        }
      }
      grid_dependency_wait();
      for (int t = pair; t < args.total_items && ok; t += npairs) {
        int pi, m0, n0, width;
        decode_item2(args, t, BN, pi, m0, n0, width);
        const bool slice = width < BN;
        const CUtensorMap* mA = pi ? &tmA1 : &tmA0;
        const CUtensorMap* mB = slice ? (pi ? &tmB1n : &tmB0n) : (pi ? &tmB1 : &tmB0);
        const uint32_t bytes = C::A_BYTES + (slice ? (uint32_t)(width / 2) * 128u : C::B_BYTES);
        const int kblocks = args.p[pi].K / C::BK;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (t == pair && kb < npre) {   // armed and B issued above
            tma_load_2d_pair(sA + stage * C::A_BYTES, mA, &full[stage], kb * C::BK, m0 + 128 * (int)rank);
            ++prod_issued;
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1;
            }
            continue;
          }
          if (!mbar_wait(&empty[stage], phase ^ 1, args.err)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_expect_tx(&full[stage], 2 * bytes);
          tma_load_2d_pair(sA + stage * C::A_BYTES, mA, &full[stage], kb * C::BK, m0 + 128 * (int)rank);
          // a column slice loads its own width / 2 rows through the narrow map
          tma_load_2d_pair(sB + stage * C::B_BYTES, mB, &full[stage], kb * C::BK, n0 + (width / 2) * (int)rank);
          ++prod_issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      prod_ok = ok;
      // the leader reconciles both CTAs' loads if the pair aborts
      if (rank == 1) st_shared_cluster_u32(mapa_shared(smem_u32(peer_issued), 0), prod_issued);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      uint32_t stage = 0, phase = 0;
      int li = 0;
      bool ok = true;
      for (int t = pair; t < args.total_items && ok; t += npairs, ++li) {
        int pi, m0, n0, width;
        decode_item2(args, t, BN, pi, m0, n0, width);
        const uint32_t idesc = umma_idesc_bf16(256, width);
        const int kblocks = args.p[pi].K / C::BK;
        const uint32_t acc = li & 1;
        const uint32_t use = li >> 1;
        if (!mbar_wait_sleep(&tempty[acc], (use & 1) ^ 1, args.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_sleep(&full[stage], phase, args.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = umma_desc_sw128(smem_u32(sA + stage * C::A_BYTES));
          const uint64_t bd = umma_desc_sw128(smem_u32(sB + stage * C::B_BYTES));
#pragma unroll
          for (int k = 0; k < C::BK / 16; ++k)
            umma_bf16_pair(d_tmem, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          umma_commit_pair(&empty[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_pair(&tfull[acc], 0x3);
      }
      if (!ok) umma_drain_pair(drain);   // no UMMA of the pair still runs when the pair leaves
    }
    __syncwarp();
  } else {
    grid_dependency_wait();                       // gates, biases and outputs follow earlier kernels
    const int quarter = warp & 3;                 // TMEM lanes 32 quarter .. + 31
    const int part = (warp - 2) >> 2;             // which part of the tile's columns
    uint8_t* slots = sEpi + (warp - 2) * C::EPI_SLOTS * C::EPI_SLOT;
    uint32_t slot = 0;
    const uint32_t leader_tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
    int li = 0;
    for (int t = pair; t < args.total_items; t += npairs, ++li) {
      int pi, m0, n0, width;
      decode_item2(args, t, BN, pi, m0, n0, width);
      const uint32_t acc = li & 1;
      const uint32_t use = li >> 1;
      const int row0 = m0 + 128 * (int)rank + quarter * 32;
      float4 pre[16];
      epilogue_prefetch<BN, EPI>(args.p[pi], row0 + lane, n0, part, C::EPI_PARTS, pre, width);
      if (!mbar_wait(&tfull[acc], use & 1, args.err)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16) + acc * BN;
      epilogue_tile<BN, EPI, C::EPI_SLOTS>(args.p[pi], pi ? &tmC1 : &tmC0, row0 + lane, row0, n0, taddr, slots,
                                           slot, sAux + pi * 128, pre, part, C::EPI_PARTS, width);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_tempty0 + acc * 8);
    }
    if constexpr (C::EPI_BYTES > 0) {
      if (lane == 0) bulk_wait_read<0>();      // as above
      __syncwarp();
    }
  }

  tc_fence_before();
  cluster_sync_all();          // every role of both CTAs has left its loop; rank 1's count is in place
  if (warp == 0 && lane == 0 && rank == 0 && (!prod_ok || err_raised(args.err)))
    drain_pair_stages<STAGES>(
        full,
        [&](uint32_t i) { return pair_use_bytes(args, pair, npairs, i, BN, C::A_BYTES, C::B_BYTES, C::BK); },
        prod_issued, *peer_issued);
  cluster_sync_all();          // no MMA, TMA or remote arrive of the pair is still in flight
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace lens
