// Host interface of the tcgen05 GEMM (see gemm_tc.cuh for the kernel).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lens {

struct GemmArgs;

// 2D bf16 tensor map over a row-major [rows, cols] matrix (K = cols contiguous),
// box = 64 columns x box_rows rows, 128-byte swizzle, zero fill out of bounds.
bool encode_tmap_bf16(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint64_t row_stride_elems,
                      uint32_t box_rows);

// 2D tensor map of fp32 (elem_bytes 4) or bf16 (2) rows used as a TMA store /
// reduce target: box = (128 / elem_bytes) columns x 32 rows, 128-byte swizzle.
bool encode_tmap_out(CUtensorMap* m, const void* ptr, int elem_bytes, uint64_t rows, uint64_t cols,
                     uint64_t row_stride_elems);

// 3D bf16 tensor map over [d2][d1][d0] (d0 contiguous, d0 * 2 bytes a multiple of 16),
// box = d0 x box_rows x 1, 128-byte swizzle, zero fill out of bounds.
bool encode_tmap_bf16_3d(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box_rows);

// 4-bit weights (int4 weight-only path, w4.cu).  A quantized [rows, k] matrix is
//   codes  uint8 [rows, k / 2]: 32-bit word w of a row holds the codes of k in
//          [8w, 8w + 8); the code of k = 8w + 2j sits in bits [4j, 4j + 4), that of
//          k = 8w + 2j + 1 in bits [16 + 4j, 20 + 4j) (j = 0..3), so one shift and
//          mask gives the bf16 pair (128 + q_2j, 128 + q_2j+1) after an OR with 0x43004300
//   scales uint32 [k / 64, rows]: group g of row r at [g][r], bf16 scale in the low
//          half, bf16 bias in the high half; w = scale * q + bias
// codes map: box 32 bytes (one 64-wide k block) x box_rows rows, no swizzle;
// scales map: box box_rows x 1 group (box_rows a multiple of 4).
bool encode_tmap_w4_codes(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t k, uint32_t box_rows);
bool encode_tmap_w4_scales(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t k, uint32_t box_rows);

// Quantize bf16 w [rows, k] (k a multiple of 64) into the layout above: per group of
// 64 along k, scale = bf16((max - min) / 15), bias = bf16(min), code =
// clamp(rint((w - bias) / scale), 0, 15) in fp32 (0 where scale = 0).  The scales of
// group g, row r go to scales[g * scale_ld + r] (scale_ld >= rows: the rows of a
// larger matrix this one is a row slice of, with scales pre-offset by its first row).
cudaError_t launch_quantize_w4(const void* w_bf16, int64_t rows, int64_t k, uint8_t* codes, uint32_t* scales,
                               int64_t scale_ld, cudaStream_t st);

// GEMM with one 4-bit operand, dequantized in shared memory.  quant_a = false: B
// (the N side, weights [N, K]) is 4-bit, A0/A1 are bf16 maps as for launch_gemm;
// quant_a = true: A (the M side, weights of the swap-AB modulation GEMM) is 4-bit
// and B0 is a bf16 map.  Q*/S* are the codes / scales maps (box rows = bn for B,
// 128 for A).  bm = 128, or 256 with a 4-bit B (one widened B tile feeds two 128-row
// MMAs; instantiated for bn = 128).  Same problems, epilogues and output maps as
// launch_gemm.
cudaError_t launch_gemm_w4(int bm, int bn, int epi, bool quant_a, const CUtensorMap* A0, const CUtensorMap* B0,
                           const CUtensorMap* Q0, const CUtensorMap* S0, const CUtensorMap* A1, const CUtensorMap* B1,
                           const CUtensorMap* Q1, const CUtensorMap* S1, const CUtensorMap* C0, const CUtensorMap* C1,
                           GemmArgs& args, int sms, cudaStream_t st);

// Fill tile counts of args.p[0..num_problems) for tile width bn and launch the
// persistent kernel (grid = min(tiles, sms)).  (bn, epi) must be an instantiated pair.
// C0 / C1 are the output maps of the TMA-store epilogues (EPI_F32, EPI_RESID,
// EPI_SWIGLU; encode_tmap_out), ignored by the others.
cudaError_t launch_gemm(int bn, int epi, const CUtensorMap* A0, const CUtensorMap* B0, const CUtensorMap* A1,
                        const CUtensorMap* B1, const CUtensorMap* C0, const CUtensorMap* C1, GemmArgs& args, int sms,
                        cudaStream_t st);

// B maps of the same weights with boxes of bn / 4 and bn / 8 rows (index 0 and 1):
// the tail items of a pair launch cut into 2 or 4 column slices load only their own
// rows through them.  A null entry rules that split out.
struct NarrowB {
  const CUtensorMap* b0[2];
  const CUtensorMap* b1[2];
};

// The same on 256 x bn tiles computed by CTA pairs (cta_group::2): A maps keep a box
// of 128 rows, B maps need a box of bn / 2 rows.  Grid = 2 x min(tiles, sms / 2).
// With `narrow`, the last, partly filled round of tiles may run as column slices.
cudaError_t launch_gemm_pair(int bn, int epi, const CUtensorMap* A0, const CUtensorMap* B0, const CUtensorMap* A1,
                             const CUtensorMap* B1, const CUtensorMap* C0, const CUtensorMap* C1, GemmArgs& args,
                             int sms, cudaStream_t st, const NarrowB* narrow = nullptr);

}  // namespace lens
