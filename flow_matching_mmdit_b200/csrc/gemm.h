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

// Fill tile counts of args.p[0..num_problems) for tile width bn and launch the
// persistent kernel (grid = min(tiles, sms)).  (bn, epi) must be an instantiated pair.
// C0 / C1 are the output maps of the TMA-store epilogues (EPI_F32, EPI_RESID,
// EPI_SWIGLU; encode_tmap_out), ignored by the others.
cudaError_t launch_gemm(int bn, int epi, const CUtensorMap* A0, const CUtensorMap* B0, const CUtensorMap* A1,
                        const CUtensorMap* B1, const CUtensorMap* C0, const CUtensorMap* C1, GemmArgs& args, int sms,
                        cudaStream_t st);

// The same on 256 x bn tiles computed by CTA pairs (cta_group::2): A maps keep a box
// of 128 rows, B maps need a box of bn / 2 rows.  Grid = 2 x min(tiles, sms / 2).
cudaError_t launch_gemm_pair(int bn, int epi, const CUtensorMap* A0, const CUtensorMap* B0, const CUtensorMap* A1,
                             const CUtensorMap* B1, const CUtensorMap* C0, const CUtensorMap* C1, GemmArgs& args,
                             int sms, cudaStream_t st);

}  // namespace lens
