// Host side of the tcgen05 GEMM: tensor-map encoding and the launch dispatcher.
#include <mutex>

#include "gemm.h"
#include "gemm_tc.cuh"
#include "smem_attr.h"

namespace lens {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

template <int BN, int EPI>
cudaError_t launch_one(const CUtensorMap& A0, const CUtensorMap& B0, const CUtensorMap& A1, const CUtensorMap& B1,
                       const CUtensorMap& C0, const CUtensorMap& C1, const GemmArgs& args, int sms, cudaStream_t st) {
  using C = GemmCfg<BN, EPI>;
  static std::atomic<uint64_t> attr{0};
  {
    const cudaError_t e = ensure_smem_limit(gemm_tc_kernel<BN, EPI>, (int)C::SMEM, attr);
    if (e != cudaSuccess) return e;
  }
  const int grid = args.total_tiles < sms ? args.total_tiles : sms;
  return launch_pdl(gemm_tc_kernel<BN, EPI>, dim3(grid), dim3(192), C::SMEM, st, A0, B0, A1, B1, C0, C1, args);
}

// Tail of a CTA-pair launch: the last round of whole tiles (T mod pairs of them) would
// leave the other pairs idle for a whole tile time.  Split each of those tiles into s
// column slices (s = 4 or 2, the largest whose slices all fit in one round, whose
// width the MMA (multiple of 16) and the epilogue's unit allow: 32 columns for the
// fp32 and residual epilogues, a 64-column head for QKV, a 128-column w1|w3 group for
// SwiGLU, and for which narrow B maps were given).  Every output element is still one
// MMA chain over the whole K.  Returns the index into NarrowB (-1: no split).
static int plan_tail(GemmArgs& a, int pairs, int bn, int epi, const NarrowB* nb) {
  const int rounds = a.total_tiles / pairs;
  const int tail = a.total_tiles - rounds * pairs;
  if (!nb || rounds < 1 || tail == 0) return -1;
  const int unit = epi == EPI_SWIGLU ? 128 : (epi == EPI_QKV ? 64 : 32);
  for (int i = 1; i >= 0; --i) {
    const int s = 2 << i;
    const int w = bn / s;
    if (bn % s || w % unit || w % 16 || tail * s > pairs) continue;
    if (!nb->b0[i] || (a.num_problems > 1 && !nb->b1[i])) continue;
    a.tail_begin = rounds * pairs;
    a.tail_split = s;
    a.total_items = a.tail_begin + tail * s;
    return i;
  }
  return -1;
}

template <int BN, int EPI>
cudaError_t launch_pair(const CUtensorMap& A0, const CUtensorMap& B0, const CUtensorMap& A1, const CUtensorMap& B1,
                        const CUtensorMap& C0, const CUtensorMap& C1, const GemmArgs& args, int sms,
                        cudaStream_t st, const NarrowB* nb) {
  using C = Gemm2Cfg<BN, EPI>;
  static std::atomic<uint64_t> attr{0};
  {
    const cudaError_t e = ensure_smem_limit(gemm2_tc_kernel<BN, EPI>, (int)C::SMEM, attr);
    if (e != cudaSuccess) return e;
  }
  const int pairs = args.total_tiles < sms / 2 ? args.total_tiles : sms / 2;
  GemmArgs a = args;
  const int n = plan_tail(a, pairs, BN, EPI, nb);
  const CUtensorMap& B0n = n >= 0 ? *nb->b0[n] : B0;
  const CUtensorMap& B1n = n >= 0 && a.num_problems > 1 ? *nb->b1[n] : B0n;
  return launch_pdl(gemm2_tc_kernel<BN, EPI>, dim3(2 * pairs), dim3(C::THREADS), C::SMEM, st, A0, B0, A1, B1, C0,
                    C1, B0n, B1n, a);
}

}  // namespace

bool encode_tmap_bf16(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint64_t row_stride_elems,
                      uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0 || cols == 0) return false;
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || (row_stride_elems * 2) % 16 || box_rows == 0 || box_rows > 256)
    return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_stride_elems * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tmap_out(CUtensorMap* m, const void* ptr, int elem_bytes, uint64_t rows, uint64_t cols,
                     uint64_t row_stride_elems) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0 || cols == 0 || (elem_bytes != 2 && elem_bytes != 4)) return false;
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || (row_stride_elems * elem_bytes) % 16) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_stride_elems * elem_bytes};
  const cuuint32_t box[2] = {(cuuint32_t)(128 / elem_bytes), 32};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, elem_bytes == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tmap_bf16_3d(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || d0 == 0 || d1 == 0 || d2 == 0) return false;
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || (d0 * 2) % 16 || d0 * 2 > 128 || box_rows == 0 || box_rows > 256)
    return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  const cuuint32_t box[3] = {(cuuint32_t)d0, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tmap_w4_codes(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t k, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0 || k == 0 || k % 64 || box_rows == 0 || box_rows > 256) return false;
  if (reinterpret_cast<uintptr_t>(ptr) & 15) return false;
  const cuuint64_t dims[2] = {k / 2, rows};
  const cuuint64_t strides[1] = {k / 2};
  const cuuint32_t box[2] = {32, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tmap_w4_scales(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t k, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0 || rows % 4 || k == 0 || k % 64 || box_rows == 0 || box_rows > 256 || box_rows % 4)
    return false;
  if (reinterpret_cast<uintptr_t>(ptr) & 15) return false;
  const cuuint64_t dims[2] = {rows, k / 64};
  const cuuint64_t strides[1] = {rows * 4};
  const cuuint32_t box[2] = {box_rows, 1};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

void finalize_problems(GemmArgs& a, int bn, int bm) {
  int begin = 0;
  for (int i = 0; i < a.num_problems; ++i) {
    GemmProblem& p = a.p[i];
    p.tiles_m = (p.M + bm - 1) / bm;
    p.tiles_n = (p.N + bn - 1) / bn;
    p.tile_begin = begin;
    begin += p.tiles_m * p.tiles_n;
  }
  a.total_tiles = begin;
  a.tail_begin = begin;
  a.tail_split = 1;
  a.total_items = begin;
}

cudaError_t launch_gemm(int bn, int epi, const CUtensorMap* A0, const CUtensorMap* B0, const CUtensorMap* A1,
                        const CUtensorMap* B1, const CUtensorMap* C0, const CUtensorMap* C1, GemmArgs& args, int sms,
                        cudaStream_t st) {
  finalize_problems(args, bn, 128);
  if (args.total_tiles == 0) return cudaSuccess;
  if ((epi == EPI_F32 || epi == EPI_RESID || epi == EPI_SWIGLU) && (!C0 || (args.num_problems > 1 && !C1)))
    return cudaErrorInvalidValue;
  const CUtensorMap& a1 = A1 ? *A1 : *A0;
  const CUtensorMap& b1 = B1 ? *B1 : *B0;
  const CUtensorMap& c0 = C0 ? *C0 : *A0;
  const CUtensorMap& c1 = C1 ? *C1 : c0;
#define LENS_GEMM_CASE(BN_, EPI_) \
  if (bn == BN_ && epi == EPI_) return launch_one<BN_, EPI_>(*A0, *B0, a1, b1, c0, c1, args, sms, st);
  LENS_GEMM_CASE(256, EPI_F32)
  LENS_GEMM_CASE(192, EPI_F32)
  LENS_GEMM_CASE(128, EPI_F32)
  LENS_GEMM_CASE(64, EPI_F32)
  LENS_GEMM_CASE(32, EPI_F32)
  LENS_GEMM_CASE(256, EPI_RESID)
  LENS_GEMM_CASE(192, EPI_RESID)
  LENS_GEMM_CASE(128, EPI_RESID)
  LENS_GEMM_CASE(256, EPI_SWIGLU)
  LENS_GEMM_CASE(256, EPI_QKV)
  LENS_GEMM_CASE(192, EPI_QKV)
  LENS_GEMM_CASE(16, EPI_F32_T)
  LENS_GEMM_CASE(32, EPI_F32_T)
  LENS_GEMM_CASE(64, EPI_F32_T)
#undef LENS_GEMM_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemm_pair(int bn, int epi, const CUtensorMap* A0, const CUtensorMap* B0, const CUtensorMap* A1,
                             const CUtensorMap* B1, const CUtensorMap* C0, const CUtensorMap* C1, GemmArgs& args,
                             int sms, cudaStream_t st, const NarrowB* narrow) {
  finalize_problems(args, bn, 256);
  if (args.total_tiles == 0) return cudaSuccess;
  if ((epi == EPI_F32 || epi == EPI_RESID || epi == EPI_SWIGLU) && (!C0 || (args.num_problems > 1 && !C1)))
    return cudaErrorInvalidValue;
  const CUtensorMap& a1 = A1 ? *A1 : *A0;
  const CUtensorMap& b1 = B1 ? *B1 : *B0;
  const CUtensorMap& c0 = C0 ? *C0 : *A0;
  const CUtensorMap& c1 = C1 ? *C1 : c0;
#define LENS_GEMM2_CASE(BN_, EPI_) \
  if (bn == BN_ && epi == EPI_) return launch_pair<BN_, EPI_>(*A0, *B0, a1, b1, c0, c1, args, sms, st, narrow);
  LENS_GEMM2_CASE(256, EPI_F32)
  LENS_GEMM2_CASE(128, EPI_F32)
  LENS_GEMM2_CASE(192, EPI_RESID)
  LENS_GEMM2_CASE(256, EPI_RESID)
  LENS_GEMM2_CASE(256, EPI_SWIGLU)
  LENS_GEMM2_CASE(192, EPI_QKV)
  LENS_GEMM2_CASE(256, EPI_QKV)
#undef LENS_GEMM2_CASE
  return cudaErrorInvalidValue;
}

}  // namespace lens
