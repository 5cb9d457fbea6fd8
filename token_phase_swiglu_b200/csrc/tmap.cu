// TMA tensor-map encoding through cuTensorMapEncodeTiled, fetched from the
// driver once per process with cudaGetDriverEntryPointByVersion (no -lcuda).
#include "tmap.h"

#include <cudaTypedefs.h>

#include <mutex>

namespace fmlp {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
cudaError_t g_encode_err = cudaSuccess;
std::once_flag g_once;

cudaError_t encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::call_once(g_once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    g_encode_err = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                                    cudaEnableDefault, &q);
    if (g_encode_err == cudaSuccess && q != cudaDriverEntryPointSuccess)
      g_encode_err = cudaErrorNotSupported;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  *fn = g_encode;
  return g_encode_err;
}

}  // namespace

cudaError_t encode_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                                uint64_t row_bytes, uint32_t box_rows, uint32_t box_cols,
                                CUtensorMapSwizzle swizzle) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  cudaError_t e = encoder(&fn);
  if (e != cudaSuccess) return e;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t elem[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_tmap_blocks_bf16(CUtensorMap* map, const void* base, uint64_t rows,
                                    uint64_t cols, uint64_t row_bytes, uint32_t block_cols,
                                    uint32_t box_rows, uint32_t box_blocks,
                                    CUtensorMapSwizzle swizzle) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  cudaError_t e = encoder(&fn);
  if (e != cudaSuccess) return e;
  if (block_cols == 0 || cols % block_cols != 0) return cudaErrorInvalidValue;
  const cuuint64_t dims[3] = {block_cols, rows, cols / block_cols};
  const cuuint64_t strides[2] = {row_bytes, (cuuint64_t)block_cols * 2};
  const cuuint32_t box[3] = {block_cols, box_rows, box_blocks};
  const cuuint32_t elem[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_tmap_kblocks_bf16(CUtensorMap* map, const void* base, uint64_t rows,
                                     uint64_t cols, uint64_t row_bytes, uint32_t box_rows,
                                     uint32_t box_kblocks) {
  return encode_tmap_blocks_bf16(map, base, rows, cols, row_bytes, 64, box_rows, box_kblocks,
                                 CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace fmlp
