// TMA tensor-map encoding (driver entry point looked up once through the runtime).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fmlp {

// 2-D bf16 tensor map over a row-major matrix of `rows` x `cols` elements
// (row stride `row_bytes`), copying boxes of box_rows x box_cols with no
// swizzle (or the given swizzle); out-of-range elements read as zero.
cudaError_t encode_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                                uint64_t row_bytes, uint32_t box_rows, uint32_t box_cols,
                                CUtensorMapSwizzle swizzle);

// 3-D bf16 tensor map that views a row-major `rows` x `cols` matrix (row
// stride `row_bytes`, cols % 64 == 0) as k-blocks of 64 columns: dimension 0
// is the column inside a k-block, 1 the row, 2 the k-block (stride 128
// bytes).  A box of box_rows x 64 x box_kblocks lands in shared memory as
// box_kblocks consecutive box_rows x 128-byte tiles, each with the 128-byte
// swizzle; k-blocks past the end read as zero.
cudaError_t encode_tmap_kblocks_bf16(CUtensorMap* map, const void* base, uint64_t rows,
                                     uint64_t cols, uint64_t row_bytes, uint32_t box_rows,
                                     uint32_t box_kblocks);

// The same view with blocks of block_cols columns (32 with the 64-byte
// swizzle, 64 with the 128-byte one): a box of box_rows x block_cols x
// box_blocks lands as box_blocks consecutive box_rows x (2 block_cols)-byte
// tiles.
cudaError_t encode_tmap_blocks_bf16(CUtensorMap* map, const void* base, uint64_t rows,
                                    uint64_t cols, uint64_t row_bytes, uint32_t block_cols,
                                    uint32_t box_rows, uint32_t box_blocks,
                                    CUtensorMapSwizzle swizzle);

}  // namespace fmlp
