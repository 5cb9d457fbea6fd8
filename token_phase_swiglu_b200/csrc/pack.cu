// Step a0: interleave W_gate and W_up rows at tile granularity T.
//
// "FastTPS: An Optimized Method for LLM Token Phase for AI Accelerators"
// (xllm-io review), section 三 component 3: the gate and up projections are
// interleaved so one matmul produces both; "CUDAカーネル融合で推論が最大10%高速化"
// (blog.cecily.jp), llama.cpp PR #29948 paragraph: gate/up rows alternate.
// packed[2T t + j] = W_gate[T t + j], packed[2T t + T + j] = W_up[T t + j].
// A pure row permutation: one CTA copies whole rows as 16-byte vectors.
#include "common.cuh"
#include "internal.h"

namespace fmlp {
namespace {

__global__ void __launch_bounds__(256)
pack_rows(const uint4* __restrict__ Wg, const uint4* __restrict__ Wu, int64_t dv, int64_t I,
          int T, uint4* __restrict__ P) {
  for (int64_t row = blockIdx.x; row < 2 * I; row += gridDim.x) {
    const int64_t t = row / (2 * T);
    const int64_t w = row - t * 2 * T;
    const uint4* src = (w < T) ? Wg + (t * T + w) * dv : Wu + (t * T + w - T) * dv;
    uint4* dst = P + row * dv;
    for (int64_t c = threadIdx.x; c < dv; c += blockDim.x) dst[c] = src[c];
  }
}

}  // namespace

cudaError_t launch_pack(const void* W_gate, const void* W_up, int64_t d, int64_t I, int T,
                        void* packed, cudaStream_t stream) {
  const int64_t rows = 2 * I;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(rows < 65535 * 4 ? rows : 65535 * 4));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  // cudaLaunchKernelEx reports this launch's own error (no stale sticky state)
  cudaError_t e = cudaLaunchKernelEx(&cfg, pack_rows, (const uint4*)W_gate, (const uint4*)W_up,
                                     d / 8, I, T, (uint4*)packed);
  if (e == cudaSuccess) note_launches(1);
  return e;
}

}  // namespace fmlp
