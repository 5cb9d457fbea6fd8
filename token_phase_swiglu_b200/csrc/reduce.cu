// Sum of partial MLP outputs (the reduction step of a tensor-parallel MLP).
//
// When the intermediate dimension is split over ranks, each rank's
// fmlp_forward on its columns gives a partial out_r, and the block's output
// is their sum (Eq(1) of "FastTPS: An Optimized Method for LLM Token Phase
// for AI Accelerators", xllm-io review, section 三, is linear in the columns
// of a; the tensor-parallel split of "Together AI 的推测解码内核融合优化",
// blog.hotdry.top, reduces the partial outputs before the next norm).  The
// kernel reads the n partials through plain loads, so a partial may live in
// another GPU's memory mapped into this one (a peer pointer): each rank then
// sums its own copy of the output straight over NVLink, with no copy through
// a staging buffer and no multicast.
#include "common.cuh"
#include "internal.h"

#include <algorithm>

namespace fmlp {
namespace {

struct SumParams {
  const float* parts[kMaxPartials];
  int n;
  const __nv_bfloat16* residual;  // [M x d] or null
  float* out_f32;                 // [M x d] or null
  __nv_bfloat16* out_bf16;        // [M x d] or null
  int64_t n4;                     // M * d / 4
};

__global__ void __launch_bounds__(256) sum_partials(const __grid_constant__ SumParams p) {
  grid_launch_dependents();
  grid_dependency_wait();  // the partials and the residual come from earlier work
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < p.n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p.residual) {
      const uint2 r = __ldg(reinterpret_cast<const uint2*>(p.residual) + i);
      s = make_float4(bf16lo(r.x), bf16hi(r.x), bf16lo(r.y), bf16hi(r.y));
    }
    // rank order, so every rank sums in the same order and gets the same bits
    for (int r = 0; r < p.n; ++r) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(p.parts[r]) + i);
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    if (p.out_f32) reinterpret_cast<float4*>(p.out_f32)[i] = s;
    if (p.out_bf16) {
      uint2 w;
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w.x) : "f"(s.y), "f"(s.x));
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w.y) : "f"(s.w), "f"(s.z));
      reinterpret_cast<uint2*>(p.out_bf16)[i] = w;
    }
  }
}

}  // namespace

cudaError_t launch_sum_partials(const float* const* parts, int n, int64_t M, int64_t d,
                                const void* residual, float* out_f32, void* out_bf16,
                                const DeviceInfo& dev, cudaStream_t stream) {
  SumParams p = {};
  for (int r = 0; r < n; ++r) p.parts[r] = parts[r];
  p.n = n;
  p.residual = (const __nv_bfloat16*)residual;
  p.out_f32 = out_f32;
  p.out_bf16 = (__nv_bfloat16*)out_bf16;
  p.n4 = M * d / 4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::max<int64_t>(
      1, std::min<int64_t>((p.n4 + 255) / 256, 4 * dev.sm_count)));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, sum_partials, p);
  if (e == cudaSuccess) note_launches(1);
  return e;
}

}  // namespace fmlp
