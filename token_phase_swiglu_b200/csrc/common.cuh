// Device helpers shared by the fused-MLP kernels (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fmlp {

// ---------------------------------------------------------------------------
// Programmatic dependent launch (grid dependency control).
//
// A kernel launched with cudaLaunchAttributeProgrammaticStreamSerialization
// may start while the previous kernel on the stream is still running.  It
// must call grid_dependency_wait() before touching anything that kernel
// writes; everything before the wait (weight prefetches) overlaps the tail
// of the previous kernel.  grid_launch_dependents() lets the next kernel's
// CTAs be scheduled once every CTA of this grid has issued it.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Bulk L2 prefetch of a contiguous byte range (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// L2 policy for read-once weights: evict first, so streamed weights do not
// push the reused activations out of L2.
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 16-byte streaming load of read-once weights: no L1 allocation, L2 hint.
__device__ __forceinline__ uint4 ld_stream(const void* ptr, uint64_t policy) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(ptr), "l"(policy));
  return v;
}

// 16-byte load of small, reused operands (activations): normal caching.
__device__ __forceinline__ uint4 ld_keep(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// bf16 pair in a 32-bit word -> two floats (exact: bf16 is the top half of f32).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// SiLU(g) * u in f32.  For g << 0, expf(-g) overflows to +inf and g/inf = -0.
__device__ __forceinline__ float silu_mul(float g, float u) {
  return g / (1.0f + expf(-g)) * u;
}

}  // namespace fmlp
