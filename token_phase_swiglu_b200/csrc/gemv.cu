// CUDA-core weight-streaming kernels for decode-sized token counts.
//
// Gate-up (steps a1-a4) and down projection (a5-a6) of the MLP block in
// "FastTPS: An Optimized Method for LLM Token Phase for AI Accelerators"
// (xllm-io review), section 三 Eq(1) and Figure 4, for M <= 4 token rows at
// a time.  At these sizes the block is a matrix-vector product whose time is
// the time to stream the weights from HBM once: each warp owns whole rows,
// each lane issues 16-byte loads eight vectors deep per row (32-64 KB per SM
// in flight), activations sit in shared memory or L1, and the row dot
// products finish with warp shuffles.  Both kernels are launched with
// programmatic dependent launch: they prefetch their first weight rows into
// L2 before waiting for the previous kernel on the stream.
#include "common.cuh"
#include "internal.h"

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

namespace fmlp {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kVec = 8;          // bf16 per 16-byte vector
constexpr int kDepth = 8;        // vectors per row per lane in flight
constexpr int kStride = 32 * kVec;  // columns covered by one warp-wide vector load

__device__ __forceinline__ void unpack8(const uint4& v, float f[8]) {
  f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
  f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

__device__ __forceinline__ float dot8(const uint4& w, const float4& s0, const float4& s1, float acc) {
  acc = fmaf(bf16lo(w.x), s0.x, acc); acc = fmaf(bf16hi(w.x), s0.y, acc);
  acc = fmaf(bf16lo(w.y), s0.z, acc); acc = fmaf(bf16hi(w.y), s0.w, acc);
  acc = fmaf(bf16lo(w.z), s1.x, acc); acc = fmaf(bf16hi(w.z), s1.y, acc);
  acc = fmaf(bf16lo(w.w), s1.z, acc); acc = fmaf(bf16hi(w.w), s1.w, acc);
  return acc;
}

__device__ __forceinline__ float dot8bf(const uint4& w, const uint4& v, float acc) {
  acc = fmaf(bf16lo(w.x), bf16lo(v.x), acc); acc = fmaf(bf16hi(w.x), bf16hi(v.x), acc);
  acc = fmaf(bf16lo(w.y), bf16lo(v.y), acc); acc = fmaf(bf16hi(w.y), bf16hi(v.y), acc);
  acc = fmaf(bf16lo(w.z), bf16lo(v.z), acc); acc = fmaf(bf16hi(w.z), bf16hi(v.z), acc);
  acc = fmaf(bf16lo(w.w), bf16lo(v.w), acc); acc = fmaf(bf16hi(w.w), bf16hi(v.w), acc);
  return acc;
}

// Packed-row index of gate row i (its up row is T rows further on).
__device__ __forceinline__ int64_t gate_row(int i, int T) {
  const int t = i / T;
  return (int64_t)2 * T * t + (i - t * T);
}

// ---------------------------------------------------------------------------
// Fused RMSNorm -> interleaved gate-up contraction -> SiLU*up, MT token rows.
//
// Grid: x strides over the I gate/up pairs (one warp per pair at a time),
// y over chunks of MT token rows.  Shared memory holds s = x*gamma in f32
// (exact: the product of two bf16 values has at most 16 significant bits) for
// the chunk's rows; r = 1/sqrt(mean x^2 + eps) is applied in the epilogue,
// g = r * (P_gate . s), u = r * (P_up . s).
// ---------------------------------------------------------------------------
template <int MT>
__global__ void __launch_bounds__(kThreads)
gateup_swiglu_gemv(const __nv_bfloat16* __restrict__ x, int M,
                   const __nv_bfloat16* __restrict__ gamma, float eps,
                   const __nv_bfloat16* __restrict__ P, int T, int d, int I,
                   __nv_bfloat16* __restrict__ a) {
  extern __shared__ float4 smem4[];
  float* s = reinterpret_cast<float*>(smem4);  // [MT][d]
  __shared__ float red[kWarps][MT];
  __shared__ float rinv[MT];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * MT;
  const int mt = min(MT, M - m0);
  const int gw = blockIdx.x * kWarps + warp;
  const int nw = gridDim.x * kWarps;

  // Weights do not depend on the previous kernel: start pulling this warp's
  // first gate/up rows into L2 before the dependency wait.
  if (lane == 0 && gw < I) {
    const __nv_bfloat16* pg = P + gate_row(gw, T) * d;
    prefetch_l2_bulk(pg, (uint32_t)d * 2u);
    prefetch_l2_bulk(pg + (int64_t)T * d, (uint32_t)d * 2u);
  }
  grid_dependency_wait();
  grid_launch_dependents();

  // Stage s = x * gamma and the row sums of squares.
  float ss[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) ss[m] = 0.f;
  const int dv = d / kVec;
  for (int v = threadIdx.x; v < dv; v += kThreads) {
    float gf[8];
    unpack8(ld_keep(gamma + (int64_t)v * kVec), gf);
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float xf[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (m < mt) unpack8(ld_keep(x + (int64_t)(m0 + m) * d + (int64_t)v * kVec), xf);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss[m] = fmaf(xf[e], xf[e], ss[m]);
      float4* dst = reinterpret_cast<float4*>(s + (int64_t)m * d + (int64_t)v * kVec);
      dst[0] = make_float4(xf[0] * gf[0], xf[1] * gf[1], xf[2] * gf[2], xf[3] * gf[3]);
      dst[1] = make_float4(xf[4] * gf[4], xf[5] * gf[5], xf[6] * gf[6], xf[7] * gf[7]);
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const float t = warp_sum(ss[m]);
    if (lane == 0) red[warp][m] = t;
  }
  __syncthreads();
  if (threadIdx.x < MT) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += red[w][threadIdx.x];
    rinv[threadIdx.x] = 1.0f / sqrtf(t / (float)d + eps);
  }
  __syncthreads();

  const uint64_t pol = evict_first_policy();
  for (int i = gw; i < I; i += nw) {
    const __nv_bfloat16* pg = P + gate_row(i, T) * d;
    const __nv_bfloat16* pu = pg + (int64_t)T * d;
    float ag[MT], au[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) ag[m] = au[m] = 0.f;

    for (int k0 = lane * kVec; k0 < d; k0 += kStride * kDepth) {
      uint4 wg[kDepth], wu[kDepth];
#pragma unroll
      for (int u = 0; u < kDepth; ++u) {
        const int k = k0 + u * kStride;
        if (k < d) {
          wg[u] = ld_stream(pg + k, pol);
          wu[u] = ld_stream(pu + k, pol);
        } else {
          wg[u] = wu[u] = make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int u = 0; u < kDepth; ++u) {
        const int k = k0 + u * kStride;
        if (k < d) {
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const float4* sp = reinterpret_cast<const float4*>(s + (int64_t)m * d + k);
            const float4 s0 = sp[0], s1 = sp[1];
            ag[m] = dot8(wg[u], s0, s1, ag[m]);
            au[m] = dot8(wu[u], s0, s1, au[m]);
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float g = warp_sum(ag[m]);
      const float u = warp_sum(au[m]);
      if (lane == m && m < mt) {
        const float r = rinv[m];
        a[(int64_t)(m0 + m) * I + i] = __float2bfloat16_rn(silu_mul(g * r, u * r));
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Down projection (+ residual), MT token rows: out[m, n] = W_down[n, :] . a[m, :].
// One warp per output column n at a time; a (bf16, written by the gate-up
// kernel) is read through L1, where every warp of the CTA reuses it.
// ---------------------------------------------------------------------------
template <int MT>
__global__ void __launch_bounds__(kThreads)
down_gemv(const __nv_bfloat16* __restrict__ a, int M, const __nv_bfloat16* __restrict__ Wd,
          int d, int I, const __nv_bfloat16* __restrict__ residual, float* __restrict__ out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * MT;
  const int mt = min(MT, M - m0);
  const int gw = blockIdx.x * kWarps + warp;
  const int nw = gridDim.x * kWarps;

  if (lane == 0 && gw < d) prefetch_l2_bulk(Wd + (int64_t)gw * I, (uint32_t)I * 2u);
  grid_dependency_wait();
  grid_launch_dependents();

  const uint64_t pol = evict_first_policy();
  for (int n = gw; n < d; n += nw) {
    const __nv_bfloat16* w = Wd + (int64_t)n * I;
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.f;
    for (int k0 = lane * kVec; k0 < I; k0 += kStride * kDepth) {
      uint4 wv[kDepth];
#pragma unroll
      for (int u = 0; u < kDepth; ++u) {
        const int k = k0 + u * kStride;
        wv[u] = (k < I) ? ld_stream(w + k, pol) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kDepth; ++u) {
        const int k = k0 + u * kStride;
        if (k < I) {
#pragma unroll
          for (int m = 0; m < MT; ++m)
            if (m < mt) acc[m] = dot8bf(wv[u], ld_keep(a + (int64_t)(m0 + m) * I + k), acc[m]);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float t = warp_sum(acc[m]);
      if (lane == m && m < mt) {
        float o = t;
        if (residual) o += __bfloat162float(residual[(int64_t)(m0 + m) * d + n]);
        out[(int64_t)(m0 + m) * d + n] = o;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Launch helpers
// ---------------------------------------------------------------------------
template <typename Kernel, typename... Args>
cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e == cudaSuccess) note_launches(1);
  return e;
}

// Resident CTAs per SM for a kernel at a given dynamic smem size, queried
// once per (device, kernel, smem) and cached.
template <typename Kernel>
int blocks_per_sm(Kernel kernel, size_t smem, int device) {
  static std::mutex mu;
  static std::map<std::tuple<int, const void*, size_t>, int> cache;
  const auto key = std::make_tuple(device, (const void*)kernel, smem);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int n = 0;
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kThreads, smem) != cudaSuccess)
    n = 0;
  n = std::max(n, 1);
  cache.emplace(key, n);
  return n;
}

template <int MT>
cudaError_t gateup_mt(const void* x, int64_t M, const void* gamma, float eps, const void* P,
                      int T, int64_t d, int64_t I, void* a, const DeviceInfo& dev,
                      cudaStream_t stream) {
  const size_t smem = (size_t)MT * d * sizeof(float);
  auto kernel = gateup_swiglu_gemv<MT>;
  const int per_sm = blocks_per_sm(kernel, smem, dev.device);
  const int64_t want = (I + kWarps - 1) / kWarps;
  const int gx = (int)std::min<int64_t>(want, (int64_t)dev.sm_count * per_sm);
  const int gy = (int)((M + MT - 1) / MT);
  return launch_pdl(kernel, dim3(gx, gy), dim3(kThreads), smem, stream,
                    (const __nv_bfloat16*)x, (int)M, (const __nv_bfloat16*)gamma, eps,
                    (const __nv_bfloat16*)P, T, (int)d, (int)I, (__nv_bfloat16*)a);
}

template <int MT>
cudaError_t down_mt(const void* a, int64_t M, const void* Wd, int64_t d, int64_t I,
                    const void* residual, float* out, const DeviceInfo& dev,
                    cudaStream_t stream) {
  auto kernel = down_gemv<MT>;
  const int per_sm = blocks_per_sm(kernel, 0, dev.device);
  const int64_t want = (d + kWarps - 1) / kWarps;
  const int gx = (int)std::min<int64_t>(want, (int64_t)dev.sm_count * per_sm);
  const int gy = (int)((M + MT - 1) / MT);
  return launch_pdl(kernel, dim3(gx, gy), dim3(kThreads), 0, stream,
                    (const __nv_bfloat16*)a, (int)M, (const __nv_bfloat16*)Wd, (int)d, (int)I,
                    (const __nv_bfloat16*)residual, out);
}

}  // namespace

cudaError_t launch_gateup_gemv(const void* x, int64_t M, const void* gamma, float eps,
                               const void* P, int T, int64_t d, int64_t I, void* a,
                               const DeviceInfo& dev, cudaStream_t stream) {
  // Token rows per pass: as many (<= 4) as fit s = x*gamma in shared memory.
  const int64_t fit = (int64_t)dev.max_smem_optin / (d * (int64_t)sizeof(float));
  const int64_t mt = std::min<int64_t>({M, 4, fit});
  switch (mt) {
    case 1: return gateup_mt<1>(x, M, gamma, eps, P, T, d, I, a, dev, stream);
    case 2: return gateup_mt<2>(x, M, gamma, eps, P, T, d, I, a, dev, stream);
    case 3: return gateup_mt<3>(x, M, gamma, eps, P, T, d, I, a, dev, stream);
    case 4: return gateup_mt<4>(x, M, gamma, eps, P, T, d, I, a, dev, stream);
    default: return cudaErrorInvalidConfiguration;
  }
}

cudaError_t launch_down_gemv(const void* a, int64_t M, const void* W_down, int64_t d,
                             int64_t I, const void* residual, float* out,
                             const DeviceInfo& dev, cudaStream_t stream) {
  switch (std::min<int64_t>(M, 4)) {
    case 1: return down_mt<1>(a, M, W_down, d, I, residual, out, dev, stream);
    case 2: return down_mt<2>(a, M, W_down, d, I, residual, out, dev, stream);
    case 3: return down_mt<3>(a, M, W_down, d, I, residual, out, dev, stream);
    default: return down_mt<4>(a, M, W_down, d, I, residual, out, dev, stream);
  }
}

}  // namespace fmlp
