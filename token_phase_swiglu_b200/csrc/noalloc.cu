// fmlp_forward_noalloc: the MLP block for callers that cannot allocate device
// memory.
//
// fmlp_forward needs a caller-provided workspace (status and barrier words,
// and the bf16 intermediate a).  Some callers have no way to provide one: a
// plug-in run by a host engine that owns all of device memory and gives its
// plug-ins no allocator, or a latency-critical serving loop that must never
// call cudaMalloc/cudaFree because those calls can synchronise the device.
// For them this file keeps one fixed scratch buffer in device memory for the
// whole process and runs the ordinary fmlp_forward path on it.
//
// The buffer is a file-scope __device__ array, so every GPU that loads the
// library reserves FMLP_NOALLOC_SCRATCH_BYTES until the process exits.  On
// the host the array's name is only a stand-in for the symbol, not a device
// address; the address is looked up with cudaGetSymbolAddress, with the
// device current, once per device and CUDA context, and cached.  The cache
// is keyed by the context as well as the device number: after
// cudaDeviceReset, or under a context other than the primary one, the
// module is loaded again at a new address and the old one must not be used.
#include "fmlp.h"
#include "internal.h"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

namespace {

constexpr size_t kScratchBytes = FMLP_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
struct ScratchEntry {
  CUcontext ctx = nullptr;  // context the address belongs to
  void* ptr = nullptr;
};
ScratchEntry g_scratch_ptr[kMaxDevices];

// cuCtxGetCurrent from the driver, fetched once through the runtime (the
// library does not link libcuda).
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
cudaError_t g_ctx_err = cudaSuccess;
std::once_flag g_ctx_once;

cudaError_t current_context(CUcontext* ctx) {
  std::call_once(g_ctx_once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    g_ctx_err = cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000,
                                                 cudaEnableDefault, &q);
    if (g_ctx_err == cudaSuccess && q != cudaDriverEntryPointSuccess)
      g_ctx_err = cudaErrorNotSupported;
    g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  });
  if (g_ctx_err != cudaSuccess) return g_ctx_err;
  *ctx = nullptr;  // none current yet is not an error here
  return g_ctx_current(ctx) == CUDA_SUCCESS ? cudaSuccess : cudaErrorDeviceUninitialized;
}

// Device address of g_scratch in the current device's current context,
// looked up on the first call in that context and cached for it.
cudaError_t scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  CUcontext ctx = nullptr;
  e = current_context(&ctx);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  ScratchEntry& ent = g_scratch_ptr[dev];
  if (ctx && ent.ctx == ctx && ent.ptr) {
    *out = ent.ptr;
    return cudaSuccess;
  }
  // The lookup also makes the device's primary context current when no
  // context is, so the context is read again after it.
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_scratch);
  if (e != cudaSuccess) return e;
  e = current_context(&ctx);
  if (e != cudaSuccess) return e;
  if (!ctx) return cudaErrorDeviceUninitialized;
  ent.ctx = ctx;
  ent.ptr = p;
  *out = p;
  return cudaSuccess;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// The argument rules of fmlp_forward, checked here first so that a rejected
// call enqueues nothing at all (not even the clear of the control words).
bool arguments_ok(const void* x, int64_t M, const void* gamma, float eps,
                  const void* packed_Wgu, int tile_T, const void* W_down, int64_t I,
                  const void* residual, const float* out) {
  if (!gamma || !packed_Wgu || !W_down) return false;
  if (M > 0 && (!x || !out)) return false;
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(packed_Wgu) || !aligned16(W_down) ||
      !aligned16(out) || !aligned16(residual))
    return false;
  if (!std::isfinite(eps) || !(eps > 0.f)) return false;
  return tile_T > 0 && tile_T % 8 == 0 && I % tile_T == 0;
}

}  // namespace

extern "C" fmlp_status fmlp_forward_noalloc(const void* x, int64_t M, const void* gamma,
                                            float eps, const void* packed_Wgu, int tile_T,
                                            const void* W_down, int64_t d, int64_t I,
                                            const void* residual, float* out, void* stream) {
  const size_t need = fmlp_workspace_bytes(M, d, I);
  if (need == 0) return FMLP_ERR_INVALID_ARG;
  if (!arguments_ok(x, M, gamma, eps, packed_Wgu, tile_T, W_down, I, residual, out))
    return FMLP_ERR_INVALID_ARG;
  if (need > kScratchBytes) return FMLP_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  cudaError_t e = scratch_on_current_device(&scratch);
  if (e != cudaSuccess) return fmlp::record_cuda_error(e);
  if (M > 0) {
    // The buffer keeps whatever the previous call left.  The control words
    // (status word and the fused kernel's counters) must start at zero; every
    // other region is rewritten before it is read.
    const size_t zero_bytes = fmlp::workspace_layout(M, d, I).zero_end;
    e = cudaMemsetAsync(scratch, 0, zero_bytes, (cudaStream_t)stream);
    if (e != cudaSuccess) return fmlp::record_cuda_error(e);
  }
  return fmlp_forward(x, M, gamma, eps, packed_Wgu, tile_T, W_down, d, I, residual, out, scratch,
                      kScratchBytes, stream);
}
