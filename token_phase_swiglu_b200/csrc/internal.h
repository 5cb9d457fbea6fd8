// Internal interfaces between the C-ABI layer (fmlp_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace fmlp {

// Device attributes, queried once per device and cached (a per-launch
// cudaGetDeviceProperties costs more than a small kernel).
struct DeviceInfo {
  int device = -1;
  int sm_count = 0;
  int cc_major = 0, cc_minor = 0;
  int max_smem_optin = 0;   // bytes of dynamic shared memory a CTA may opt into
};
cudaError_t current_device_info(const DeviceInfo** out);

// Workspace layout (byte offsets from the workspace base, 256-aligned).
struct WorkspaceLayout {
  size_t status = 0;     // uint32 device status word (+ reserved control words)
  size_t a = 0;          // bf16 [M x I] intermediate
  size_t total = 0;
};
WorkspaceLayout workspace_layout(int64_t M, int64_t d, int64_t I);

constexpr uint32_t kStatusTimeout = 1u;

// Count of kernels enqueued by the library (fmlp_kernel_launch_count).
void note_launches(int n);

// ---- kernels ---------------------------------------------------------------
cudaError_t launch_pack(const void* W_gate, const void* W_up, int64_t d, int64_t I, int T,
                        void* packed, cudaStream_t stream);

// a[m, i] = bf16(SiLU(r g) * r u) for all M rows, CUDA-core weight streaming.
cudaError_t launch_gateup_gemv(const void* x, int64_t M, const void* gamma, float eps,
                               const void* P, int T, int64_t d, int64_t I, void* a,
                               const DeviceInfo& dev, cudaStream_t stream);

// out[m, n] = sum_i W_down[n, i] a[m, i] (+ residual), CUDA-core weight streaming.
cudaError_t launch_down_gemv(const void* a, int64_t M, const void* W_down, int64_t d,
                             int64_t I, const void* residual, float* out,
                             const DeviceInfo& dev, cudaStream_t stream);

}  // namespace fmlp
