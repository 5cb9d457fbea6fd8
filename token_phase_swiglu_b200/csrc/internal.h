// Internal interfaces between the C-ABI layer (fmlp_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "fmlp.h"

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
// The first 256 bytes are control words: the device status word at 0, and
// the single-launch kernels' counters: set-up shares done at 64, finished
// CTAs at 128, arrival tickets at 192, and for the tensor-core layer kernel
// gate-up tiles finished at 224 and operand shares written at 240.  They must read zero when a call starts and every
// call (a timed-out one too) leaves them at zero, so one workspace serves
// calls of any M, d and I that fit in it.
struct WorkspaceLayout {
  size_t status = 0;     // uint32 device status word
  size_t inited = 64;    // uint32 out shares set (fused kernels)
  size_t done = 128;     // uint32 finished-CTA counter (fused kernels)
  size_t ticket = 192;   // uint32 CTA arrival tickets (fused kernels)
  size_t gu_done = 224;  // uint32 gate-up tiles finished (tensor-core layer kernel)
  size_t hl_done = 240;  // uint32 operand shares written (tensor-core layer kernel)
  size_t zero_end = 256;
  size_t a = 0;          // bf16 [M x I] intermediate
  size_t b_hl = 0, rinv = 0, partials = 0, counters = 0;  // tensor-core path
  size_t a_ready = 0;    // tensor-core layer kernel: per gate-up tile flags
  size_t out_acc = 0;    // f32 [M x d] sum of a call with a bf16 output
  size_t ncounters = 0;
  size_t total = 0;
};
constexpr int kFusedMaxM = 4;  // token rows handled by the fused decode kernel
WorkspaceLayout workspace_layout(int64_t M, int64_t d, int64_t I);

constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusBadInput = 2u;  // a device-side input out of range (attention position)

// Count of kernels enqueued by the library (fmlp_kernel_launch_count).
void note_launches(int n);

// Keep `e` for fmlp_last_cuda_error() and return FMLP_ERR_CUDA.
fmlp_status record_cuda_error(cudaError_t e);

// ---- kernels ---------------------------------------------------------------
cudaError_t launch_pack(const void* W_gate, const void* W_up, int64_t d, int64_t I, int T,
                        void* packed, cudaStream_t stream);

// Deadline of every bounded device-side wait (fmlp_set_wait_timeout_ns).
uint64_t wait_timeout_ns();
// Testing aid (fmlp_set_fault_injection): nonzero makes every producer
// withhold its last stage so the consumers' bounded waits expire.
int fault_injection();

// a[m, i] = bf16(SiLU(r g) * r u) for all M rows: TMA-bulk weight streaming,
// CUDA-core dot products.  `status` is the workspace's device status word.
cudaError_t launch_gateup_stream(const void* x, int64_t M, const void* gamma, float eps,
                                 const void* P, int T, int64_t d, int64_t I, void* a,
                                 uint32_t* status, const DeviceInfo& dev, cudaStream_t stream);

// Both steps in one launch, split over the intermediate dimension (M <= 4,
// fused_decode_supported).  CTAs add their partial down projections into
// out once the first CTAs to arrive have set it; ticket / inited / done: the
// workspace's counters of arrivals, of out shares set and of CTAs finished,
// zero on entry and on exit.
bool fused_decode_supported(int64_t M, int64_t d, int64_t I, const DeviceInfo& dev);
// out_bf16 (or null): the last CTA to finish rounds out to it.
cudaError_t launch_fused_decode(const void* x, int64_t M, const void* gamma, float eps,
                                const void* P, int T, const void* W_down, int64_t d, int64_t I,
                                const void* residual, float* out, void* out_bf16,
                                uint32_t* ticket, uint32_t* inited, uint32_t* done,
                                uint32_t* status, const DeviceInfo& dev, cudaStream_t stream);

// Tensor-core path (tcgen05, csrc/tc.cu) for M above the decode range.
constexpr int kTcMaxCtas = 160;  // workspace sizing bound on the grid (>= SMs of a B200)
struct TcWorkspace {
  void* b_hl;          // bf16 token-tiled [hi; lo] rows of x*gamma
  float* rinv;         // [M] 1/RMS
  float* partials;     // stream-K partial accumulators
  uint32_t* counters;  // per-tile arrival counters (zeroed by the prologue)
  int ncounters;
  uint32_t* status;
};
struct TcSizes {
  size_t b_hl = 0, rinv = 0, partials = 0, counters = 0;
};
TcSizes tc_sizes(int64_t M, int64_t d, int64_t I, int sm_count);
bool tc_supported(int64_t M, int64_t d, int64_t I, int T);
// The prologue of the gate-up GEMM also sets out_init (if not null) to the
// residual (or zero) for a down GEMM that follows.
cudaError_t launch_tc_gateup(const void* x, int64_t M, const void* gamma, float eps,
                             const void* P, int T, int64_t d, int64_t I, void* a,
                             float* out_init, const void* residual, const TcWorkspace& ws,
                             const DeviceInfo& dev, cudaStream_t stream);
// One-launch tensor-core layer (csrc/layer.cu) for 1 <= M <= 64 token rows:
// the whole block in one persistent kernel (gate-up stream-K range, then the
// down stream-K range, per CTA).
struct LayerWorkspace {
  void* b_hl;          // bf16 [2 Mt x d] hi/lo operand of x*gamma
  void* a;             // bf16 [M x I] intermediate
  float* rinv;         // [M] 1/RMS
  float* partials;     // stream-K partial accumulators
  uint32_t* counters;  // per gate-up tile arrival counters
  int ncounters;
  uint32_t* a_ready;   // per gate-up tile: its k-block of a is written
  uint32_t *ticket, *inited, *done, *gu_done, *hl_done, *status;  // control words
};
struct LayerSizes {
  size_t b_hl = 0, rinv = 0, partials = 0, counters = 0, a_ready = 0;
};
LayerSizes layer_sizes(int64_t M, int64_t d, int64_t I, int sm_count);
bool layer_supported(int64_t M, int64_t d, int64_t I, int T, const DeviceInfo& dev);
cudaError_t launch_tc_layer(const void* x, int64_t M, const void* gamma, float eps,
                            const void* P, int T, const void* W_down, int64_t d, int64_t I,
                            const void* residual, float* out, void* out_bf16,
                            const LayerWorkspace& ws, const DeviceInfo& dev,
                            cudaStream_t stream);
// dst (bf16 [M x d]) = src (f32) rounded, after the previous kernel on the stream.
cudaError_t launch_out_bf16(const float* src, void* dst, int64_t M, int64_t d,
                            const DeviceInfo& dev, cudaStream_t stream);

// Sum of n partial outputs (+ residual) into out_f32 and/or out_bf16
// (csrc/reduce.cu); the partials may be peer pointers.
constexpr int kMaxPartials = 16;
cudaError_t launch_sum_partials(const float* const* parts, int n, int64_t M, int64_t d,
                                const void* residual, float* out_f32, void* out_bf16,
                                const DeviceInfo& dev, cudaStream_t stream);

// int8 weights (csrc/q8.cu): groups of 64 along K with one f32 scale each.
bool q8_supported(int64_t M, int64_t d, int64_t I, int T, const DeviceInfo& dev);
cudaError_t launch_quantize_q8(const void* W, int64_t rows, int64_t K, void* q, float* s,
                               const DeviceInfo& dev, cudaStream_t stream);
cudaError_t launch_forward_q8(const void* x, int64_t M, const void* gamma, float eps,
                              const void* Pq, const float* Ps, int T, const void* Wdq,
                              const float* Wds, int64_t d, int64_t I, const void* residual,
                              float* out, void* out_bf16, void* a, uint32_t* status,
                              const DeviceInfo& dev, cudaStream_t stream);

// Token-phase attention (csrc/attn.cu): GKVC append + TPSFLAT-style fused
// RoPE / QK^T / softmax / PV over the cache.
struct AttnLayout {
  size_t counters = 0;  // [B H_kv] uint32 arrival counters (zero between calls)
  size_t partials = 0;  // f32 pieces of the segments split over CTAs
  size_t total = 0;
};
bool attn_shape_ok(int H, int H_kv, int D);
AttnLayout attn_layout(int64_t B, int H, int H_kv, int D);
cudaError_t launch_attn_decode(const void* q, const void* k_new, const void* v_new, void* k_cache,
                               void* v_cache, const int32_t* pos, int64_t B, int H, int H_kv,
                               int D, int64_t n_max, int n_ctx, float theta, float* out,
                               void* workspace, const DeviceInfo& dev, cudaStream_t stream);

// out = residual or zero (for a down GEMM with no gate-up prologue before it).
cudaError_t launch_out_init(float* out, const void* residual, int64_t M, int64_t d,
                            const DeviceInfo& dev, cudaStream_t stream);
// out += a W_down^T: split-K shares are added into out, which must already
// hold the residual (or zero).
cudaError_t launch_tc_down(const void* a, int64_t M, const void* W_down, int64_t d, int64_t I,
                           float* out, const TcWorkspace& ws, const DeviceInfo& dev,
                           cudaStream_t stream);

// out[m, n] = sum_i W_down[n, i] a[m, i] (+ residual), same streaming scheme.
cudaError_t launch_down_stream(const void* a, int64_t M, const void* W_down, int64_t d,
                               int64_t I, const void* residual, float* out, uint32_t* status,
                               const DeviceInfo& dev, cudaStream_t stream);

}  // namespace fmlp
