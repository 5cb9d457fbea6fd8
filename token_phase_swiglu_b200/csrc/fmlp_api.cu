// C ABI of libfmlp.so: argument validation, path selection and launches.
// The contract (layouts, ownership, errors) is documented in include/fmlp.h.
#include "fmlp.h"
#include "internal.h"

#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>

namespace fmlp {
namespace {

thread_local int g_last_cuda_error = 0;
std::atomic<uint64_t> g_launches{0};
constexpr uint64_t kDefaultWaitNs = 1000000000ull;  // 1 s
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
std::atomic<int> g_fault{0};

constexpr int kMaxDevices = 64;
DeviceInfo g_info[kMaxDevices];
std::once_flag g_once[kMaxDevices];
cudaError_t g_info_err[kMaxDevices];

constexpr int64_t kMaxD = 32768;
constexpr int64_t kMaxI = 65536;
constexpr int64_t kMaxAttnBatch = 65536;  // sequences per attention call

inline size_t align256(size_t n) { return (n + 255) & ~size_t(255); }
inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }  // NULL passes

inline uint32_t* status_word(void* workspace) { return (uint32_t*)workspace; }

// The tensor-core path takes token counts above the fused decode kernel's
// range, and from 2 rows on where it is the faster one.  The fused kernel's
// CUDA-core consumers do M dot products per weight and fall behind HBM after
// a row or two; the tensor-core path pays about 10 us per layer for its three
// launches whatever M.  Measured per layer on B200 (fused / tensor-core):
// Phi-3-shaped (151 MB of weights) M=2 28.3 / 36.9 us, M=3 33.8 / 37.1,
// M=4 39.7 / 37.0; 8B-shaped (352 MB) M=2 63.7 / 60.4, M=3 72.4 / 61.4.
bool use_tc(int64_t M, int64_t d, int64_t I, int T) {
  if (M < 2 || !tc_supported(M, d, I, T)) return false;
  return M > kFusedMaxM || M >= 4 || 6 * d * I > (int64_t)200000000;
}

LayerWorkspace layer_workspace(void* workspace, const WorkspaceLayout& L) {
  char* w = (char*)workspace;
  LayerWorkspace t;
  t.b_hl = w + L.b_hl;
  t.a = w + L.a;
  t.rinv = (float*)(w + L.rinv);
  t.partials = (float*)(w + L.partials);
  t.counters = (uint32_t*)(w + L.counters);
  t.ncounters = (int)L.ncounters;
  t.ticket = (uint32_t*)(w + L.ticket);
  t.inited = (uint32_t*)(w + L.inited);
  t.done = (uint32_t*)(w + L.done);
  t.gu_done = (uint32_t*)(w + L.gu_done);
  t.hl_done = (uint32_t*)(w + L.hl_done);
  t.a_ready = (uint32_t*)(w + L.a_ready);
  t.status = status_word(workspace);
  return t;
}

// Of the tensor-core batches, the one-launch layer kernel takes 2-8 rows of
// a layer above 200 MB of weights, where it is the faster one; the three
// launches the rest.  Measured on B200, four 8B-shaped layers back to back
// (d = 4096, I = 14336; us per layer, three launches / one launch): M=2 63.1 /
// 61.9, M=4 63.8 / 62.2, M=8 63.8 / 62.5, M=12 65.4 / 66.1, M=16 65.6 / 66.6,
// M=32 71.0 / 72.3, M=64 84.6 / 88.6; Phi-3-shaped (151 MB) M=4 36.7 / 38.6.
bool use_layer(int64_t M, int64_t d, int64_t I, int T, const DeviceInfo& dev) {
  return M >= 2 && M <= 8 && 6 * d * I > (int64_t)200000000 &&
         layer_supported(M, d, I, T, dev);
}

TcWorkspace tc_workspace(void* workspace, const WorkspaceLayout& L) {
  char* w = (char*)workspace;
  TcWorkspace t;
  t.b_hl = w + L.b_hl;
  t.rinv = (float*)(w + L.rinv);
  t.partials = (float*)(w + L.partials);
  t.counters = (uint32_t*)(w + L.counters);
  t.ncounters = (int)L.ncounters;
  t.status = status_word(workspace);
  return t;
}

fmlp_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return FMLP_ERR_CUDA;
}

bool sizes_ok(int64_t M, int64_t d, int64_t I) {
  return M >= 0 && d > 0 && I > 0 && d % 8 == 0 && I % 8 == 0 && d <= kMaxD && I <= kMaxI &&
         M <= (int64_t)1 << 24;
}

bool tile_ok(int T, int64_t I) { return T > 0 && T % 8 == 0 && I % T == 0; }

bool eps_ok(float eps) { return std::isfinite(eps) && eps > 0.f; }

// Resolve the current device's cached attributes and check it is sm_100.
fmlp_status device_for_launch(const DeviceInfo** info) {
  cudaError_t e = current_device_info(info);
  if (e != cudaSuccess) return cuda_fail(e);
  if ((*info)->cc_major != 10) return FMLP_ERR_UNSUPPORTED;
  return FMLP_OK;
}

}  // namespace

void note_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

fmlp_status record_cuda_error(cudaError_t e) { return cuda_fail(e); }

uint64_t wait_timeout_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

int fault_injection() { return g_fault.load(std::memory_order_relaxed); }

cudaError_t current_device_info(const DeviceInfo** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_once[dev], [dev] {
    DeviceInfo& di = g_info[dev];
    di.device = dev;
    cudaError_t err = cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (err == cudaSuccess)
      err = cudaDeviceGetAttribute(&di.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    if (err == cudaSuccess)
      err = cudaDeviceGetAttribute(&di.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (err == cudaSuccess)
      err = cudaDeviceGetAttribute(&di.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                                   dev);
    g_info_err[dev] = err;
  });
  *out = &g_info[dev];
  return g_info_err[dev];
}

WorkspaceLayout workspace_layout(int64_t M, int64_t d, int64_t I) {
  WorkspaceLayout L;
  size_t off = 0;
  L.status = off;
  L.inited = off + 64;
  L.done = off + 128;
  L.ticket = off + 192;
  L.gu_done = off + 224;
  L.hl_done = off + 240;
  off += 256;
  L.zero_end = off;
  L.a = off;
  off += align256((size_t)M * (size_t)I * 2);
  if (M >= 2 && tc_supported(M, d, I, 16)) {  // the tensor-core paths may run
    const TcSizes z = tc_sizes(M, d, I, kTcMaxCtas);
    const LayerSizes zl = layer_sizes(M, d, I, kTcMaxCtas);
    L.b_hl = off;
    off += align256(std::max(z.b_hl, zl.b_hl));
    L.rinv = off;
    off += align256(std::max(z.rinv, zl.rinv));
    L.partials = off;
    off += align256(std::max(z.partials, zl.partials));
    L.counters = off;
    const size_t counters = std::max(z.counters, zl.counters);
    L.ncounters = counters / 4;
    off += align256(counters);
    L.a_ready = off;
    off += align256(zl.a_ready);
  }
  // the f32 sum of a call with a bf16 output (fmlp_forward_bf16)
  L.out_acc = off;
  off += align256((size_t)M * (size_t)d * 4);
  L.total = off;
  return L;
}

}  // namespace fmlp

using namespace fmlp;

extern "C" {

const char* fmlp_status_string(fmlp_status s) {
  switch (s) {
    case FMLP_OK: return "FMLP_OK";
    case FMLP_ERR_INVALID_ARG: return "FMLP_ERR_INVALID_ARG: invalid argument";
    case FMLP_ERR_UNSUPPORTED: return "FMLP_ERR_UNSUPPORTED: request outside the implemented kernels";
    case FMLP_ERR_CUDA: return "FMLP_ERR_CUDA: a CUDA call or launch failed";
    case FMLP_ERR_TIMEOUT: return "FMLP_ERR_TIMEOUT: a bounded device wait expired";
  }
  return "unknown fmlp_status";
}

int fmlp_last_cuda_error(void) { return g_last_cuda_error; }

uint64_t fmlp_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

void fmlp_set_wait_timeout_ns(uint64_t ns) {
  g_wait_ns.store(ns ? ns : kDefaultWaitNs, std::memory_order_relaxed);
}

void fmlp_set_fault_injection(int mode) { g_fault.store(mode ? 1 : 0, std::memory_order_relaxed); }

size_t fmlp_workspace_bytes(int64_t M, int64_t d, int64_t I) {
  if (!sizes_ok(M, d, I)) return 0;
  return workspace_layout(M, d, I).total;
}

fmlp_status fmlp_pack(const void* W_gate, const void* W_up, int64_t d, int64_t I, int tile_T,
                      void* packed, void* stream) {
  if (!W_gate || !W_up || !packed) return FMLP_ERR_INVALID_ARG;
  if (!aligned16(W_gate) || !aligned16(W_up) || !aligned16(packed)) return FMLP_ERR_INVALID_ARG;
  if (!sizes_ok(0, d, I) || !tile_ok(tile_T, I)) return FMLP_ERR_INVALID_ARG;
  // the output must not overlap either input
  const uintptr_t p0 = (uintptr_t)packed, p1 = p0 + (uintptr_t)(2 * I * d * 2);
  const uintptr_t in_bytes = (uintptr_t)(I * d * 2);
  for (const void* src : {W_gate, W_up}) {
    const uintptr_t s0 = (uintptr_t)src, s1 = s0 + in_bytes;
    if (s0 < p1 && p0 < s1) return FMLP_ERR_INVALID_ARG;
  }
  const DeviceInfo* dev = nullptr;
  fmlp_status st = device_for_launch(&dev);
  if (st != FMLP_OK) return st;
  cudaError_t e = launch_pack(W_gate, W_up, d, I, tile_T, packed, (cudaStream_t)stream);
  return e == cudaSuccess ? FMLP_OK : cuda_fail(e);
}

static fmlp_status check_common(int64_t M, int64_t d, int64_t I, void* workspace,
                                size_t workspace_bytes) {
  if (!sizes_ok(M, d, I)) return FMLP_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace)) return FMLP_ERR_INVALID_ARG;
  if (workspace_bytes < workspace_layout(M, d, I).total) return FMLP_ERR_INVALID_ARG;
  return FMLP_OK;
}

fmlp_status fmlp_gate_up_swiglu(const void* x, int64_t M, const void* gamma, float eps,
                                const void* packed_Wgu, int tile_T, int64_t d, int64_t I,
                                void* a, void* workspace, size_t workspace_bytes,
                                void* stream) {
  fmlp_status st = check_common(M, d, I, workspace, workspace_bytes);
  if (st != FMLP_OK) return st;
  if (!gamma || !packed_Wgu) return FMLP_ERR_INVALID_ARG;
  if (M > 0 && (!x || !a)) return FMLP_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(packed_Wgu) || !aligned16(a))
    return FMLP_ERR_INVALID_ARG;
  if (!eps_ok(eps) || !tile_ok(tile_T, I)) return FMLP_ERR_INVALID_ARG;
  if (M == 0) return FMLP_OK;
  const DeviceInfo* dev = nullptr;
  st = device_for_launch(&dev);
  if (st != FMLP_OK) return st;
  cudaError_t e;
  if (use_tc(M, d, I, tile_T))
    e = launch_tc_gateup(x, M, gamma, eps, packed_Wgu, tile_T, d, I, a, nullptr, nullptr,
                         tc_workspace(workspace, workspace_layout(M, d, I)), *dev,
                         (cudaStream_t)stream);
  else
    e = launch_gateup_stream(x, M, gamma, eps, packed_Wgu, tile_T, d, I, a,
                             status_word(workspace), *dev, (cudaStream_t)stream);
  return e == cudaSuccess ? FMLP_OK : cuda_fail(e);
}

fmlp_status fmlp_down_proj(const void* a, int64_t M, const void* W_down, int64_t d, int64_t I,
                           const void* residual, float* out, void* workspace,
                           size_t workspace_bytes, void* stream) {
  fmlp_status st = check_common(M, d, I, workspace, workspace_bytes);
  if (st != FMLP_OK) return st;
  if (!W_down) return FMLP_ERR_INVALID_ARG;
  if (M > 0 && (!a || !out)) return FMLP_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(W_down) || !aligned16(out) || !aligned16(residual))
    return FMLP_ERR_INVALID_ARG;
  if (M == 0) return FMLP_OK;
  const DeviceInfo* dev = nullptr;
  st = device_for_launch(&dev);
  if (st != FMLP_OK) return st;
  cudaError_t e;
  if (use_tc(M, d, I, 16)) {
    // Run alone, the down GEMM has no gate-up prologue to set out first.
    const TcWorkspace tw = tc_workspace(workspace, workspace_layout(M, d, I));
    e = launch_out_init(out, residual, M, d, *dev, (cudaStream_t)stream);
    if (e == cudaSuccess) e = launch_tc_down(a, M, W_down, d, I, out, tw, *dev, (cudaStream_t)stream);
  } else
    e = launch_down_stream(a, M, W_down, d, I, residual, out, status_word(workspace), *dev,
                           (cudaStream_t)stream);
  return e == cudaSuccess ? FMLP_OK : cuda_fail(e);
}

// The MLP block into out (f32), or, with out_bf16 set, into the workspace's
// f32 sum and then rounded to out_bf16.
static fmlp_status forward_impl(const void* x, int64_t M, const void* gamma, float eps,
                                const void* packed_Wgu, int tile_T, const void* W_down,
                                int64_t d, int64_t I, const void* residual, float* out,
                                void* out_bf16, void* workspace, size_t workspace_bytes,
                                void* stream) {
  fmlp_status st = check_common(M, d, I, workspace, workspace_bytes);
  if (st != FMLP_OK) return st;
  if (!gamma || !packed_Wgu || !W_down) return FMLP_ERR_INVALID_ARG;
  if (M > 0 && (!x || (!out && !out_bf16))) return FMLP_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(packed_Wgu) || !aligned16(W_down) ||
      !aligned16(out) || !aligned16(residual))
    return FMLP_ERR_INVALID_ARG;
  if (!eps_ok(eps) || !tile_ok(tile_T, I)) return FMLP_ERR_INVALID_ARG;
  if (M == 0) return FMLP_OK;
  const DeviceInfo* dev = nullptr;
  st = device_for_launch(&dev);
  if (st != FMLP_OK) return st;
  const WorkspaceLayout L = workspace_layout(M, d, I);
  void* a = (char*)workspace + L.a;
  uint32_t* status = status_word(workspace);
  cudaStream_t s = (cudaStream_t)stream;
  if (out_bf16) out = (float*)((char*)workspace + L.out_acc);
  cudaError_t e;
  bool rounded = false;  // the kernel rounded out to out_bf16 itself
  if (!use_tc(M, d, I, tile_T) && fused_decode_supported(M, d, I, *dev)) {
    uint32_t* ticket = (uint32_t*)((char*)workspace + L.ticket);
    uint32_t* inited = (uint32_t*)((char*)workspace + L.inited);
    uint32_t* done = (uint32_t*)((char*)workspace + L.done);
    e = launch_fused_decode(x, M, gamma, eps, packed_Wgu, tile_T, W_down, d, I, residual, out,
                            out_bf16, ticket, inited, done, status, *dev, s);
    rounded = true;
  } else if (use_tc(M, d, I, tile_T) && use_layer(M, d, I, tile_T, *dev)) {
    e = launch_tc_layer(x, M, gamma, eps, packed_Wgu, tile_T, W_down, d, I, residual, out,
                        out_bf16, layer_workspace(workspace, L), *dev, s);
    rounded = true;
  } else if (use_tc(M, d, I, tile_T)) {
    const TcWorkspace tw = tc_workspace(workspace, L);
    e = launch_tc_gateup(x, M, gamma, eps, packed_Wgu, tile_T, d, I, a, out, residual, tw,
                         *dev, s);
    if (e == cudaSuccess) e = launch_tc_down(a, M, W_down, d, I, out, tw, *dev, s);
  } else {
    e = launch_gateup_stream(x, M, gamma, eps, packed_Wgu, tile_T, d, I, a, status, *dev, s);
    if (e == cudaSuccess)
      e = launch_down_stream(a, M, W_down, d, I, residual, out, status, *dev, s);
  }
  if (e == cudaSuccess && out_bf16 && !rounded) e = launch_out_bf16(out, out_bf16, M, d, *dev, s);
  return e == cudaSuccess ? FMLP_OK : cuda_fail(e);
}

fmlp_status fmlp_forward(const void* x, int64_t M, const void* gamma, float eps,
                         const void* packed_Wgu, int tile_T, const void* W_down, int64_t d,
                         int64_t I, const void* residual, float* out, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return forward_impl(x, M, gamma, eps, packed_Wgu, tile_T, W_down, d, I, residual, out,
                      nullptr, workspace, workspace_bytes, stream);
}

fmlp_status fmlp_forward_bf16(const void* x, int64_t M, const void* gamma, float eps,
                              const void* packed_Wgu, int tile_T, const void* W_down, int64_t d,
                              int64_t I, const void* residual, void* out, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (M > 0 && !out) return FMLP_ERR_INVALID_ARG;
  if (!aligned16(out)) return FMLP_ERR_INVALID_ARG;
  // out may be x or the residual itself (it is written after every read of
  // them), but must not overlap the workspace
  if (M > 0) {
    const uintptr_t o0 = (uintptr_t)out, o1 = o0 + (uintptr_t)(M * d * 2);
    const uintptr_t w0 = (uintptr_t)workspace, w1 = w0 + workspace_bytes;
    if (workspace && o0 < w1 && w0 < o1) return FMLP_ERR_INVALID_ARG;
  }
  return forward_impl(x, M, gamma, eps, packed_Wgu, tile_T, W_down, d, I, residual, nullptr,
                      out, workspace, workspace_bytes, stream);
}

fmlp_status fmlp_quantize_q8(const void* W, int64_t rows, int64_t K, void* q, float* scales,
                             void* stream) {
  if (!W || !q || !scales || rows < 1 || K < 64 || K % 64 != 0 || K > kMaxI)
    return FMLP_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(q) || !aligned16(scales)) return FMLP_ERR_INVALID_ARG;
  const DeviceInfo* dev = nullptr;
  fmlp_status st = device_for_launch(&dev);
  if (st != FMLP_OK) return st;
  cudaError_t e = launch_quantize_q8(W, rows, K, q, scales, *dev, (cudaStream_t)stream);
  return e == cudaSuccess ? FMLP_OK : cuda_fail(e);
}

fmlp_status fmlp_forward_q8(const void* x, int64_t M, const void* gamma, float eps,
                            const void* packed_q, const float* packed_scales, int tile_T,
                            const void* W_down_q, const float* W_down_scales, int64_t d,
                            int64_t I, const void* residual, float* out, void* workspace,
                            size_t workspace_bytes, void* stream) {
  fmlp_status st = check_common(M, d, I, workspace, workspace_bytes);
  if (st != FMLP_OK) return st;
  if (!gamma || !packed_q || !packed_scales || !W_down_q || !W_down_scales)
    return FMLP_ERR_INVALID_ARG;
  if (M > 0 && (!x || !out)) return FMLP_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(packed_q) || !aligned16(packed_scales) ||
      !aligned16(W_down_q) || !aligned16(W_down_scales) || !aligned16(out) ||
      !aligned16(residual))
    return FMLP_ERR_INVALID_ARG;
  if (!eps_ok(eps) || !tile_ok(tile_T, I)) return FMLP_ERR_INVALID_ARG;
  if (M == 0) return FMLP_OK;
  const DeviceInfo* dev = nullptr;
  st = device_for_launch(&dev);
  if (st != FMLP_OK) return st;
  if (!q8_supported(M, d, I, tile_T, *dev)) return FMLP_ERR_UNSUPPORTED;
  void* a = (char*)workspace + workspace_layout(M, d, I).a;
  cudaError_t e = launch_forward_q8(x, M, gamma, eps, packed_q, packed_scales, tile_T, W_down_q,
                                    W_down_scales, d, I, residual, out, nullptr, a,
                                    (uint32_t*)workspace, *dev, (cudaStream_t)stream);
  return e == cudaSuccess ? FMLP_OK : cuda_fail(e);
}

fmlp_status fmlp_sum_partials(const float* const* partials, int n, int64_t M, int64_t d,
                              const void* residual, void* out, int out_bf16, void* stream) {
  if (n < 1 || n > kMaxPartials || M < 0 || d <= 0 || d % 8 != 0 || d > kMaxD)
    return FMLP_ERR_INVALID_ARG;
  if (M == 0) return FMLP_OK;
  if (!partials || !out || !aligned16(out) || !aligned16(residual)) return FMLP_ERR_INVALID_ARG;
  const uintptr_t o0 = (uintptr_t)out, o1 = o0 + (uintptr_t)(M * d * (out_bf16 ? 2 : 4));
  for (int r = 0; r < n; ++r) {
    if (!partials[r] || !aligned16(partials[r])) return FMLP_ERR_INVALID_ARG;
    // out may not overlap a partial, unless it is that partial itself (f32)
    const uintptr_t p0 = (uintptr_t)partials[r], p1 = p0 + (uintptr_t)(M * d * 4);
    if (o0 < p1 && p0 < o1 && !(o0 == p0 && !out_bf16)) return FMLP_ERR_INVALID_ARG;
  }
  const DeviceInfo* dev = nullptr;
  fmlp_status st = device_for_launch(&dev);
  if (st != FMLP_OK) return st;
  cudaError_t e = launch_sum_partials(partials, n, M, d, residual,
                                      out_bf16 ? nullptr : (float*)out, out_bf16 ? out : nullptr,
                                      *dev, (cudaStream_t)stream);
  return e == cudaSuccess ? FMLP_OK : cuda_fail(e);
}

size_t fmlp_attn_workspace_bytes(int64_t B, int H, int H_kv, int D) {
  if (B < 1 || B > kMaxAttnBatch || !attn_shape_ok(H, H_kv, D)) return 0;
  return attn_layout(B, H, H_kv, D).total;
}

fmlp_status fmlp_attn_decode(const void* q, const void* k_new, const void* v_new, void* k_cache,
                             void* v_cache, const int32_t* pos, int64_t B, int H, int H_kv, int D,
                             int64_t n_max, int64_t n_ctx, float theta, float* out,
                             void* workspace, size_t workspace_bytes, void* stream) {
  if (B < 1 || B > kMaxAttnBatch || !attn_shape_ok(H, H_kv, D)) return FMLP_ERR_INVALID_ARG;
  // TMA row coordinates (int32) run to the end of the last 64-row unit
  if (n_ctx < 1 || n_max < n_ctx || (int64_t)B * H_kv * n_max + 64 > (int64_t)INT32_MAX)
    return FMLP_ERR_INVALID_ARG;
  if (!(theta > 0.f) || !std::isfinite(theta)) return FMLP_ERR_INVALID_ARG;
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !pos || !out || !workspace)
    return FMLP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) ||
      !aligned16(v_cache) || !aligned16(out) || !aligned16(workspace) || ((uintptr_t)pos & 3u))
    return FMLP_ERR_INVALID_ARG;
  if (workspace_bytes < attn_layout(B, H, H_kv, D).total) return FMLP_ERR_INVALID_ARG;
  const DeviceInfo* dev = nullptr;
  fmlp_status st = device_for_launch(&dev);
  if (st != FMLP_OK) return st;
  cudaError_t e = launch_attn_decode(q, k_new, v_new, k_cache, v_cache, pos, B, H, H_kv, D,
                                     n_max, (int)n_ctx, theta, out, workspace, *dev,
                                     (cudaStream_t)stream);
  return e == cudaSuccess ? FMLP_OK : cuda_fail(e);
}

fmlp_status fmlp_device_status(void* workspace, void* stream) {
  if (!workspace || !aligned16(workspace)) return FMLP_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && word != 0) {
    // reset the whole control block along with the status word
    e = cudaMemsetAsync(workspace, 0, workspace_layout(0, 8, 8).a, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  if (word & kStatusTimeout) return FMLP_ERR_TIMEOUT;
  return word & kStatusBadInput ? FMLP_ERR_INVALID_ARG : FMLP_OK;
}

}  // extern "C"
