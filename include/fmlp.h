/*
 * fmlp.h -- C ABI of the B200 fused gated-MLP library (libfmlp.so).
 *
 * The library computes the MLP block of a decoder-only transformer layer over
 * a small batch of token rows:
 *
 *     r[m] = 1 / sqrt(mean_k x[m,k]^2 + eps)                 RMSNorm
 *     h    = x * r * gamma
 *     a    = SiLU(h W_gate^T) * (h W_up^T),  SiLU(t) = t/(1+e^-t)
 *     out  = a W_down^T  (+ residual)
 *
 * Sources: "FastTPS: An Optimized Method for LLM Token Phase for AI
 * Accelerators" (xllm-io paper review), section 三: Eq(1), the MLP execution
 * flow (RMSNorm -> interleaved gate-up Matmul -> siLu_Mul -> down projection)
 * and component 3 "Fusion MLP"; section 五, Fusion MLP Steps 1-3; and
 * "CUDAカーネル融合で推論が最大10%高速化" (blog.cecily.jp), the llama.cpp PR
 * #29948 paragraph on alternating gate/up rows.  The pages define no API;
 * the calls below are this library's own.
 *
 * Conventions for every call
 *   - All tensors are dense, row-major, in DEVICE memory owned by the caller.
 *     bf16 is IEEE bfloat16 (2 bytes), f32 is IEEE binary32.  Every pointer
 *     must be 16-byte aligned.  The library never writes an input and never
 *     allocates device memory per call.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     are asynchronous on it; a returned FMLP_OK means the work was enqueued.
 *   - Arguments are validated on the host first; on any validation failure
 *     nothing is launched and FMLP_ERR_INVALID_ARG or FMLP_ERR_UNSUPPORTED is
 *     returned.  A CUDA launch or runtime failure returns FMLP_ERR_CUDA (the
 *     CUDA error code is kept for fmlp_last_cuda_error()).  There is no CPU
 *     fallback: without a usable sm_100 device every compute call fails.
 *   - Sizes: d (hidden) and I (intermediate) must be positive multiples of 8
 *     (rows are whole 16-byte vectors), d <= 32768, I <= 65536.  M (token
 *     rows) may be 0, which is a no-op; then the pointers to M-row tensors
 *     (x, a, out, residual) may be NULL.
 */
#ifndef FMLP_H
#define FMLP_H

#include <stddef.h>
#include <stdint.h>

#if defined(FMLP_BUILD) && defined(__GNUC__)
#define FMLP_API __attribute__((visibility("default")))
#else
#define FMLP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fmlp_status {
  FMLP_OK = 0,
  FMLP_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, bad eps, small workspace */
  FMLP_ERR_UNSUPPORTED = 2,  /* valid request outside what the kernels implement        */
  FMLP_ERR_CUDA = 3,         /* a CUDA call or launch failed                             */
  FMLP_ERR_TIMEOUT = 4       /* a bounded device-side wait expired (device status word)  */
} fmlp_status;

/*
 * fmlp_pack -- interleave W_gate and W_up rows into one matrix (step a0).
 *
 * FastTPS section 三, component 3 (gate/up projections interleaved into one
 * large matmul) and the llama.cpp PR paragraph (gate and up rows alternate).
 * With tile T, packed rows [2T*t, 2T*t+T) are W_gate rows [T*t, T*t+T) and
 * packed rows [2T*t+T, 2T*(t+1)) are the W_up rows [T*t, T*t+T):
 *     packed[2T*t + j]     = W_gate[T*t + j]
 *     packed[2T*t + T + j] = W_up  [T*t + j],   0 <= j < T.
 * A pure permutation of rows: the bytes are copied unchanged.
 *
 *   W_gate, W_up : bf16 [I x d]   (nn.Linear layout: out x in)
 *   d, I         : d % 8 == 0, I % 8 == 0
 *   tile_T       : tile_T % 8 == 0 and I % tile_T == 0 (16 is the canonical tile)
 *   packed       : bf16 [2I x d], caller-allocated, must not overlap the inputs
 */
FMLP_API fmlp_status fmlp_pack(const void* W_gate, const void* W_up, int64_t d, int64_t I,
                      int tile_T, void* packed, void* stream);

/*
 * fmlp_workspace_bytes -- bytes of device workspace fmlp_forward (and
 * fmlp_forward_bf16) needs for (M, d, I).  The workspace holds a device
 * status word, the single-launch kernels' counters, the bf16 intermediate
 * a [M x I], the tensor-core paths' operand copy, stream-K partials and tile
 * flags, and an f32 [M x d] sum for a bf16 output.  A workspace
 * must be zero-filled before its first use; after that, every call (a
 * timed-out one too) leaves it ready for the next call of any sizes whose
 * fmlp_workspace_bytes it does not exceed.  Returns 0 for invalid sizes.
 */
FMLP_API size_t fmlp_workspace_bytes(int64_t M, int64_t d, int64_t I);

/*
 * fmlp_forward -- the whole MLP block (steps a1-a6): RMSNorm, interleaved
 * gate-up contraction, SiLU*up epilogue, down projection, optional residual.
 *
 * FastTPS section 三: Eq(1), O = W_down(SiLU(W_gate h) * (W_up h)), and the
 * MLP execution flow RMSNorm -> interleaved gate-up Matmul -> siLu_Mul ->
 * down projection (Figure 4 parts 1-3); section 五, Fusion MLP Steps 1-3 (the
 * block as one kernel).  The residual add is this library's own option; the
 * pages do not name it.
 *
 *   x          : bf16 [M x d] token rows
 *   M          : token rows, >= 0
 *   gamma      : bf16 [d] RMSNorm weight (multiplies directly)
 *   eps        : RMSNorm epsilon, finite and > 0
 *   packed_Wgu : bf16 [2I x d] from fmlp_pack with the same tile_T
 *   W_down     : bf16 [d x I]
 *   residual   : bf16 [M x d] added to the output, or NULL
 *   out        : f32 [M x d]
 *   workspace  : >= fmlp_workspace_bytes(M, d, I) bytes, zeroed as described
 *                there, not shared by calls that may overlap on the GPU
 *
 * Precision: x*gamma is formed exactly in f32 and the contraction keeps it at
 * f32 precision (CUDA-core path) or as an exact hi+lo bf16 pair (tensor-core
 * path); accumulation is f32; SiLU is evaluated in f32 (on the tensor-core
 * path with the hardware exp2 and reciprocal approximations, relative error
 * about 1e-6); a is rounded once to bf16 (round to nearest even); out is
 * f32.  out is written by several thread blocks adding into it (f32
 * atomics), so the summation order, and the last bits of out, may differ
 * from run to run.  out must not overlap any input.
 *
 * Kernels: one row (M = 1), and 2-3 rows of a layer whose weights (6 d I
 * bytes) are at most 200 MB, run one fused launch (CUDA-core dot products
 * over a TMA-streamed weight ring).  Other batches run three launches on the
 * tensor cores (prologue, gate-up GEMM with the SiLU*up epilogue, down GEMM)
 * when d and I are multiples of 64 and tile_T is 8 or 16.  Failing that, up
 * to 4 rows run the fused launch where its shared memory allows, and the
 * rest two CUDA-core streaming launches.
 *
 * Ordering: the kernels use programmatic dependent launch.  A kernel of this
 * library may start streaming packed_Wgu, W_down and gamma while the
 * previous kernel on the stream is still running, if that kernel is one of
 * this library's (fmlp_pack excepted), which never write those buffers.
 * Everything else (x, residual, out, workspace) is touched only after the
 * previous work on the stream has completed.
 */
FMLP_API fmlp_status fmlp_forward(const void* x, int64_t M, const void* gamma, float eps,
                         const void* packed_Wgu, int tile_T, const void* W_down,
                         int64_t d, int64_t I, const void* residual, float* out,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * fmlp_forward_bf16 -- the MLP block with a bf16 output, for chaining layers:
 *     out = bf16_RN( a W_down^T + residual )
 * rounded once, after the residual add (round to nearest even), so that the
 * result can be fed to the next layer as its x.  FastTPS section 三, Eq(1)
 * and the MLP execution flow as in fmlp_forward; section 六 (bf16 simulation:
 * the tensors passed between operators are bf16).
 *
 * Arguments as in fmlp_forward, except
 *   out : bf16 [M x d].  It may be the same buffer as x or as residual (an
 *         in-place update of the residual stream): it is written only after
 *         every read of them.  It must not overlap the workspace or a weight.
 * The f32 sum is kept in the workspace (fmlp_workspace_bytes covers it).
 * Precision: as fmlp_forward up to the f32 sum, then one rounding to bf16;
 * against the binary64 block the output differs by that rounding (at most
 * half a bf16 step per element) on top of fmlp_forward's error.
 *
 * Kernels: the single-launch paths of fmlp_forward round the sum in their
 * last thread block to finish (still one launch); the multi-launch paths add
 * one small rounding launch.
 */
FMLP_API fmlp_status fmlp_forward_bf16(const void* x, int64_t M, const void* gamma, float eps,
                                       const void* packed_Wgu, int tile_T, const void* W_down,
                                       int64_t d, int64_t I, const void* residual, void* out,
                                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * fmlp_gate_up_swiglu -- steps a1-a4 alone: writes the bf16 intermediate
 *     a[m,i] = bf16( SiLU(r[m] * g[m,i]) * r[m] * u[m,i] )
 * with g, u the contractions of x*gamma with the gate and up rows of
 * packed_Wgu.  FastTPS section 三, Eq(1) inside W_down(...) and Figure 4
 * parts 1-2 (RMSNorm, interleaved gate-up Matmul, siLu_Mul); section 五,
 * Fusion MLP Steps 1-2; the llama.cpp PR paragraph (gate and up rows
 * alternate and the GLU is applied in the same pass).  Arguments as in fmlp_forward; `a` is bf16 [M x I] and must not
 * overlap the workspace.
 */
FMLP_API fmlp_status fmlp_gate_up_swiglu(const void* x, int64_t M, const void* gamma, float eps,
                                const void* packed_Wgu, int tile_T, int64_t d, int64_t I,
                                void* a, void* workspace, size_t workspace_bytes,
                                void* stream);

/*
 * fmlp_down_proj -- steps a5-a6 alone: out = a W_down^T (+ residual).
 * FastTPS section 三, the outer W_down(...) of Eq(1) and Figure 4 part 3
 * (down projection); section 五, Fusion MLP Step 3 (read with Eq(1): the
 * element-wise product is already in a).
 *   a : bf16 [M x I]; other arguments as in fmlp_forward.
 */
FMLP_API fmlp_status fmlp_down_proj(const void* a, int64_t M, const void* W_down, int64_t d,
                           int64_t I, const void* residual, float* out, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * fmlp_quantize_q8 -- this library's int8 weight format (the pages name
 * quantized weight streaming over interleaved gate/up rows -- the llama.cpp
 * PR #29948 paragraph of "CUDAカーネル融合で推論が最大10%高速化",
 * blog.cecily.jp -- but give no block format).  Each row of W is cut along K
 * into groups of 64 consecutive elements; group g gets one binary32 scale
 *     s_g = fl32(max |w| / 127)            (IEEE division, round to nearest)
 * and each weight the int8
 *     q = clamp(rint(fl32(w / s_g)), -127, 127)   (rint: halves to even)
 * (q = 0 in a group of zeros).  The weight stands for q * s_g.  Quantizing
 * works row by row, so quantizing fmlp_pack's output equals packing the
 * quantized matrices: quantize packed_Wgu [2I x d] (K = d) and W_down
 * [d x I] (K = I) for fmlp_forward_q8.
 *
 *   W      : bf16 [rows x K], K a multiple of 64
 *   q      : int8 [rows x K], caller-allocated
 *   scales : f32 [rows x K/64], caller-allocated
 * Bit-exact: the same q and scales on every run.
 */
FMLP_API fmlp_status fmlp_quantize_q8(const void* W, int64_t rows, int64_t K, void* q,
                                      float* scales, void* stream);

/*
 * fmlp_forward_q8 -- the MLP block (steps a1-a6) on int8 weights from
 * fmlp_quantize_q8: fmlp_forward with W_gate, W_up and W_down replaced by
 * their dequantized values q * s.  Decode batches only: 1 <= M <= 4 token
 * rows, d and I multiples of 512, and the M rows' activations in f32
 * (M*d*4 and M*I*4 bytes) plus a ring of at least three stages within a
 * CTA's shared memory (with I = 14336: up to 3 rows); other requests return
 * FMLP_ERR_UNSUPPORTED before anything is launched.  About 1.06 bytes of
 * weights per element are streamed instead of 2.  Every device-side wait is
 * bounded; a kernel that gives one up sets the workspace status word
 * (fmlp_device_status reports FMLP_ERR_TIMEOUT).
 *
 *   packed_q, packed_scales : fmlp_pack's [2I x d] matrix quantized (int8,
 *                             f32 [2I x d/64]) with the same tile_T
 *   W_down_q, W_down_scales : W_down [d x I] quantized (int8, f32 [d x I/64])
 *   out                     : f32 [M x d], written by one thread per element
 *                             (no atomics: the same bits on every run)
 *   other arguments, workspace included, as in fmlp_forward.
 * Two launches (gate-up GEMV with the SwiGLU epilogue, down GEMV with the
 * residual) on the CUDA cores; a is rounded to bf16 in between, as in
 * fmlp_forward.
 */
FMLP_API fmlp_status fmlp_forward_q8(const void* x, int64_t M, const void* gamma, float eps,
                                     const void* packed_q, const float* packed_scales, int tile_T,
                                     const void* W_down_q, const float* W_down_scales, int64_t d,
                                     int64_t I, const void* residual, float* out, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * fmlp_sum_partials -- the reduction of a tensor-parallel MLP block:
 *     out = sum_r partials[r] (+ residual)
 * When the intermediate dimension I is split over n ranks (each rank holding
 * whole interleave tiles of packed_Wgu and the matching columns of W_down),
 * each rank's fmlp_forward with residual = NULL gives a partial output, and
 * the block's output is their sum: Eq(1) is linear in the columns of a
 * (FastTPS section 三), and the tensor-parallel layers of "Together AI 的推测
 * 解码内核融合优化" (blog.hotdry.top) reduce the partial outputs across GPUs
 * before the next norm.
 *
 *   partials  : host array of n device pointers, each f32 [M x d].  A pointer
 *               may address another GPU's memory mapped into this one (peer
 *               access); it is read with plain loads, in rank order, so every
 *               rank computing the sum gets the same bits.
 *   n         : 1..16
 *   residual  : bf16 [M x d] added once, or NULL
 *   out       : f32 [M x d] (out_bf16 == 0) or bf16 [M x d] (out_bf16 != 0,
 *               rounded once, to nearest even).  An f32 out may be one of the
 *               partials itself; otherwise it must not overlap them.
 * Runs after the previous work on `stream` (which wrote the partials).
 */
FMLP_API fmlp_status fmlp_sum_partials(const float* const* partials, int n, int64_t M, int64_t d,
                                       const void* residual, void* out, int out_bf16,
                                       void* stream);

/*
 * Token-phase attention step: the GKVC and TPSFLAT components of "FastTPS:
 * An Optimized Method for LLM Token Phase for AI Accelerators" (xllm-io
 * paper review), section 三, components 1-2, Figure 3 and Eq(2).
 *
 * fmlp_attn_workspace_bytes -- bytes of the workspace fmlp_attn_decode needs
 * for B sequences of H query heads over H_kv KV heads of dimension D (0 if
 * the shape is not taken).  Zero-fill it once; the calls keep it zero.
 */
FMLP_API size_t fmlp_attn_workspace_bytes(int64_t B, int H, int H_kv, int D);

/*
 * fmlp_attn_decode -- one new token per sequence: RoPE on q and k at the
 * token's position, in-place append of the new K and V rows to the cache,
 * and the attention of every query head over the cache rows 0..pos.
 *
 *   q        : bf16 [B x H x D], the new token's queries (before RoPE)
 *   k_new    : bf16 [B x H_kv x D], its keys (before RoPE)
 *   v_new    : bf16 [B x H_kv x D], its values
 *   k_cache,
 *   v_cache  : bf16 [B x H_kv x n_max x D], head-major regions of n_max rows
 *              (N_p + N_r of Eq(2)); rows 0..pos[b]-1 hold the earlier tokens.
 *              The call writes row pos[b] of every KV head of sequence b --
 *              the rotated key rounded to bf16 (nearest even), and v_new --
 *              at the Eq(2) offset ((b H_kv + g) n_max + pos[b]) D; rows past
 *              pos[b] do not enter the result.
 *   pos      : int32 [B] on the device, the new token's position (rows held);
 *              0 <= pos[b] < n_ctx <= n_max.  A position outside that range is
 *              not processed: its sequence's outputs and cache are left as
 *              they were and fmlp_device_status reports FMLP_ERR_INVALID_ARG.
 *   n_ctx    : host-side bound on every pos[b] + 1.  The call streams the
 *              rows below n_ctx of every region (rows at and past pos[b] are
 *              read and not used), so n_ctx should be tight: max(pos) + 1.
 *   theta    : RoPE base (> 0): angle_i = pos * theta^(-2i/D), pairs (i, i + D/2)
 *   out      : f32 [B x H x D]: o_h = softmax(q'_h . K_g / sqrt(D)) V_g with
 *              g = h / (H / H_kv), accumulated in f32
 *   workspace: fmlp_attn_workspace_bytes(B, H, H_kv, D) bytes, 16-byte
 *              aligned, zero-filled before first use.  After a call that
 *              reported FMLP_ERR_TIMEOUT or FMLP_ERR_INVALID_ARG through
 *              fmlp_device_status, zero it again before reuse.
 * Shapes taken: D in {64, 96, 128}; H / H_kv in {1, 2, 4, 8}; B * H_kv * n_max
 * + 64 < 2^31.  All pointers 16-byte aligned (pos 4-byte).  Runs after the
 * previous work on `stream` (which may have written the cache or pos).
 * Returns FMLP_ERR_INVALID_ARG before launching anything if an argument is
 * outside these limits.
 */
FMLP_API fmlp_status fmlp_attn_decode(const void* q, const void* k_new, const void* v_new,
                                      void* k_cache, void* v_cache, const int32_t* pos,
                                      int64_t B, int H, int H_kv, int D, int64_t n_max,
                                      int64_t n_ctx, float theta, float* out, void* workspace,
                                      size_t workspace_bytes, void* stream);

/*
 * fmlp_device_status -- synchronise `stream`, read the device status word in
 * `workspace` and reset it to zero.  Returns FMLP_ERR_TIMEOUT if a kernel
 * gave up a bounded wait since the last check, FMLP_ERR_INVALID_ARG if a
 * kernel met a device-side input out of range (an attention position),
 * FMLP_OK otherwise (or FMLP_ERR_CUDA / FMLP_ERR_INVALID_ARG for the call).  After a timeout it also resets the
 * workspace's other control words, so the workspace can be used again; no
 * other call may be using the workspace meanwhile.
 */
FMLP_API fmlp_status fmlp_device_status(void* workspace, void* stream);

/*
 * fmlp_forward_noalloc -- fmlp_forward for callers that cannot allocate
 * device memory.  The pages have no counterpart; this call exists for code
 * that is given no allocator, for example a plug-in run by a host engine that
 * owns all of device memory, or a serving loop that must never call
 * cudaMalloc/cudaFree because those calls can synchronise the device.
 *
 * Instead of a caller workspace it uses one scratch buffer of
 * FMLP_NOALLOC_SCRATCH_BYTES that the library keeps in every GPU's memory
 * from the moment the library is loaded until the process exits.  The call
 * itself allocates nothing.  The first call on a device, and the first after
 * the device's context changed (cudaDeviceReset, or another context made
 * current), looks up the buffer's address in that context
 * (cudaGetSymbolAddress) and caches it for that device and context; make
 * that first call before any stream capture.
 *
 * Arguments, layouts and precision are those of fmlp_forward, minus the
 * workspace.  Requests whose workspace (fmlp_workspace_bytes(M, d, I)) would
 * exceed FMLP_NOALLOC_SCRATCH_BYTES are rejected with FMLP_ERR_UNSUPPORTED
 * before anything is enqueued.  Of the benchmarked shapes, the tiny layer
 * (M=4, d=256, I=688), the Phi-3-mini decode layer (M=1, d=3072, I=8192)
 * and the Llama-3.1-8B decode layer at M=1 and M=8 (d=4096, I=14336) fit;
 * the 8B layer at M=32 (11.9 MiB), the 70B verify layer (M=128, 55 MiB)
 * and the 8B prefill chunk (M=2048, 160 MiB) do not.  Each call first clears the buffer's control
 * words on `stream`, then runs the fmlp_forward kernels on it.  Every call in
 * the process shares the one buffer: calls that may overlap on the GPU (two
 * streams, or two threads) race and must not be issued.  A device-side
 * timeout of such a call is not reported (its outputs are then undefined);
 * use fmlp_forward with a workspace to read the status word.
 */
#define FMLP_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
FMLP_API fmlp_status fmlp_forward_noalloc(const void* x, int64_t M, const void* gamma, float eps,
                                          const void* packed_Wgu, int tile_T, const void* W_down,
                                          int64_t d, int64_t I, const void* residual, float* out,
                                          void* stream);

/* Static, human-readable name of a status code. */
FMLP_API const char* fmlp_status_string(fmlp_status status);

/* The cudaError_t behind the calling thread's most recent FMLP_ERR_CUDA (0 if none). */
FMLP_API int fmlp_last_cuda_error(void);

/*
 * fmlp_set_wait_timeout_ns -- deadline for every bounded wait inside the
 * kernels (a stage of the shared-memory ring that never fills or drains).
 * On expiry a kernel sets the timeout bit of its workspace status word, lets
 * its own in-flight copies land and returns; fmlp_device_status then reports
 * FMLP_ERR_TIMEOUT and the outputs of that call are undefined.  Process-wide;
 * 0 restores the default of one second.  Meant for diagnosis and for testing
 * the timeout path; normal waits last microseconds.
 */
FMLP_API void fmlp_set_wait_timeout_ns(uint64_t ns);

/*
 * fmlp_set_fault_injection -- testing aid.  mode != 0 makes every kernel's
 * producer withhold its last stage of weights, so the consumers' bounded
 * waits expire and the call ends with FMLP_ERR_TIMEOUT in the status word
 * (no GPU fault: the kernels give up and return).  0 turns it off.
 * Process-wide; outputs of affected calls are undefined.
 */
FMLP_API void fmlp_set_fault_injection(int mode);

/* Kernels this library has enqueued in this process so far (all threads, all
 * devices; a launch captured into a CUDA graph counts once, at capture). */
FMLP_API uint64_t fmlp_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* FMLP_H */
