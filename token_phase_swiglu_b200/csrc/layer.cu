// One-launch tensor-core MLP layer (tcgen05 / TMEM) for batches of 1..64
// token rows: RMSNorm, the interleaved gate-up contraction with its SiLU*up
// epilogue, and the down projection with the residual, all in one kernel.
//
// The MLP block of "FastTPS: An Optimized Method for LLM Token Phase for AI
// Accelerators" (xllm-io review): section 三, Eq(1) and the execution flow
// RMSNorm -> interleaved gate-up Matmul -> siLu_Mul -> down projection
// (Figure 4 parts 1-3, fine-grain pipeline scheduling); section 五, Fusion
// MLP Steps 1-3 (the whole block as one kernel).
//
// Both contractions are swap-AB GEMMs D[r, n] = sum_k A[r, k] B[n, k] with
// the weights as A (128 rows per MMA tile) and the token rows as B: for the
// gate-up GEMM N = 2 Mt rows, hi(x*gamma) then lo(x*gamma) of the Mt-row
// token tile (the batch rounded up to 8; hi + lo is x*gamma exactly); for the
// down GEMM N = Nd, the batch rounded up to 16.  Every CTA (one per SM) works
// through its stream-K range of the gate-up GEMM and then its stream-K range
// of the down GEMM, through one continuous ring of shared-memory stages:
//
//   warp 0      weight producer: per stage one TMA copy of KS k-blocks of
//               the packed gate/up rows, then of W_down.  Weights depend on
//               nothing, so the first ring is requested before the
//               dependency on the previous kernel is resolved, and after
//               that the copies wait for nothing but a free stage: HBM keeps
//               streaming W_down while the last gate-up tiles are finished;
//   warp 1      TMEM owner and MMA issuer;
//   warps 2-5   epilogue.  At the start the first CTAs to arrive write the
//               hi/lo operand of x*gamma to the workspace, set out to the
//               residual (or zero), compute 1/RMS per token and clear the
//               tile counters and flags.  Then: SwiGLU
//               of finished gate-up tiles into a (bf16, workspace), and
//               red.add of down tiles into out;
//   warp 6      activation loader: per stage one TMA copy of the hi/lo
//               operand (gate-up) or of a (down).  The operand waits once
//               for the builders' shares; a down stage waits for the gate-up
//               tiles that wrote its k-blocks of a (per-tile flags), until a
//               count shows every tile finished.
//
// Order of the work: each CTA runs the stream-K part of the gate-up GEMM
// first, so the tiles split between two CTAs are finished a third of the way
// in, then its whole tiles; the down GEMM starts with the stages whose
// k-blocks of a come from the split tiles, so it never waits for the last
// whole tiles while there is other work.
//
// Waits on other CTAs: the epilogue waits once for the set-up shares of the
// first CTAs to arrive (running by construction), and the activation loader
// waits for the operand shares of the first CTAs to arrive and for gate-up
// tiles of other CTAs,
// so the kernel assumes that its CTAs (never more than the SMs, one per SM)
// become resident together, as they do when nothing else holds SMs
// indefinitely.  Every wait is bounded: on expiry the CTA flags the status
// word, lets its copies land, frees its TMEM and returns.
#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"
#include "tmap.h"

#include <algorithm>
#include <cstring>
#include <mutex>
#include <set>

namespace fmlp {
namespace {

constexpr int kLayerThreads = 224;     // warps 0-6
constexpr int kLayerMaxStages = 8;
constexpr int kLayerMaxMt = 64;
constexpr int kLayerMaxInit = 8;       // CTAs that do the set-up shares
constexpr int kLayerMaxBuild = 32;     // CTAs that write the hi/lo operand
constexpr uint64_t kLayerDrainNs = 2000000ull;  // copies land within microseconds
constexpr int kBarEpi = 1;             // named barrier of the epilogue warps (0 is __syncthreads)

struct LayerParams {
  CUtensorMap p_map;   // packed gate/up [2I x d], 3-D k-block view, box (64, 128, KS)
  CUtensorMap wd_map;  // W_down [d x I], box (64, 128, KS)
  CUtensorMap b_map;   // hi/lo operand [2 Mt x d] (workspace), box (64, 2 Mt, KS)
  CUtensorMap a_map;   // a [M x I] (workspace), box (64, Nd, KS): rows past M land as zeros
  Sched sg;            // gate-up: stream-K over the tiles past dp waves, then the dp
                       // whole tiles of this CTA
  Sched sd1, sd2;      // down, stream-K: stages [S1, KBd) (part 1), [0, S1) (part 2)
  const __nv_bfloat16* x;
  const __nv_bfloat16* gamma;
  const __nv_bfloat16* residual;
  __nv_bfloat16* b_hl; // [2 Mt x d]: rows [0, Mt) hi(x*gamma), [Mt, 2 Mt) lo
  __nv_bfloat16* a;    // [M x I] intermediate
  float* out;          // [M x d] f32 sum (set to the residual or zero, then added into)
  __nv_bfloat16* out_bf16;  // [M x d] or null: out rounded to bf16 by the last CTA to finish
  float* rinv;         // [M]
  float* partials;     // [ctas][2][2 Mt][128]
  uint32_t* counters;  // gate-up tile arrivals [tiles_g]
  int ncounters;
  uint32_t* ticket;    // arrival order of the CTAs
  uint32_t* inited;    // set-up shares done
  uint32_t* done;      // CTAs finished
  uint32_t* gu_done;   // gate-up tiles finished (a written)
  uint32_t* a_ready;   // [tiles_g] gate-up tile j finished: k-block j of a is written
  uint32_t* hl_done;   // operand shares written
  uint32_t* status;
  uint64_t wait_ns;
  float eps;
  int M, d, I, T;
  int Mt;              // gate-up token tile (M rounded up to 8): MMA N = 2 Mt
  int Nd;              // down GEMM MMA N (M rounded up to 16)
  int Cg, Cd;          // accumulator chains per tile (gate-up, down)
  int KS;              // k-blocks per stage
  int KBg, KBd;        // k-blocks of d and of I
  int S1;              // first down stage of part 1 (all its k-blocks from stream-K tiles)
  int stages, stage_bytes;
  int bufcols;         // TMEM columns per accumulator buffer
  uint32_t tmem_cols;
  int n_init;          // CTAs that do the set-up shares
  int n_build;         // CTAs that write the hi/lo operand (the first to arrive)
  int drop_last;       // fault injection: the producers withhold their last stage
};

struct LayerShared {
  uint64_t full[kLayerMaxStages];   // 2 arrivals: weight copy, activation copy
  uint64_t empty[kLayerMaxStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  int last;
  int head_done;
  int k_issued;        // stages whose weights the producer issued
  int kb_issued;       // stages whose activations the loader issued
  uint32_t ticket;
  int ready;           // epilogue: set-up shares seen (1) or gave up (-1)
  int last_cta;        // this CTA was the last to finish
  float rinv_s[kLayerMaxMt];
};

__device__ __forceinline__ void layer_flag(LayerShared* sh, uint32_t* status) {
  sh->abort = 1;
  atomicOr(status, kStatusTimeout);
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// One thread waits until *ctr >= target (acquire), at most limit_ns, giving
// up early if *abort is set; false if it gave up.
__device__ bool wait_count(const uint32_t* ctr, uint32_t target, uint64_t limit_ns,
                           volatile int* abort) {
  if (ld_acquire_gpu(ctr) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    __nanosleep(64);
    if (ld_acquire_gpu(ctr) >= target) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// mbar_wait_bounded for long waits: polls with a short sleep between tries,
// so that the waiting warp leaves its scheduler's issue slots to others.
__device__ bool mbar_wait_backoff(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                  volatile int* abort) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    __nanosleep(128);
    if (mbar_test(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// Segment s of a schedule, stream-K part first: the range [u0, u1) over the
// tiles past the data-parallel waves (segments 0..nsk-1), then the dp whole
// tiles s * ctas + this CTA.  Tile t, stages [kb0, kb1); false past the end.
__device__ __forceinline__ bool sched_segment(const Sched& S, int64_t u0, int64_t u1, int nsk,
                                              int s, int& t, int& kb0, int& kb1) {
  if (s >= nsk) {
    s -= nsk;
    if (s >= S.dp) return false;
    t = s * S.ctas + (int)blockIdx.x;
    kb0 = 0;
    kb1 = S.KB;
    return true;
  }
  if (u0 >= u1) return false;
  const int tl = (int)(u0 / S.KB) + s;
  const int64_t tb = (int64_t)tl * S.KB;
  if (tb >= u1) return false;
  t = S.sk_tile0() + tl;
  kb0 = (int)(max(u0, tb) - tb);
  kb1 = (int)(min(u1, tb + S.KB) - tb);
  return true;
}

// Stream-K segments of [u0, u1).
__device__ __forceinline__ int sk_segments(const Sched& S, int64_t u0, int64_t u1) {
  if (u0 >= u1) return 0;
  return (int)((u1 - 1) / S.KB - u0 / S.KB) + 1;
}

enum Phase { kGateUp = 0, kDown1 = 1, kDown2 = 2 };

// This CTA's whole work: its gate-up segments (stream-K part, then its whole
// tiles), then its segments of down part 1 (stages from S1 on) and of down
// part 2 (stages below S1).  Stage indices are absolute.
struct Work {
  int64_t ug0, ug1, u10, u11, u20, u21;
  int nskg, nsg, ns1, ns2, nk;
  __device__ void init(const LayerParams& p) {
    p.sg.range(blockIdx.x, ug0, ug1);
    p.sd1.range(blockIdx.x, u10, u11);
    p.sd2.range(blockIdx.x, u20, u21);
    nskg = sk_segments(p.sg, ug0, ug1);
    nsg = nskg + p.sg.dp;
    ns1 = sk_segments(p.sd1, u10, u11);
    ns2 = sk_segments(p.sd2, u20, u21);
    nk = (int)(ug1 - ug0) + p.sg.dp * p.sg.KB + (int)(u11 - u10) + (int)(u21 - u20);
  }
  __device__ __forceinline__ int segments() const { return nsg + ns1 + ns2; }
  __device__ __forceinline__ int stages() const { return nk; }
  __device__ __forceinline__ bool seg(const LayerParams& p, int s, int& phase, int& t, int& kb0,
                                      int& kb1) const {
    if (s < nsg) {
      phase = kGateUp;
      return sched_segment(p.sg, ug0, ug1, nskg, s, t, kb0, kb1);
    }
    if (s < nsg + ns1) {
      phase = kDown1;
      const bool r = sched_segment(p.sd1, u10, u11, ns1, s - nsg, t, kb0, kb1);
      kb0 += p.S1;
      kb1 += p.S1;
      return r;
    }
    phase = kDown2;
    return sched_segment(p.sd2, u20, u21, ns2, s - nsg - ns1, t, kb0, kb1);
  }
};

// ---------------------------------------------------------------------------
// Epilogue helpers (warps 2-5; thread = TMEM lane = accumulator row)
// ---------------------------------------------------------------------------
// CW consecutive columns at `col` of an accumulator, summed over its C chains
// (chain c at column offset c * stride).
template <int CW>
__device__ __forceinline__ void acc_cols(uint32_t tb, int col, int C, int stride,
                                         float (&v)[CW]) {
  uint32_t r[CW];
  tmem_ld<CW>(tb + col, r);
  tmem_wait();
#pragma unroll
  for (int j = 0; j < CW; ++j) v[j] = __uint_as_float(r[j]);
  for (int c = 1; c < C; ++c) {
    tmem_ld<CW>(tb + (uint32_t)(c * stride) + col, r);
    tmem_wait();
#pragma unroll
    for (int j = 0; j < CW; ++j) v[j] += __uint_as_float(r[j]);
  }
}

// SwiGLU of CW token columns [c0, c0 + CW) of a finished gate-up row: the
// gate row and its up row sit in lanes T apart of the same warp (rows
// [0, T) of each 2T-row interleave tile are gate, [T, 2T) up).  The gate lane
// finishes the first half of the chunk's tokens, the up lane the second.
template <int CW>
__device__ __forceinline__ void swiglu_columns(const LayerParams& p, int row,
                                               const float (&vals)[CW], int c0,
                                               const float* rv) {
  constexpr int H = CW / 2;
  const int T = p.T;
  const bool is_gate = (row % (2 * T)) < T;
  float g[H], u[H];
#pragma unroll
  for (int j = 0; j < H; ++j) {
    const float send = is_gate ? vals[H + j] : vals[j];
    const float recv = __shfl_xor_sync(0xffffffffu, send, T);
    g[j] = is_gate ? vals[j] : recv;
    u[j] = is_gate ? recv : vals[H + j];
  }
  const int pair = (row / (2 * T)) * T + (row % T);
  const int m0 = c0 + (is_gate ? 0 : H);
  if (row < 2 * p.I) {
#pragma unroll
    for (int j = 0; j < H; ++j) {
      const int m = m0 + j;
      if (m < p.M) {
        const float r = rv[m];
        p.a[(int64_t)m * p.I + pair] = __float2bfloat16_rn(silu_mul_fast(g[j] * r, u[j] * r));
      }
    }
  }
}

// Finish gate-up tile t: this CTA's accumulator (hi + lo columns) plus the
// other contributors' partials, then SwiGLU into a.
template <int CW>
__device__ void finish_gateup(const LayerParams& p, int t, uint32_t tb, bool whole, int c_first,
                              int c_last, int r_local, const float* rv) {
  const int N = 2 * p.Mt;
  const int row = t * kBM + r_local;
  for (int c0 = 0; c0 < p.Mt; c0 += CW) {
    float vals[CW];
#pragma unroll
    for (int j = 0; j < CW; ++j) vals[j] = 0.f;
    if (!whole) {
      for (int cc = c_first; cc <= c_last; ++cc) {
        if (cc == (int)blockIdx.x) continue;
        int64_t cu0, cu1;
        p.sg.range(cc, cu0, cu1);
        const int slot = (t == p.sg.sk_tile0() + (int)(cu0 / p.sg.KB)) ? 0 : 1;
        const float* part = p.partials + ((size_t)cc * 2 + slot) * (size_t)N * kBM;
#pragma unroll
        for (int j = 0; j < CW; ++j)
          vals[j] += __ldcg(part + (size_t)(c0 + j) * kBM + r_local) +
                     __ldcg(part + (size_t)(p.Mt + c0 + j) * kBM + r_local);
      }
    }
    float acc[CW];
    acc_cols<CW>(tb, c0, p.Cg, N, acc);  // hi half of x*gamma
#pragma unroll
    for (int j = 0; j < CW; ++j) vals[j] += acc[j];
    acc_cols<CW>(tb, p.Mt + c0, p.Cg, N, acc);  // lo half
#pragma unroll
    for (int j = 0; j < CW; ++j) vals[j] += acc[j];
    swiglu_columns<CW>(p, row, vals, c0, rv);
  }
}

// Store this CTA's partial accumulator of gate-up tile t (chains summed).
template <int CW>
__device__ void store_partial(const LayerParams& p, uint32_t tb, float* part, int r_local) {
  const int N = 2 * p.Mt;
  for (int c = 0; c < N; c += CW) {
    float v[CW];
    acc_cols<CW>(tb, c, p.Cg, N, v);
#pragma unroll
    for (int j = 0; j < CW; ++j) __stcg(part + (size_t)(c + j) * kBM + r_local, v[j]);
  }
}

// Down tile t: add this CTA's accumulator (its split-K share) into out.
template <int CW>
__device__ void add_down(const LayerParams& p, int t, uint32_t tb, int r_local) {
  const int n = t * kBM + r_local;
  for (int c0 = 0; c0 < p.Nd; c0 += CW) {
    float v[CW];
    acc_cols<CW>(tb, c0, p.Cd, p.Nd, v);
    if (n < p.d) {
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        const int m = c0 + j;
        if (m < p.M) atomicAdd(p.out + (int64_t)m * p.d + n, v[j]);
      }
    }
  }
}

// The set-up share of the CTA that arrived t-th (t < n_init), by the 128
// epilogue threads: clear a share of the tile counters (and, for t == 0, the
// gate-up completion count), set a share of out to the residual or zero, and
// compute 1/RMS of the token rows m == t (mod n_init).
__device__ void setup_share(const LayerParams& p, int t, int et) {
  for (int i = t * 128 + et; i < p.ncounters; i += p.n_init * 128) p.counters[i] = 0u;
  if (t == 0 && et == 0) *p.gu_done = 0u;
  const int64_t n4 = (int64_t)p.M * p.d / 4;
  const int64_t q0 = n4 * t / p.n_init, q1 = n4 * (t + 1) / p.n_init;
  for (int64_t i = q0 + et; i < q1; i += 128) {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p.residual) {
      const uint2 r = __ldg(reinterpret_cast<const uint2*>(p.residual) + i);
      v = make_float4(bf16lo(r.x), bf16hi(r.x), bf16lo(r.y), bf16hi(r.y));
    }
    reinterpret_cast<float4*>(p.out)[i] = v;
  }
  const int e = et >> 5, lane = et & 31;
  const int nv = p.d / 8;
  for (int m = t + p.n_init * e; m < p.M; m += p.n_init * 4) {
    float ss = 0.f;
    for (int v = lane; v < nv; v += 32) {
      const uint4 xv = ld_keep(p.x + (int64_t)m * p.d + (int64_t)v * 8);
      const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float x0 = bf16lo(w[q]), x1 = bf16hi(w[q]);
        ss = fmaf(x0, x0, ss);
        ss = fmaf(x1, x1, ss);
      }
    }
    ss = warp_sum(ss);
    if (lane == 0) p.rinv[m] = 1.0f / sqrtf(ss / (float)p.d + p.eps);
  }
}

// Two f32 values rounded to nearest-even bf16, packed (lo in the low half).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Split 8 values s = x * gamma (exact in f32: two 8-bit significands) into
// hi = bf16(s) and lo = bf16(s - hi), which is exact as well (s - hi is an
// integer multiple of s's last bit, at most 2^7 of them).
__device__ __forceinline__ void split8(const uint4& xv, const uint4& gv, uint4& hv, uint4& lv) {
  const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
  uint32_t hw[4], lw[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float s0 = bf16lo(xw[e]) * bf16lo(gw[e]), s1 = bf16hi(xw[e]) * bf16hi(gw[e]);
    hw[e] = pack_bf16x2(s0, s1);
    lw[e] = pack_bf16x2(s0 - bf16lo(hw[e]), s1 - bf16hi(hw[e]));
  }
  hv = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  lv = make_uint4(lw[0], lw[1], lw[2], lw[3]);
}

// One thread waits until the a k-blocks of down stage kb are written: every
// gate-up tile finished (one count, after which *all is set and no further
// stage waits), or the tiles of this stage's k-blocks.  False on expiry.
__device__ bool wait_ready(const LayerParams& p, int kb, bool* all, volatile int* abort) {
  const int j0 = kb * p.KS, j1 = min(j0 + p.KS, p.KBd);
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (ld_acquire_gpu(p.gu_done) >= (uint32_t)p.sg.tiles) {
      *all = true;
      return true;
    }
    bool ready = true;
    for (int j = j0; j < j1; ++j) ready = ready && ld_acquire_gpu(p.a_ready + j) != 0u;
    if (ready) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > p.wait_ns) return false;
    __nanosleep(64);
  }
}

// Share b (of n_build) of the hi/lo operand, by the 128 epilogue threads of
// the CTA that arrived b-th: the [2 Mt x d] matrix of hi(x*gamma) rows then
// lo(x*gamma) rows (zeros for the padding rows M..Mt-1), cut into equal
// shares of 16-byte chunks.
__device__ void operand_share(const LayerParams& p, int b, int et) {
  // and share b of the a-ready flags: every share is written before the
  // first gate-up MMA anywhere, so before any tile can finish
  {
    const int j0 = p.sg.tiles * b / p.n_build, j1 = p.sg.tiles * (b + 1) / p.n_build;
    for (int j = j0 + et; j < j1; j += 128) p.a_ready[j] = 0u;
  }
  const int nv = p.d / 8;
  const int64_t n_items = (int64_t)p.Mt * nv;
  const int64_t q0 = n_items * b / p.n_build;
  const int64_t q1 = n_items * (b + 1) / p.n_build;
  for (int64_t i = q0 + et; i < q1; i += 128) {
    const int m = (int)(i / nv), v = (int)(i - (int64_t)m * nv);
    uint4 xv = make_uint4(0, 0, 0, 0);
    if (m < p.M) xv = ld_keep(p.x + (int64_t)m * p.d + (int64_t)v * 8);
    const uint4 gv = ld_keep(p.gamma + (int64_t)v * 8);
    uint4 hv, lv;
    split8(xv, gv, hv, lv);
    reinterpret_cast<uint4*>(p.b_hl + (int64_t)m * p.d)[v] = hv;
    reinterpret_cast<uint4*>(p.b_hl + (int64_t)(p.Mt + m) * p.d)[v] = lv;
  }
}

__global__ void __launch_bounds__(kLayerThreads, 1) tc_layer(const __grid_constant__ LayerParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ LayerShared sh;
  uint8_t* stage0 = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int a_bytes = p.KS * kATileBytes;   // weights of a stage
  const int gb = p.KS * 2 * p.Mt * 128;     // gate-up activations of a stage
  const int db = p.KS * p.Nd * 128;         // down activations of a stage
  Work w;
  w.init(p);
  const int nseg = w.segments(), nk = w.stages();

  if (threadIdx.x == 0) {
    for (int j = 0; j < p.stages; ++j) {
      mbar_init(&sh.full[j], 2);
      mbar_init(&sh.empty[j], 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(&sh.acc_full[j], 1);
      mbar_init(&sh.acc_empty[j], 4);
    }
    mbar_init(&sh.mma_done, 1);
    sh.abort = 0;
    sh.k_issued = sh.kb_issued = 0;
    sh.ready = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(&sh.tmem_base, p.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_launch_dependents();
  const uint32_t tmem = sh.tmem_base;
  volatile int* abort = &sh.abort;

  if (warp == 0) {
    // ---------------- weight producer ----------------
    if (lane == 0) {
      const uint64_t pol_w = evict_first_policy();
      int k = 0;
      bool ok = true;
      for (int s = 0; s < nseg && ok && !*abort; ++s) {
        int phase, t, kb0, kb1;
        w.seg(p, s, phase, t, kb0, kb1);
        const bool gu = phase == kGateUp;
        for (int kb = kb0; kb < kb1; ++kb, ++k) {
          if (p.drop_last && k == nk - 1) {
            ok = false;
            break;
          }
          const int slot = k % p.stages;
          if (k >= p.stages &&
              !mbar_wait_bounded(&sh.empty[slot], (uint32_t)(((k / p.stages) - 1) & 1),
                                 p.wait_ns, abort)) {
            if (!*abort) layer_flag(&sh, p.status);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sh.full[slot], (uint32_t)a_bytes);
          tma_load_3d(stage0 + (size_t)slot * p.stage_bytes, gu ? &p.p_map : &p.wd_map, 0,
                      t * kBM, kb * p.KS, &sh.full[slot], pol_w);
          sh.k_issued = k + 1;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc_g = idesc_bf16(2 * p.Mt), idesc_d = idesc_bf16(p.Nd);
      int k = 0;
      bool ok = true;
      for (int s = 0; s < nseg && ok; ++s) {
        int phase, t, kb0, kb1;
        w.seg(p, s, phase, t, kb0, kb1);
        const bool gu = phase == kGateUp;
        const int buf = s & 1;
        if (!mbar_wait_bounded(&sh.acc_empty[buf], (uint32_t)(((s >> 1) & 1) ^ 1), p.wait_ns,
                               abort)) {
          if (!*abort) layer_flag(&sh, p.status);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(buf * p.bufcols);
        const int C = gu ? p.Cg : p.Cd;
        const int N = gu ? 2 * p.Mt : p.Nd;
        const uint32_t idesc = gu ? idesc_g : idesc_d;
        const uint32_t b_kblock = (uint32_t)(N * kBK * 2);
        const int KBtot = gu ? p.KBg : p.KBd;
        for (int kb = kb0; kb < kb1; ++kb, ++k) {
          const int slot = k % p.stages;
          if (!mbar_wait_bounded(&sh.full[slot], (uint32_t)((k / p.stages) & 1), p.wait_ns,
                                 abort)) {
            if (!*abort) layer_flag(&sh, p.status);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(stage0 + (size_t)slot * p.stage_bytes);
          const uint32_t b_addr = a_addr + (uint32_t)a_bytes;
          // the last stage of K may hold fewer than KS k-blocks (zero fill)
          const int nkb = min(p.KS, KBtot - kb * p.KS);
          for (int kbi = 0; kbi < nkb; ++kbi) {
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              // k-slice kk accumulates into chain kk % C: C independent MMA chains
              const int c = kk % C;
              const uint32_t acc = (kb == kb0 && kbi == 0 && kk < C) ? 0u : 1u;
              mma_bf16(d_tmem + (uint32_t)(c * N),
                       sw128_desc(a_addr + (uint32_t)(kbi * kATileBytes) + kk * 32),
                       sw128_desc(b_addr + (uint32_t)kbi * b_kblock + kk * 32), idesc, acc);
            }
          }
          mma_commit(&sh.empty[slot]);  // stage reusable once these MMAs finish
        }
        if (ok) mma_commit(&sh.acc_full[buf]);
      }
      // every MMA issued so far has completed once this commit arrives
      mma_commit(&sh.mma_done);
      mbar_wait_bounded(&sh.mma_done, 0, kLayerDrainNs * 500, nullptr);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ---------------- epilogue (warps 2-5) ----------------
    const int q = warp & 3;               // TMEM lane quadrant of this warp
    const int r_local = 32 * q + lane;    // accumulator row = TMEM lane
    const int et = threadIdx.x - 64;      // 0..127
    grid_dependency_wait();  // out, x, the residual and the workspace belong to this call now
    if (et == 0) sh.ticket = atomicAdd(p.ticket, 1u);
    named_barrier_sync(kBarEpi, 128);
    const uint32_t tk = sh.ticket;
    if (tk < (uint32_t)p.n_build) {
      operand_share(p, (int)tk, et);
      __threadfence();
      fence_proxy_async_global();  // the operand is read by TMA copies (async proxy)
      named_barrier_sync(kBarEpi, 128);
      if (et == 0) atomicAdd(p.hl_done, 1u);
    }
    if (tk < (uint32_t)p.n_init) {
      setup_share(p, (int)tk, et);
      __threadfence();
      named_barrier_sync(kBarEpi, 128);
      if (et == 0) atomicAdd(p.inited, 1u);
    }
    if (et == 0) {
      const bool ok = wait_count(p.inited, (uint32_t)p.n_init, p.wait_ns, abort);
      if (!ok && !*abort) layer_flag(&sh, p.status);
      sh.ready = ok ? 1 : -1;
    }
    named_barrier_sync(kBarEpi, 128);
    bool failed = sh.ready != 1;
    if (!failed)
      for (int i = et; i < p.Mt; i += 128) sh.rinv_s[i] = i < p.M ? __ldcg(p.rinv + i) : 0.f;
    named_barrier_sync(kBarEpi, 128);
    for (int s = 0; s < nseg && !failed; ++s) {
      int phase, t, kb0, kb1;
      w.seg(p, s, phase, t, kb0, kb1);
      const bool gu = phase == kGateUp;
      const int buf = s & 1;
      // A gate-up tile shared by two CTAs: the one holding its first k-blocks
      // reaches it at the end of its range, long after the other has stored
      // its partial.  Look at the tile's counter while the MMAs still run: if
      // the other contributor has arrived, finish the tile directly.
      bool head_only = false;
      if (gu && !(kb0 == 0 && kb1 == p.sg.KB) && kb0 == 0) {
        const int64_t tu = (int64_t)(t - p.sg.sk_tile0()) * p.sg.KB;
        if (p.sg.cta_of(tu + p.sg.KB - 1) == (int)blockIdx.x + 1) {
          if (et == 0) sh.head_done = ld_acquire_gpu(p.counters + t) == 1u;
          head_only = true;
        }
      }
      // One thread waits for the accumulator; the others block in the
      // barrier, which issues nothing.
      bool got = true;
      if (et == 0) {
        got = mbar_wait_backoff(&sh.acc_full[buf], (uint32_t)((s >> 1) & 1), p.wait_ns, abort);
        if (!got && !*abort) layer_flag(&sh, p.status);
      }
      if (epilogue_barrier_any(!got)) break;  // also publishes sh.head_done
      mbar_test(&sh.acc_full[buf], (uint32_t)((s >> 1) & 1));  // acquire in every thread
      tc_fence_after();
      const uint32_t tb = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * p.bufcols);
      if (!gu) {
        // split-K by accumulation: out already holds the residual (or zero)
        if (p.Nd % 32 == 0) add_down<32>(p, t, tb, r_local);
        else add_down<16>(p, t, tb, r_local);
      } else {
        const bool whole = kb0 == 0 && kb1 == p.sg.KB;
        const int64_t tu = (int64_t)(t - p.sg.sk_tile0()) * p.sg.KB;  // stream-K tiles only
        const int c_first = whole ? 0 : p.sg.cta_of(tu);
        const int c_last = whole ? 0 : p.sg.cta_of(tu + p.sg.KB - 1);
        bool finalize = whole;
        if (head_only && sh.head_done) {
          finalize = true;  // the other contributor's partial is visible (acquire above)
        } else if (!whole) {
          const int slot = (t == p.sg.sk_tile0() + (int)(w.ug0 / p.sg.KB)) ? 0 : 1;
          float* part = p.partials + ((size_t)blockIdx.x * 2 + slot) * (size_t)(2 * p.Mt) * kBM;
          if ((2 * p.Mt) % 32 == 0) store_partial<32>(p, tb, part, r_local);
          else store_partial<16>(p, tb, part, r_local);
          __threadfence();
          named_barrier_sync(kBarEpi, 128);
          if (et == 0) sh.last = atomicAdd(p.counters + t, 1u) == (uint32_t)(c_last - c_first);
          named_barrier_sync(kBarEpi, 128);
          finalize = sh.last;
          if (finalize) __threadfence();
        }
        if (finalize) {
          // a chunk width that divides the token tile (a multiple of 8)
          if (p.Mt % 32 == 0)
            finish_gateup<32>(p, t, tb, whole, c_first, c_last, r_local, sh.rinv_s);
          else if (p.Mt % 16 == 0)
            finish_gateup<16>(p, t, tb, whole, c_first, c_last, r_local, sh.rinv_s);
          else
            finish_gateup<8>(p, t, tb, whole, c_first, c_last, r_local, sh.rinv_s);
          // a of this tile is written: count it for the down phase's copies
          __threadfence();
          fence_proxy_async_global();
          named_barrier_sync(kBarEpi, 128);
          if (et == 0) {
            if (!whole) atomicExch(p.counters + t, 0u);
            atomicExch(p.a_ready + t, 1u);
            atomicAdd(p.gu_done, 1u);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.acc_empty[buf]);
    }
    // with a bf16 output the last CTA to finish reads the sum: this thread's
    // adds into it are visible before its CTA counts itself finished
    if (p.out_bf16) __threadfence();
  } else {
    // ---------------- activation loader (warp 6) ----------------
    if (lane == 0) {
      uint64_t pol_act;
      asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol_act));
      grid_dependency_wait();  // the counters below belong to this call only after it
      bool ok = wait_count(p.hl_done, (uint32_t)p.n_build, p.wait_ns, abort);
      if (!ok && !*abort) layer_flag(&sh, p.status);
      fence_proxy_async_global();  // the operand was written by generic stores
      bool all_ready = false;  // every gate-up tile finished
      int k = 0;
      for (int s = 0; s < nseg && ok && !*abort; ++s) {
        int phase, t, kb0, kb1;
        w.seg(p, s, phase, t, kb0, kb1);
        const bool gu = phase == kGateUp;
        for (int kb = kb0; kb < kb1; ++kb, ++k) {
          if (p.drop_last && k == nk - 1) {
            ok = false;
            break;
          }
          const int slot = k % p.stages;
          if (k >= p.stages &&
              !mbar_wait_bounded(&sh.empty[slot], (uint32_t)(((k / p.stages) - 1) & 1),
                                 p.wait_ns, abort)) {
            if (!*abort) layer_flag(&sh, p.status);
            ok = false;
            break;
          }
          uint8_t* b_dst = stage0 + (size_t)slot * p.stage_bytes + a_bytes;
          if (gu) {
            mbar_arrive_expect_tx(&sh.full[slot], (uint32_t)gb);
            tma_load_3d(b_dst, &p.b_map, 0, 0, kb * p.KS, &sh.full[slot], pol_act);
          } else {
            // The stage reads a k-blocks [kb KS, kb KS + nkb): those of gate-up
            // tiles [kb KS, kb KS + nkb).  Part 1 takes the stream-K tiles,
            // finished a third of the way into the gate-up phase; part 2 the
            // whole tiles, finished at the end of it, each waited for alone.
            if (!all_ready) {
              if (!wait_ready(p, kb, &all_ready, abort)) {
                if (!*abort) layer_flag(&sh, p.status);
                ok = false;
                break;
              }
              fence_proxy_async_global();  // a was written by generic stores
            }
            mbar_arrive_expect_tx(&sh.full[slot], (uint32_t)db);
            tma_load_3d(b_dst, &p.a_map, 0, 0, kb * p.KS, &sh.full[slot], pol_act);
          }
          sh.kb_issued = k + 1;
        }
      }
    }
    __syncwarp();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (sh.abort) {
      // let every issued copy land before the CTA leaves (bounded: a stage
      // whose other copy was never issued does not complete)
      const int n = max(sh.k_issued, sh.kb_issued);
      for (int k = max(0, n - p.stages); k < n; ++k)
        mbar_wait_bounded(&sh.full[k % p.stages], (uint32_t)((k / p.stages) & 1),
                          kLayerDrainNs, nullptr);
    }
    // this CTA's adds into out are visible before it counts itself finished
    if (p.out_bf16) __threadfence();
    // Every CTA took its ticket, wrote its shares and finished its waits on
    // the counters: the last one here leaves them at zero for the next call.
    const bool last = atomicAdd(p.done, 1u) == gridDim.x - 1;
    if (last) {
      atomicExch(p.ticket, 0u);
      atomicExch(p.inited, 0u);
      atomicExch(p.gu_done, 0u);
      atomicExch(p.hl_done, 0u);
      atomicExch(p.done, 0u);
    }
    sh.last_cta = last;
  }
  __syncthreads();
  if (p.out_bf16 && sh.last_cta) {
    // the last CTA rounds the finished sum to the bf16 output
    __threadfence();
    const int64_t n4 = (int64_t)p.M * p.d / 4;
    for (int64_t i = threadIdx.x; i < n4; i += blockDim.x) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(p.out) + i);
      reinterpret_cast<uint2*>(p.out_bf16)[i] =
          make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
struct LayerPlan {
  int Mt = 0, Nd = 0, Cg = 0, Cd = 0, KS = 0, stages = 0, stage_bytes = 0, bufcols = 0;
  uint32_t tmem_cols = 0;
  size_t smem = 0;
};

uint32_t pow2_cols(uint32_t n) {
  uint32_t c = 32;
  while (c < n) c <<= 1;
  return c;
}

// Token tile Mt = M rounded up to 8 (the gate-up MMA's N = 2 Mt and the down
// MMA's Nd, M rounded up to 16, are multiples of 16 as an MMA of 128 rows
// requires); C accumulator chains per tile so that 2 C N <= 512 TMEM columns
// with two buffers; KS k-blocks per stage, the largest that leaves a ring of
// three stages (or two stages of one k-block).
bool make_layer_plan(int64_t M, int max_smem_optin, LayerPlan& pl) {
  if (M < 1 || M > kLayerMaxMt) return false;
  pl.Mt = (int)((M + 7) / 8 * 8);
  pl.Nd = (int)((M + 15) / 16 * 16);
  const int Ng = 2 * pl.Mt;
  pl.Cg = 4 * Ng <= 256 ? 4 : (2 * Ng <= 256 ? 2 : 1);
  pl.Cd = 4 * pl.Nd <= 256 ? 4 : (2 * pl.Nd <= 256 ? 2 : 1);
  pl.bufcols = std::max(pl.Cg * Ng, pl.Cd * pl.Nd);
  pl.tmem_cols = pow2_cols((uint32_t)(2 * pl.bufcols));
  if (pl.tmem_cols > 512) return false;
  // static shared memory (LayerShared, 1 KB with its alignment) and the
  // 1024-byte alignment slack of the stages come off the opt-in maximum
  const size_t budget = (size_t)max_smem_optin - 2048 - 1024;
  for (int ks = 4; ks >= 1; --ks) {
    const int bytes = ks * kATileBytes + ks * std::max(Ng, pl.Nd) * 128;
    const int sb = (bytes + 1023) / 1024 * 1024;
    const int st = (int)std::min<size_t>(kLayerMaxStages, budget / sb);
    if (st >= 3 || (ks == 1 && st >= 2)) {
      pl.KS = ks;
      pl.stage_bytes = sb;
      pl.stages = st;
      break;
    }
  }
  if (pl.stages < 2) return false;
  pl.smem = (size_t)pl.stages * pl.stage_bytes + 1024;
  return true;
}

cudaError_t allow_layer_smem(const DeviceInfo& dev) {
  static std::mutex mu;
  static std::set<int> done;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count(dev.device)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(tc_layer, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       dev.max_smem_optin - 2048);
  if (e == cudaSuccess) done.insert(dev.device);
  return e;
}

Sched layer_sched(int tiles, int KB, int ctas, int dp) {
  Sched S;
  S.KB = KB;
  S.ntok = 1;
  S.tiles = tiles;
  S.ctas = ctas;
  S.dp = dp;
  return S;
}

}  // namespace

bool layer_supported(int64_t M, int64_t d, int64_t I, int T, const DeviceInfo& dev) {
  LayerPlan pl;
  return M >= 1 && M <= kLayerMaxMt && d % 64 == 0 && I % 64 == 0 && (T == 8 || T == 16) &&
         make_layer_plan(M, dev.max_smem_optin, pl);
}

LayerSizes layer_sizes(int64_t M, int64_t d, int64_t I, int sm_count) {
  LayerSizes z;
  if (M < 1 || M > kLayerMaxMt) return z;
  const int Mt = (int)((M + 7) / 8 * 8);
  z.b_hl = (size_t)2 * Mt * d * 2;
  z.rinv = (size_t)M * 4;
  z.partials = (size_t)sm_count * 2 * (2 * Mt) * kBM * 4;
  z.counters = (size_t)(((2 * I + kBM - 1) / kBM) + 2) * 4;
  z.a_ready = (size_t)((2 * I + kBM - 1) / kBM) * 4;
  return z;
}

cudaError_t launch_tc_layer(const void* x, int64_t M, const void* gamma, float eps,
                            const void* P, int T, const void* W_down, int64_t d, int64_t I,
                            const void* residual, float* out, void* out_bf16,
                            const LayerWorkspace& ws, const DeviceInfo& dev,
                            cudaStream_t stream) {
  LayerPlan pl;
  if (!make_layer_plan(M, dev.max_smem_optin, pl)) return cudaErrorInvalidValue;
  cudaError_t e = allow_layer_smem(dev);
  if (e != cudaSuccess) return e;
  static_assert(sizeof(LayerParams) <= 4096, "kernel parameters");
  LayerParams p;
  memset(&p, 0, sizeof(p));
  e = encode_tmap_kblocks_bf16(&p.p_map, P, (uint64_t)(2 * I), (uint64_t)d, (uint64_t)d * 2, kBM,
                               (uint32_t)pl.KS);
  if (e == cudaSuccess)
    e = encode_tmap_kblocks_bf16(&p.wd_map, W_down, (uint64_t)d, (uint64_t)I, (uint64_t)I * 2,
                                 kBM, (uint32_t)pl.KS);
  if (e == cudaSuccess)
    e = encode_tmap_kblocks_bf16(&p.b_map, ws.b_hl, (uint64_t)(2 * pl.Mt), (uint64_t)d,
                                 (uint64_t)d * 2, (uint32_t)(2 * pl.Mt), (uint32_t)pl.KS);
  if (e == cudaSuccess)
    e = encode_tmap_kblocks_bf16(&p.a_map, ws.a, (uint64_t)M, (uint64_t)I, (uint64_t)I * 2,
                                 (uint32_t)pl.Nd, (uint32_t)pl.KS);
  if (e != cudaSuccess) return e;
  // Gate-up: 2I/128 row tiles of KBg stages; down: d/128 row tiles of KBd
  // stages.  Gate-up tile j writes the a columns [64 j, 64 j + 64), which are
  // k-block j of the down GEMM.
  const int tiles_g = (int)((2 * I + kBM - 1) / kBM), tiles_d = (int)((d + kBM - 1) / kBM);
  const int KBg = (int)(d / kBK + pl.KS - 1) / pl.KS, KBd = (int)(I / kBK + pl.KS - 1) / pl.KS;
  const int ctas = (int)std::min<int64_t>(
      std::min<int64_t>(dev.sm_count, kTcMaxCtas),
      std::min((int64_t)tiles_g * KBg, (int64_t)tiles_d * KBd));
  // Whole waves of gate-up tiles run data-parallel (finished two thirds into
  // the phase on the 8B-shaped layer); the stream-K rest is kept at half a
  // wave or more, so that its tiles have few contributors.
  const int waves = tiles_g / ctas, rest = tiles_g % ctas;
  const int dp = 2 * rest >= ctas || rest == 0 ? waves : std::max(0, waves - 1);
  // Down part 1: the stages whose k-blocks all come from the stream-K tiles
  // (tiles dp * ctas and up), which every CTA works on first.
  const int S1 = std::min(KBd, (dp * ctas + pl.KS - 1) / pl.KS);
  p.sg = layer_sched(tiles_g, KBg, ctas, dp);
  p.sd1 = layer_sched(tiles_d, KBd - S1, ctas, 0);
  p.sd2 = layer_sched(tiles_d, S1, ctas, 0);
  p.S1 = S1;
  p.x = (const __nv_bfloat16*)x;
  p.gamma = (const __nv_bfloat16*)gamma;
  p.residual = (const __nv_bfloat16*)residual;
  p.b_hl = (__nv_bfloat16*)ws.b_hl;
  p.a = (__nv_bfloat16*)ws.a;
  p.out = out;
  p.out_bf16 = (__nv_bfloat16*)out_bf16;
  p.rinv = ws.rinv;
  p.partials = ws.partials;
  p.counters = ws.counters;
  p.ncounters = ws.ncounters;
  p.ticket = ws.ticket;
  p.inited = ws.inited;
  p.done = ws.done;
  p.gu_done = ws.gu_done;
  p.a_ready = ws.a_ready;
  p.hl_done = ws.hl_done;
  p.status = ws.status;
  p.wait_ns = wait_timeout_ns();
  p.eps = eps;
  p.M = (int)M;
  p.d = (int)d;
  p.I = (int)I;
  p.T = T;
  p.Mt = pl.Mt;
  p.Nd = pl.Nd;
  p.Cg = pl.Cg;
  p.Cd = pl.Cd;
  p.KS = pl.KS;
  p.KBg = (int)(d / kBK);
  p.KBd = (int)(I / kBK);
  p.stages = pl.stages;
  p.stage_bytes = pl.stage_bytes;
  p.bufcols = pl.bufcols;
  p.tmem_cols = pl.tmem_cols;
  p.n_init = std::min(ctas, kLayerMaxInit);
  p.n_build = std::min(ctas, kLayerMaxBuild);
  p.drop_last = fault_injection();

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(kLayerThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, tc_layer, p);
  if (e == cudaSuccess) note_launches(1);
  return e;
}

}  // namespace fmlp
