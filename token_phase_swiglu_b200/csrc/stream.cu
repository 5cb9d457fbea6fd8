// Bulk-copy pipelined weight-streaming kernels for decode-sized token counts.
//
// Gate-up (steps a1-a4) and down projection (a5-a6) of the MLP block in
// "FastTPS: An Optimized Method for LLM Token Phase for AI Accelerators"
// (xllm-io review), section 三 Eq(1) and Figure 4, for up to 4 token rows per
// pass.  At these sizes the block is a matrix-vector product whose time is
// the time to stream the weights from HBM once, so the kernels are built to
// keep HBM busy:
//   * one CTA per SM; the elected lane of warp 0 streams the CTA's
//     contiguous share of weight rows into a ring of shared-memory stages
//     with the TMA engine (cp.async.bulk, completion counted on one mbarrier
//     per stage).  A stage is a group of whole rows fetched with one or two
//     large copies (up to 64 KB): on B200 a bulk-copy ring is limited by the
//     number of copies per second far more than by the bytes in flight, so
//     copies are made as large as the rows allow;
//   * eight consumer warps share every stage: warp w owns gate/up pair w & 3
//     (or W_down row w & 3) of the group and column half w >> 2, dots it with
//     the activations held in shared memory, leaves its sums in shared memory
//     and arrives on the stage's "empty" mbarrier; the halves are combined
//     once, after the phase;
//   * fused_decode runs both steps in one launch, the "Fusion MLP" of the
//     pages.  CTA b owns a slice of the intermediate dimension: it streams the
//     gate/up rows of its pairs, keeps its slice of a (rounded to bf16) in
//     shared memory, then streams the matching column slice of W_down (2-D
//     TMA tiles of 256 rows) and adds its partial down projection straight
//     into out (red.global.add), which the first CTAs to arrive have set to
//     the residual (or zero).  No CTA waits for another CTA's results, and
//     `a` never travels through global memory;
//   * launches use programmatic dependent launch: a kernel's producer starts
//     streaming weights before the previous kernel on the stream has
//     finished; only the consumers wait for its results.
// Every wait is bounded (global-timer deadline); on expiry the CTA sets the
// timeout bit of the workspace status word, lets its in-flight copies land
// and exits.
#include "common.cuh"
#include "internal.h"
#include "ring.cuh"
#include "tmap.h"

#include <algorithm>
#include <cstring>
#include <mutex>
#include <set>

namespace fmlp {
namespace {

constexpr int kGroup = 4;                         // pairs (gate-up) or rows (down) per group
constexpr int kConsumers = 2 * kGroup;            // consumer warps: item w & 3, column half w >> 2
constexpr int kThreads = (kConsumers + 1) * 32;   // warp 0 produces
constexpr int64_t kMaxStageBytes = 64 * 1024;
constexpr int kGateRows = 2 * kGroup;             // rows per gate-up stage (4 gate + 4 up)
constexpr int kDownRows = kGroup;                 // rows per down stage
constexpr int kBarStage = 1;                      // named barrier: consumer-only sync


// bf16 pair (low half = element 2j, high half = element 2j+1) as two f32 lanes
__device__ __forceinline__ uint64_t bf2(uint32_t w) { return pk2(bf16lo(w), bf16hi(w)); }

// acc += w . s over 8 elements (w: 8 bf16; s: 8 f32), as 4 packed FMAs
__device__ __forceinline__ uint64_t dot8(const uint4& w, const float4& s0, const float4& s1,
                                         uint64_t acc) {
  acc = ffma2(bf2(w.x), pk2(s0.x, s0.y), acc);
  acc = ffma2(bf2(w.y), pk2(s0.z, s0.w), acc);
  acc = ffma2(bf2(w.z), pk2(s1.x, s1.y), acc);
  acc = ffma2(bf2(w.w), pk2(s1.z, s1.w), acc);
  return acc;
}

// acc += w . v over 8 elements (both bf16)
__device__ __forceinline__ uint64_t dot8bf(const uint4& w, const uint4& v, uint64_t acc) {
  acc = ffma2(bf2(w.x), bf2(v.x), acc);
  acc = ffma2(bf2(w.y), bf2(v.y), acc);
  acc = ffma2(bf2(w.z), bf2(v.z), acc);
  acc = ffma2(bf2(w.w), bf2(v.w), acc);
  return acc;
}



// ---------------------------------------------------------------------------
// Gate-up phase.  A group is 4 consecutive pairs (inside one T-tile, T % 8 ==
// 0): 4 gate rows and the 4 matching up rows, each run contiguous in the
// packed matrix.  Stage layout: rows 0-3 gate, rows 4-7 up, kc bf16 per row.
// ---------------------------------------------------------------------------
struct GateUpGeom {
  const __nv_bfloat16* P;
  int T, d, I;
  int kc, nchunks;
};

__device__ bool produce_gateup(Producer& pr, const GateUpGeom& g, int g0, int n_groups) {
  for (int j = 0; j < n_groups; ++j) {
    const __nv_bfloat16* pg = g.P + gate_row((g0 + j) * kGroup, g.T) * g.d;
    const __nv_bfloat16* pu = pg + (int64_t)g.T * g.d;
    for (int ch = 0; ch < g.nchunks; ++ch) {
      if (!pr.acquire()) return false;
      const int slot = pr.k % pr.ring.stages;
      const int k0 = ch * g.kc;
      const int len = min(g.kc, g.d - k0);
      uint8_t* buf = pr.ring.buf(slot);
      uint64_t* bar = &pr.ring.full[slot];
      mbar_arrive_expect_tx(bar, (uint32_t)(kGateRows * len * 2));
      if (g.nchunks == 1) {
        // 4 whole gate rows, then the 4 whole up rows: two contiguous runs
        const uint32_t run = (uint32_t)(kGroup * g.d * 2);
        bulk_copy_g2s(buf, pg, run, bar, pr.pol);
        bulk_copy_g2s(buf + run, pu, run, bar, pr.pol);
      } else {
        for (int r = 0; r < kGateRows; ++r) {
          const __nv_bfloat16* row =
              r < kGroup ? pg + (int64_t)r * g.d : pu + (int64_t)(r - kGroup) * g.d;
          bulk_copy_g2s(buf + (size_t)r * g.kc * 2, row + k0, (uint32_t)len * 2u, bar, pr.pol);
        }
      }
      ++pr.k;
    }
  }
  return true;
}

// gamma (weights: ready before the previous kernel ends) as f32 in row 0 of
// s, in the layout stage_x_gamma uses; consumer threads, before the
// dependency wait.  Each thread touches only the vectors it handles later.
__device__ void stage_gamma(const __nv_bfloat16* gamma, int d, float* s) {
  const int ct = threadIdx.x - 32;
  for (int v = ct; v < d / 8; v += kConsumers * 32) {
    const uint4 gv = ld_keep(gamma + (int64_t)v * 8);
    float4* dst = reinterpret_cast<float4*>(s);
    dst[v] = make_float4(bf16lo(gv.x), bf16hi(gv.x), bf16lo(gv.y), bf16hi(gv.y));
    dst[d / 8 + v] = make_float4(bf16lo(gv.z), bf16hi(gv.z), bf16lo(gv.w), bf16hi(gv.w));
  }
}

// s = x * gamma (exact in f32) for the CTA's token rows, and r = 1/sqrt(mean x^2 + eps).
// Row m of s holds d/8 float4 of columns 8v..8v+3, then d/8 float4 of 8v+4..8v+7.
// If `gamma` is null, row 0 of s already holds gamma (stage_gamma).
template <int MT>
__device__ void stage_x_gamma(const __nv_bfloat16* x, const __nv_bfloat16* gamma, float eps,
                              int d, int m0, int mt, float* s, float (*red)[MT], float* rinv) {
  const int lane = threadIdx.x & 31, c = (threadIdx.x >> 5) - 1, ct = threadIdx.x - 32;
  float ss[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) ss[m] = 0.f;
  for (int v = ct; v < d / 8; v += kConsumers * 32) {
    float gf[8];
    if (gamma) {
      const uint4 gv = ld_keep(gamma + (int64_t)v * 8);
      gf[0] = bf16lo(gv.x); gf[1] = bf16hi(gv.x); gf[2] = bf16lo(gv.y); gf[3] = bf16hi(gv.y);
      gf[4] = bf16lo(gv.z); gf[5] = bf16hi(gv.z); gf[6] = bf16lo(gv.w); gf[7] = bf16hi(gv.w);
    } else {
      const float4 g0 = reinterpret_cast<const float4*>(s)[v];
      const float4 g1 = reinterpret_cast<const float4*>(s)[d / 8 + v];
      gf[0] = g0.x; gf[1] = g0.y; gf[2] = g0.z; gf[3] = g0.w;
      gf[4] = g1.x; gf[5] = g1.y; gf[6] = g1.z; gf[7] = g1.w;
    }
    uint4 xv[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {  // all loads first: one L2 round trip
      xv[m] = make_uint4(0, 0, 0, 0);
      if (m < mt) xv[m] = ld_keep(x + (int64_t)(m0 + m) * d + (int64_t)v * 8);
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float xf[8] = {bf16lo(xv[m].x), bf16hi(xv[m].x), bf16lo(xv[m].y), bf16hi(xv[m].y),
                           bf16lo(xv[m].z), bf16hi(xv[m].z), bf16lo(xv[m].w), bf16hi(xv[m].w)};
#pragma unroll
      for (int e = 0; e < 8; ++e) ss[m] = fmaf(xf[e], xf[e], ss[m]);
      // two planes of float4 (columns 8v..8v+3, then 8v+4..8v+7) so that lanes
      // reading consecutive vectors touch consecutive 16-byte words
      float4* dst = reinterpret_cast<float4*>(s + (int64_t)m * d);
      dst[v] = make_float4(xf[0] * gf[0], xf[1] * gf[1], xf[2] * gf[2], xf[3] * gf[3]);
      dst[d / 8 + v] = make_float4(xf[4] * gf[4], xf[5] * gf[5], xf[6] * gf[6], xf[7] * gf[7]);
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const float t = warp_sum(ss[m]);
    if (lane == 0) red[c][m] = t;
  }
  named_barrier_sync(kBarStage, kConsumers * 32);
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) t += red[w][m];
    rinv[m] = 1.0f / sqrtf(t / (float)d + eps);
  }
}

// Gate-up consumer warps: pair w & 3 of every group, column half w >> 2, dot
// each stage against x * gamma (s: two planes of float4 per token row, see
// stage_x_gamma).  Each warp leaves its warp-reduced gate and up sums of every
// group in `part` (shared memory, [group][pair][half][gate, up][MT]) instead
// of combining the column halves group by group, so that the warps meet at no
// barrier during the phase and can run up to a ring's depth apart (the
// consumers process a stage only slightly faster than HBM delivers one, so a
// barrier per group cost bandwidth).  finish_slice (fused_decode) or
// finish_a_global (gateup_stream) combines them.
template <int MT>
__device__ bool consume_gateup_parts(Consumer& cs, const GateUpGeom& g, int n_groups,
                                     const float* s, float* part) {
  const int c = (threadIdx.x >> 5) - 1, lane = cs.lane;
  const int pr = c & (kGroup - 1), half = c / kGroup;
  for (int j = 0; j < n_groups; ++j) {
    uint64_t ag[2][MT], au[2][MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) ag[0][m] = ag[1][m] = au[0][m] = au[1][m] = 0ull;
    for (int ch = 0; ch < g.nchunks; ++ch) {
      const uint8_t* buf = cs.wait_full();
      if (!buf) return false;
      const int k0 = ch * g.kc;
      const int nv = min(g.kc, g.d - k0) / 8;
      const uint8_t* bg = buf + (size_t)pr * g.kc * 2;
      const uint8_t* bu = buf + (size_t)(kGroup + pr) * g.kc * 2;
      const int kv0 = k0 / 8;
      for (int v = lane + 32 * half; v < nv; v += 128) {  // vectors v and v + 64
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int vv = v + 64 * h;
          if (h == 0 || vv < nv) {
            const uint4 wg = lds128(bg + 16 * vv);
            const uint4 wu = lds128(bu + 16 * vv);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              const float4* sp = reinterpret_cast<const float4*>(s + (int64_t)m * g.d) + kv0 + vv;
              const float4 s0 = sp[0], s1 = sp[g.d / 8];
              ag[h][m] = dot8(wg, s0, s1, ag[h][m]);
              au[h][m] = dot8(wu, s0, s1, au[h][m]);
            }
          }
        }
      }
      cs.release();
    }
    float* dst = part + ((j * kGroup + pr) * 2 + half) * 2 * MT;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float gs = warp_sum(hsum2(ag[0][m]) + hsum2(ag[1][m]));
      const float us = warp_sum(hsum2(au[0][m]) + hsum2(au[1][m]));
      if (lane == 0) {
        dst[m] = gs;
        dst[MT + m] = us;
      }
    }
  }
  return true;
}

// a = bf16(SiLU(r g) * r u) for the CTA's w = 4 * n_groups pairs, from the
// halves' sums in `part`, into slice[m * ld + i] (as f32; rows >= mt zero).
// All consumer threads, after a barrier that follows consume_gateup_parts.
template <int MT>
__device__ void finish_slice(const float* part, int n_groups, const float* rinv, int mt,
                             float* slice, int ld) {
  const int ct = threadIdx.x - 32;
  for (int i = ct; i < n_groups * kGroup; i += kConsumers * 32) {
    const float* q = part + i * 4 * MT;  // [half 0: g, u][half 1: g, u]
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float gt = q[m] + q[2 * MT + m], ut = q[MT + m] + q[3 * MT + m];
      const __nv_bfloat16 av = __float2bfloat16_rn(silu_mul(gt * rinv[m], ut * rinv[m]));
      slice[m * ld + i] = m < mt ? __bfloat162float(av) : 0.f;
    }
  }
}

// gateup_stream: a[m0 + m, 4 g0 + i] = bf16(SiLU(r g) * r u) for the CTA's
// 4 * n_groups pairs from the halves' sums in `part` (one coalesced pass).
template <int MT>
__device__ void finish_a_global(const float* part, int n_groups, const float* rinv, int mt,
                                __nv_bfloat16* a, int64_t I, int m0, int g0) {
  const int ct = threadIdx.x - 32;
  for (int i = ct; i < n_groups * kGroup; i += kConsumers * 32) {
    const float* q = part + i * 4 * MT;  // [half 0: g, u][half 1: g, u]
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m >= mt) continue;
      const float gt = q[m] + q[2 * MT + m], ut = q[MT + m] + q[3 * MT + m];
      a[(int64_t)(m0 + m) * I + (int64_t)g0 * kGroup + i] =
          __float2bfloat16_rn(silu_mul(gt * rinv[m], ut * rinv[m]));
    }
  }
}

// Bytes of the halves' sums that gateup_stream keeps per CTA (consume_gateup_parts).
__host__ __device__ constexpr size_t gateup_part_bytes(int max_groups, int mt) {
  return align128((size_t)max_groups * kGroup * 4 * mt * sizeof(float));
}

// ---------------------------------------------------------------------------
// Down phase.  A group is 4 consecutive W_down rows (one contiguous run);
// a [MT x I] (bf16) sits in shared memory.  Stage layout: rows 0-3, kc bf16 per row.
// ---------------------------------------------------------------------------
struct DownGeom {
  const __nv_bfloat16* Wd;
  int d, I;
  int kc, nchunks;
};

__device__ bool produce_down(Producer& pr, const DownGeom& g, int g0, int n_groups) {
  for (int j = 0; j < n_groups; ++j) {
    const __nv_bfloat16* src = g.Wd + (int64_t)(g0 + j) * kDownRows * g.I;
    for (int ch = 0; ch < g.nchunks; ++ch) {
      if (!pr.acquire()) return false;
      const int slot = pr.k % pr.ring.stages;
      const int k0 = ch * g.kc;
      const int len = min(g.kc, g.I - k0);
      uint8_t* buf = pr.ring.buf(slot);
      uint64_t* bar = &pr.ring.full[slot];
      mbar_arrive_expect_tx(bar, (uint32_t)(kDownRows * len * 2));
      if (g.nchunks == 1) {
        bulk_copy_g2s(buf, src, (uint32_t)(kDownRows * g.I * 2), bar, pr.pol);
      } else {
        for (int r = 0; r < kDownRows; ++r)
          bulk_copy_g2s(buf + (size_t)r * g.kc * 2, src + (int64_t)r * g.I + k0,
                        (uint32_t)len * 2u, bar, pr.pol);
      }
      ++pr.k;
    }
  }
  return true;
}

// a [MT x I] (bf16) from global into shared memory (rows >= mt zero-filled).
template <int MT>
__device__ void stage_a(const __nv_bfloat16* a, int I, int m0, int mt, uint8_t* act) {
  const int ct = threadIdx.x - 32;
#pragma unroll
  for (int m = 0; m < MT; ++m)
    for (int v = ct; v < I / 8; v += kConsumers * 32) {
      uint4 av = make_uint4(0, 0, 0, 0);
      if (m < mt) av = ld_keep(a + (int64_t)(m0 + m) * I + (int64_t)v * 8);
      *reinterpret_cast<uint4*>(act + ((size_t)m * I + (size_t)v * 8) * 2) = av;
    }
  named_barrier_sync(kBarStage, kConsumers * 32);
}

// Consumer warps: row w & 3 of every group, column half w >> 2.  Each warp
// leaves its warp-reduced sums in `part` ([group][row][half][MT], shared
// memory); finish_down_out combines the halves after the phase, so the warps
// meet at no barrier per group.
template <int MT>
__device__ bool consume_down_parts(Consumer& cs, const DownGeom& g, int n_groups,
                                   const uint8_t* act, float* part) {
  const int c = (threadIdx.x >> 5) - 1, lane = cs.lane;
  const int row = c & (kGroup - 1), half = c / kGroup;
  for (int j = 0; j < n_groups; ++j) {
    uint64_t acc[2][MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[0][m] = acc[1][m] = 0ull;
    for (int ch = 0; ch < g.nchunks; ++ch) {
      const uint8_t* buf = cs.wait_full();
      if (!buf) return false;
      const int k0 = ch * g.kc;
      const int nv = min(g.kc, g.I - k0) / 8;
      const uint8_t* bw = buf + (size_t)row * g.kc * 2;
      const uint8_t* ak = act + (size_t)k0 * 2;
      for (int v = lane + 32 * half; v < nv; v += 128) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int vv = v + 64 * h;
          if (h == 0 || vv < nv) {
            const uint4 w = lds128(bw + 16 * vv);
#pragma unroll
            for (int m = 0; m < MT; ++m)
              acc[h][m] = dot8bf(w, lds128(ak + ((size_t)m * g.I + 8 * vv) * 2), acc[h][m]);
          }
        }
      }
      cs.release();
    }
    float* dst = part + ((j * kGroup + row) * 2 + half) * MT;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float t = warp_sum(hsum2(acc[0][m]) + hsum2(acc[1][m]));
      if (lane == 0) dst[m] = t;
    }
  }
  return true;
}

// out[m0 + m, 4 g0 + i] = the halves' sums (+ residual), one coalesced pass.
template <int MT>
__device__ void finish_down_out(const float* part, int n_groups, const __nv_bfloat16* residual,
                                float* out, int64_t d, int m0, int mt, int g0) {
  const int ct = threadIdx.x - 32;
  for (int i = ct; i < n_groups * kDownRows; i += kConsumers * 32) {
    const float* q = part + i * 2 * MT;  // [half 0][half 1]
    const int64_t n = (int64_t)g0 * kDownRows + i;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m >= mt) continue;
      float o = q[m] + q[MT + m];
      if (residual) o += __bfloat162float(residual[(int64_t)(m0 + m) * d + n]);
      out[(int64_t)(m0 + m) * d + n] = o;
    }
  }
}

__host__ __device__ constexpr size_t down_part_bytes(int max_groups, int mt) {
  return align128((size_t)max_groups * kDownRows * 2 * mt * sizeof(float));
}


// ---------------------------------------------------------------------------
// Kernels
// ---------------------------------------------------------------------------
struct StreamParams {
  const __nv_bfloat16* x;
  const __nv_bfloat16* gamma;
  const __nv_bfloat16* residual;
  __nv_bfloat16* a;      // intermediate (output of the gate-up phase)
  float* out;
  Control ctl;
  GateUpGeom gu;
  DownGeom dn;
  float eps;
  int M;
  int stages, stage_bytes;
};

// act_main: bytes of the activations at the start of the dynamic shared
// memory (x * gamma in f32, or a in bf16); the halves' sums follow them, and
// the ring starts at act_bytes.
template <int MT, bool GATE, bool DOWN>
__device__ __forceinline__ void stream_body(const StreamParams& p, size_t act_main,
                                            size_t act_bytes) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ float red[kConsumers][MT];
  __shared__ CtaState st;

  Ring ring;
  ring.full = reinterpret_cast<uint64_t*>(smem);
  ring.empty = ring.full + kMaxStages;
  uint8_t* act = smem + kHeader;
  float* part = reinterpret_cast<float*>(act + act_main);
  ring.stage0 = smem + kHeader + act_bytes;
  ring.stages = p.stages;
  ring.stage_bytes = p.stage_bytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * MT;
  const int mt = min(MT, p.M - m0);
  int ga0 = 0, nga = 0, gd0 = 0, ngd = 0;
  if (GATE) split_groups(p.gu.I / kGroup, blockIdx.x, gridDim.x, false, ga0, nga);
  if (DOWN) split_groups(p.dn.d / kDownRows, blockIdx.x, gridDim.x, false, gd0, ngd);

  if (threadIdx.x == 0) init_ring(ring, st, kConsumers);
  __syncthreads();
  grid_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      Producer pr{ring, &st, p.ctl, evict_first_policy(),
                  nga * p.gu.nchunks + ngd * p.dn.nchunks};
      bool ok = true;
      if (GATE) ok = produce_gateup(pr, p.gu, ga0, nga);
      if (DOWN && ok) produce_down(pr, p.dn, gd0, ngd);
      st.issued = pr.k;
    }
    __syncwarp();
  } else {
    if (GATE) stage_gamma(p.gamma, p.gu.d, reinterpret_cast<float*>(act));
    grid_dependency_wait();  // inputs may be written by the previous kernel
    Consumer cs{ring, &st, p.ctl, 0, lane};
    // every warp's sums of every group go to `part`; after one barrier (which
    // also agrees on failure) the halves are combined and written out
    if (GATE) {
      float rinv[MT];
      stage_x_gamma<MT>(p.x, nullptr, p.eps, p.gu.d, m0, mt, reinterpret_cast<float*>(act),
                        red, rinv);
      const bool ok = consume_gateup_parts<MT>(cs, p.gu, nga, reinterpret_cast<const float*>(act),
                                               part);
      if (!consumer_barrier_any<kConsumers * 32>(kBarStage, !ok))
        finish_a_global<MT>(part, nga, rinv, mt, p.a, p.gu.I, m0, ga0);
    }
    if (DOWN) {
      stage_a<MT>(p.a, p.dn.I, m0, mt, act);
      const bool ok = consume_down_parts<MT>(cs, p.dn, ngd, act, part);
      if (!consumer_barrier_any<kConsumers * 32>(kBarStage, !ok))
        finish_down_out<MT>(part, ngd, p.residual, p.out, p.dn.d, m0, mt, gd0);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && st.abort) drain_ring(ring, st.issued);
}

template <int MT>
__global__ void __launch_bounds__(kThreads, 1) gateup_stream(const StreamParams p) {
  const size_t act_main = align128((size_t)MT * p.gu.d * sizeof(float));
  const int max_groups = (p.gu.I / kGroup + gridDim.x - 1) / gridDim.x;
  stream_body<MT, true, false>(p, act_main, act_main + gateup_part_bytes(max_groups, MT));
}

template <int MT>
__global__ void __launch_bounds__(kThreads, 1) down_stream(const StreamParams p) {
  const size_t act_main = align128((size_t)MT * p.dn.I * 2);
  const int max_groups = (p.dn.d / kDownRows + gridDim.x - 1) / gridDim.x;
  stream_body<MT, false, true>(p, act_main, act_main + down_part_bytes(max_groups, MT));
}

// ---------------------------------------------------------------------------
// fused_decode: both steps in one launch, split over the intermediate dimension.
// ---------------------------------------------------------------------------
struct FusedParams {
  CUtensorMap wd_map;  // W_down [d x I] bf16, boxes of rows_d x swbox, no swizzle
  const __nv_bfloat16* x;
  const __nv_bfloat16* gamma;
  const __nv_bfloat16* residual;
  float* out;          // [M x d] f32: set to the residual (or 0), then CTAs add into it
  __nv_bfloat16* out_bf16;  // [M x d] or null: out rounded to bf16 by the last CTA to finish
  uint32_t* ticket;    // arrival order of the CTAs (zero between calls)
  uint32_t* inited;    // initialising CTAs whose share of out is set (zero between calls)
  uint32_t* done;      // CTAs finished (zero between calls)
  int n_init;          // CTAs that initialise out: the first n_init to arrive
  Control ctl;
  GateUpGeom gu;
  float eps;
  int M, d, I;
  int units;           // I / 8: slices are cut at multiples of 8 pairs (16-byte columns)
  int swbox;           // W_down slice box width (>= every CTA's slice, odd multiple of 8)
  int rows_d;          // W_down rows per stage (256, or 128 for wide slices; fewer if
                       // the ring would have under three slots)
  int nrb;             // row blocks = ceil(d / rows_d)
  int stages, stage_bytes;
};

__device__ void produce_down_slice(Producer& pr, const FusedParams& p, int i0) {
  const uint32_t bytes = (uint32_t)(p.swbox * p.rows_d * 2);
  for (int rb = 0; rb < p.nrb; ++rb) {
    if (!pr.acquire()) return;
    const int slot = pr.k % pr.ring.stages;
    uint64_t* bar = &pr.ring.full[slot];
    mbar_arrive_expect_tx(bar, bytes);  // a box always lands whole (zeros past the edges)
    tma_load_2d(pr.ring.buf(slot), &p.wd_map, i0, rb * p.rows_d, bar, pr.pol);
    ++pr.k;
  }
}

// Each consumer thread owns one W_down row of the stage (two threads per row,
// column halves, for slices wider than 128 columns) and adds its partial dot
// products with the CTA's slice of a into out.
template <int MT>
__device__ bool consume_down_slice(Consumer& cs, const FusedParams& p, const float* slice,
                                   int w, int mt) {
  const int ct = threadIdx.x - 32;
  const bool halves = p.swbox > 128;
  const int r = halves ? (ct & 127) : ct;
  int c0 = 0, c1 = w;
  if (halves) {
    const int hw = ((w / 2) + 7) / 8 * 8;
    if (ct < 128) c1 = hw; else c0 = hw;
  }
  for (int rb = 0; rb < p.nrb; ++rb) {
    const uint8_t* buf = cs.wait_full();
    if (!buf) return false;
    const int n = rb * p.rows_d + r;
    if (r < p.rows_d && n < p.d) {
      const uint8_t* row = buf + (size_t)r * p.swbox * 2;
      float acc[2][MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[0][m] = acc[1][m] = 0.f;
      int c = c0;
      for (; c + 8 < c1; c += 16) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint4 wv = lds128(row + 2 * (c + 8 * h));
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const float4* ap = reinterpret_cast<const float4*>(slice + m * p.swbox + c + 8 * h);
            const float4 a0 = ap[0], a1 = ap[1];
            float t = acc[h][m];
            t = fmaf(bf16lo(wv.x), a0.x, t); t = fmaf(bf16hi(wv.x), a0.y, t);
            t = fmaf(bf16lo(wv.y), a0.z, t); t = fmaf(bf16hi(wv.y), a0.w, t);
            t = fmaf(bf16lo(wv.z), a1.x, t); t = fmaf(bf16hi(wv.z), a1.y, t);
            t = fmaf(bf16lo(wv.w), a1.z, t); t = fmaf(bf16hi(wv.w), a1.w, t);
            acc[h][m] = t;
          }
        }
      }
      if (c < c1) {
        const uint4 wv = lds128(row + 2 * c);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const float4* ap = reinterpret_cast<const float4*>(slice + m * p.swbox + c);
          const float4 a0 = ap[0], a1 = ap[1];
          float t = acc[0][m];
          t = fmaf(bf16lo(wv.x), a0.x, t); t = fmaf(bf16hi(wv.x), a0.y, t);
          t = fmaf(bf16lo(wv.y), a0.z, t); t = fmaf(bf16hi(wv.y), a0.w, t);
          t = fmaf(bf16lo(wv.z), a1.x, t); t = fmaf(bf16hi(wv.z), a1.y, t);
          t = fmaf(bf16lo(wv.w), a1.z, t); t = fmaf(bf16hi(wv.w), a1.w, t);
          acc[0][m] = t;
        }
      }
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (m < mt) atomicAdd(p.out + (int64_t)m * p.d + n, acc[0][m] + acc[1][m]);
    }
    cs.release();
  }
  return true;
}

__device__ __forceinline__ void st_release_cta(int* p, int v) {
  asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_cta(const int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}

// Wait (one thread) for a shared-memory flag that another warp of the CTA
// sets to nonzero; returns it, or 0 after limit_ns or when *abort is set.
__device__ int wait_flag_cta(const int* flag, uint64_t limit_ns, volatile int* abort) {
  int v = ld_acquire_cta(flag);
  if (v) return v;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    __nanosleep(32);
    if ((v = ld_acquire_cta(flag)) != 0) return v;
    if (*abort) return 0;
    if (globaltimer_ns() - t0 > limit_ns) return 0;
  }
}

// Wait (one thread) until the counter at `ctr` reaches `target`, with
// acquire semantics, for at most limit_ns; false if it gave up.
__device__ bool wait_counter(const uint32_t* ctr, uint32_t target, uint64_t limit_ns,
                             volatile int* abort) {
  if (ld_acquire_gpu(ctr) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    __nanosleep(32);
    if (ld_acquire_gpu(ctr) >= target) return true;
    if (abort && *abort) return false;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// The block's threads round n f32 values (n % 4 == 0, read from L2, where
// other blocks' adds landed) to bf16, round to nearest even.
__device__ void out_to_bf16_block(const float* src, __nv_bfloat16* dst, int64_t n) {
  for (int64_t i = threadIdx.x; i < n / 4; i += blockDim.x) {
    const float4 v = __ldcg(reinterpret_cast<const float4*>(src) + i);
    uint2 w;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w.x) : "f"(v.y), "f"(v.x));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w.y) : "f"(v.w), "f"(v.z));
    reinterpret_cast<uint2*>(dst)[i] = w;
  }
}

// Warp 0, lanes 1-31.  The first n_init CTAs to arrive (an atomic ticket,
// taken once the previous kernel on the stream is done) set one share each
// of out (float4 granules) to the residual or zero and count it in inited.
// The consumers of every CTA wait for that count before adding into out; as
// the initialising CTAs are by construction already running, nobody waits
// on a CTA that has not been scheduled, so no co-residency is assumed.
__device__ void init_out_share(const FusedParams& p, int mt, int lane) {
  grid_dependency_wait();  // out, the residual and the counters belong to this call now
  uint32_t t = 0;
  if (lane == 1) t = atomicAdd(p.ticket, 1u);
  t = __shfl_sync(0xfffffffeu, t, 1);
  if (t >= (uint32_t)p.n_init) return;
  const int64_t n4 = (int64_t)mt * p.d / 4;
  const int64_t q0 = n4 * t / p.n_init, q1 = n4 * (t + 1) / p.n_init;
  for (int64_t i = q0 + lane - 1; i < q1; i += 31) {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p.residual) {
      const uint2 r = __ldg(reinterpret_cast<const uint2*>(p.residual) + i);
      v = make_float4(bf16lo(r.x), bf16hi(r.x), bf16lo(r.y), bf16hi(r.y));
    }
    reinterpret_cast<float4*>(p.out)[i] = v;
  }
  __threadfence();
  __syncwarp(0xfffffffeu);
  if (lane == 1) atomicAdd(p.inited, 1u);
}

template <int MT>
__global__ void __launch_bounds__(kThreads, 1) fused_decode(const __grid_constant__ FusedParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ float red[kConsumers][MT];
  __shared__ CtaState st;

  Ring ring;
  ring.full = reinterpret_cast<uint64_t*>(smem);
  ring.empty = ring.full + kMaxStages;
  float* s = reinterpret_cast<float*>(smem + kHeader);                          // [MT][d]
  float* slice = reinterpret_cast<float*>(smem + kHeader + align128((size_t)MT * p.d * 4));
  float* part = slice + align128((size_t)MT * p.swbox * 4) / 4;  // [swbox / 4][kGroup][2][2][MT]
  ring.stage0 = smem + kHeader + align128((size_t)MT * p.d * 4) +
                align128((size_t)MT * p.swbox * 4) + align128((size_t)MT * p.swbox * 16);
  ring.stages = p.stages;
  ring.stage_bytes = p.stage_bytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = min(MT, p.M);
  int u0, nu;
  split_groups(p.units, blockIdx.x, gridDim.x, false, u0, nu);
  const int i0 = u0 * 8, w = nu * 8;
  const int g0 = i0 / kGroup, ng = w / kGroup;

  if (threadIdx.x == 0) init_ring(ring, st, kConsumers);
  __syncthreads();
  grid_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      Producer pr{ring, &st, p.ctl, evict_first_policy(), ng * p.gu.nchunks + p.nrb};
      if (produce_gateup(pr, p.gu, g0, ng)) produce_down_slice(pr, p, i0);
      st.issued = pr.k;
    } else {
      init_out_share(p, mt, lane);
      // Lane 1 then waits for every share of out and tells the consumers
      // through shared memory, so that the L2 round trips of that wait stay
      // off their path between the two phases.
      if (lane == 1) {
        int r = 1;
        if (!wait_counter(p.inited, (uint32_t)p.n_init, p.ctl.wait_ns, &st.abort)) {
          if (!st.abort) flag_timeout(&st, p.ctl.status);
          r = -1;
        }
        st_release_cta(&st.out_ready, r);
      }
    }
    __syncwarp();
  } else {
    const int ct = threadIdx.x - 32;
    stage_gamma(p.gamma, p.d, s);  // weights: before the dependency wait
    grid_dependency_wait();        // x may be written by the previous kernel
    Consumer cs{ring, &st, p.ctl, 0, lane};
    float rinv[MT];
    stage_x_gamma<MT>(p.x, nullptr, p.eps, p.d, 0, mt, s, red, rinv);
    bool ok = consume_gateup_parts<MT>(cs, p.gu, ng, s, part);
    // All of out must be set before anyone adds into it.  The shares are
    // written at the start by CTAs already running, and lane 1 of warp 0 has
    // waited for them during the gate-up phase, so this normally reads its
    // flag in shared memory at once.
    if (ct == 0 && ok) {
      const int r = wait_flag_cta(&st.out_ready, p.ctl.wait_ns, &st.abort);
      if (r == 0) flag_timeout(&st, p.ctl.status);
      ok = r == 1;
    }
    // Every warp's sums are in `part` and out is ready, or someone gave up:
    // all consumer warps take the same decision.
    if (!consumer_barrier_any<kConsumers * 32>(kBarStage, !ok)) {
      finish_slice<MT>(part, ng, rinv, mt, slice, p.swbox);
      named_barrier_sync(kBarStage, kConsumers * 32);  // slice of a complete
      consume_down_slice<MT>(cs, p, slice, w, mt);
    }
    // with a bf16 output the last CTA to finish reads the sum: this thread's
    // adds into it are visible before its CTA counts itself finished
    if (p.out_bf16) __threadfence();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (st.abort) drain_ring(ring, st.issued);
    // this CTA's adds into out are visible before it counts itself finished
    if (p.out_bf16) __threadfence();
    // Every CTA has taken its ticket, finished any share of out it owned and
    // is past its wait on `inited`: the last one to get here leaves the
    // counters at zero for the next call (also after a timeout).
    const bool last = atomicAdd(p.done, 1u) == gridDim.x - 1;
    if (last) {
      atomicExch(p.ticket, 0u);
      atomicExch(p.inited, 0u);
      atomicExch(p.done, 0u);
    }
    st.last = last;
  }
  if (p.out_bf16) {
    // the last CTA rounds the finished sum to the bf16 output
    __syncthreads();
    if (st.last) {
      __threadfence();
      out_to_bf16_block(p.out, p.out_bf16, (int64_t)min(MT, p.M) * p.d);
    }
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

// Raise a kernel's dynamic shared-memory limit to the device maximum, once
// per (device, kernel).
template <typename Kernel>
cudaError_t allow_max_smem(Kernel kernel, const DeviceInfo& dev) {
  static std::mutex mu;
  static std::set<std::pair<int, const void*>> done;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(dev.device, (const void*)kernel);
  if (done.count(key)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       dev.max_smem_optin - 1024);
  if (e == cudaSuccess) done.insert(key);
  return e;
}

template <typename Kernel>
cudaError_t launch_pdl(Kernel kernel, dim3 grid, size_t smem, const DeviceInfo& dev,
                       cudaStream_t stream, const StreamParams& params) {
  cudaError_t e = allow_max_smem(kernel, dev);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kernel, params);
  if (e == cudaSuccess) note_launches(1);
  return e;
}

struct Chunking {
  int kc = 0, nchunks = 0, stage_bytes = 0;
};

// Whole rows per stage when `rows` rows of K elements fit in `target` bytes
// (one or two large copies), else equal column chunks (one copy per row).
Chunking chunk_rows(int64_t K, int rows, int64_t target) {
  Chunking c;
  const int64_t whole = rows * K * 2;
  c.nchunks = (int)((whole + target - 1) / target);
  c.kc = (int)((((K + c.nchunks - 1) / c.nchunks) + 7) / 8 * 8);
  c.nchunks = (int)((K + c.kc - 1) / c.kc);
  c.stage_bytes = (int)align128((size_t)rows * c.kc * 2);
  return c;
}

struct Plan {
  int mt = 0, stages = 0, stage_bytes = 0;
  Chunking gu, dn;
  size_t act = 0, smem = 0;
};

// Choose token rows per pass, chunking and ring depth.  Prefer (1) more token
// rows per pass (each pass streams the weights once), then (2) the largest
// stages (up to 64 KB) that still leave a ring of at least three stages.
Plan make_plan(int64_t M, int64_t d, int64_t I, bool gate, bool down, const DeviceInfo& dev) {
  const size_t budget = (size_t)dev.max_smem_optin - 1024;  // static smem + slack
  for (int min_stages = 3; min_stages >= 2; --min_stages)
    for (int mt = (int)std::min<int64_t>(M, 4); mt >= 1; --mt) {
      // activations plus the halves' sums of the CTA's groups (grid as launched)
      const int grid_g = (int)std::min<int64_t>(I / kGroup, dev.sm_count);
      const int grid_d = (int)std::min<int64_t>(d / kDownRows, dev.sm_count);
      size_t act = 0;
      if (gate)
        act = std::max(act, align128((size_t)mt * d * sizeof(float)) +
                                gateup_part_bytes((int)((I / kGroup + grid_g - 1) / grid_g), mt));
      if (down)
        act = std::max(act, align128((size_t)mt * I * 2) +
                                down_part_bytes((int)((d / kDownRows + grid_d - 1) / grid_d), mt));
      const size_t fixed = kHeader + act;
      if (fixed >= budget) continue;
      for (int64_t target = kMaxStageBytes; target >= 4096; target /= 2) {
        Plan pl;
        if (gate) pl.gu = chunk_rows(d, kGateRows, target);
        if (down) pl.dn = chunk_rows(I, kDownRows, target);
        pl.stage_bytes = std::max(pl.gu.stage_bytes, pl.dn.stage_bytes);
        const size_t fit = (budget - fixed) / pl.stage_bytes;
        if (fit < (size_t)min_stages) continue;
        pl.mt = mt;
        pl.act = act;
        pl.stages = (int)std::min<size_t>(kMaxStages, fit);
        pl.smem = fixed + (size_t)pl.stages * pl.stage_bytes;
        return pl;
      }
    }
  return Plan();  // mt == 0: does not fit
}

StreamParams make_params(const Plan& pl, const void* x, int64_t M, const void* gamma, float eps,
                         const void* P, int T, const void* W_down, int64_t d, int64_t I,
                         void* a, const void* residual, float* out, uint32_t* status) {
  StreamParams p = {};
  p.x = (const __nv_bfloat16*)x;
  p.gamma = (const __nv_bfloat16*)gamma;
  p.residual = (const __nv_bfloat16*)residual;
  p.a = (__nv_bfloat16*)a;
  p.out = out;
  p.ctl.status = status;
  p.ctl.wait_ns = wait_timeout_ns();
  p.ctl.drop_last = fault_injection();
  p.gu = GateUpGeom{(const __nv_bfloat16*)P, T, (int)d, (int)I, pl.gu.kc, pl.gu.nchunks};
  p.dn = DownGeom{(const __nv_bfloat16*)W_down, (int)d, (int)I, pl.dn.kc, pl.dn.nchunks};
  p.eps = eps;
  p.M = (int)M;
  p.stages = pl.stages;
  p.stage_bytes = pl.stage_bytes;
  return p;
}

#define FMLP_KERNEL_TAG(name)                                      \
  template <int MT>                                                \
  struct name##_tag {                                              \
    static constexpr auto fn = name<MT>;                           \
  };
FMLP_KERNEL_TAG(gateup_stream)
FMLP_KERNEL_TAG(down_stream)
#undef FMLP_KERNEL_TAG

template <template <int> class Tag>
cudaError_t launch_mt(int mt, dim3 grid, const Plan& pl, const DeviceInfo& dev,
                      cudaStream_t stream, const StreamParams& p) {
  switch (mt) {
    case 1: return launch_pdl(Tag<1>::fn, grid, pl.smem, dev, stream, p);
    case 2: return launch_pdl(Tag<2>::fn, grid, pl.smem, dev, stream, p);
    case 3: return launch_pdl(Tag<3>::fn, grid, pl.smem, dev, stream, p);
    default: return launch_pdl(Tag<4>::fn, grid, pl.smem, dev, stream, p);
  }
}

}  // namespace

cudaError_t launch_gateup_stream(const void* x, int64_t M, const void* gamma, float eps,
                                 const void* P, int T, int64_t d, int64_t I, void* a,
                                 uint32_t* status, const DeviceInfo& dev, cudaStream_t stream) {
  const Plan pl = make_plan(M, d, I, true, false, dev);
  if (pl.mt == 0) return cudaErrorInvalidConfiguration;
  const StreamParams p = make_params(pl, x, M, gamma, eps, P, T, nullptr, d, I, a, nullptr,
                                     nullptr, status);
  const dim3 grid((unsigned)std::min<int64_t>(I / kGroup, dev.sm_count),
                  (unsigned)((M + pl.mt - 1) / pl.mt));
  return launch_mt<gateup_stream_tag>(pl.mt, grid, pl, dev, stream, p);
}

cudaError_t launch_down_stream(const void* a, int64_t M, const void* W_down, int64_t d,
                               int64_t I, const void* residual, float* out, uint32_t* status,
                               const DeviceInfo& dev, cudaStream_t stream) {
  const Plan pl = make_plan(M, d, I, false, true, dev);
  if (pl.mt == 0) return cudaErrorInvalidConfiguration;
  const StreamParams p = make_params(pl, nullptr, M, nullptr, 0.f, nullptr, 0, W_down, d, I,
                                     const_cast<void*>(a), residual, out, status);
  const dim3 grid((unsigned)std::min<int64_t>(d / kDownRows, dev.sm_count),
                  (unsigned)((M + pl.mt - 1) / pl.mt));
  return launch_mt<down_stream_tag>(pl.mt, grid, pl, dev, stream, p);
}

namespace {

struct FusedPlan {
  int mt = 0, grid = 0, units = 0, swbox = 0, rows_d = 0, nrb = 0, stages = 0, stage_bytes = 0;
  Chunking gu;
  size_t smem = 0;
};

// One pass over the weights (all M <= 4 rows per CTA), a slice of at most
// 256 columns per CTA, and a ring of at least three stages.
FusedPlan make_fused_plan(int64_t M, int64_t d, int64_t I, const DeviceInfo& dev) {
  FusedPlan f;
  if (M < 1 || M > kFusedMaxM) return f;
  const size_t budget = (size_t)dev.max_smem_optin - 1024;
  f.units = (int)(I / 8);
  f.grid = std::min(f.units, dev.sm_count);
  const int max_units = (f.units + f.grid - 1) / f.grid;
  int sw_units = max_units | 1;  // odd count of 16-byte columns: conflict-free row reads
  f.swbox = 8 * sw_units;
  if (f.swbox > 256) return FusedPlan();
  const int full_rows = f.swbox <= 128 ? 256 : 128;
  const size_t down_stage = align128((size_t)f.swbox * full_rows * 2);
  // s (x * gamma), the slice of a, and the halves' gate/up sums
  const size_t act = align128((size_t)M * d * 4) + align128((size_t)M * f.swbox * 4) +
                     align128((size_t)M * f.swbox * 16);
  if (kHeader + act >= budget) return FusedPlan();
  for (int64_t target = kMaxStageBytes; target >= 4096; target /= 2) {
    const Chunking gu = chunk_rows(d, kGateRows, target);
    // W_down stages of full_rows rows, or, if the ring would then have under
    // three slots, of as many rows as a gate-up stage's bytes hold
    size_t slot = std::max<size_t>(gu.stage_bytes, down_stage);
    f.rows_d = full_rows;
    if ((budget - kHeader - act) / slot < 3) {
      slot = gu.stage_bytes;
      f.rows_d = std::min(full_rows, (int)(slot / (f.swbox * 2)) / 8 * 8);
      if (f.rows_d < 128) continue;  // too many small copies: leave it to the other paths
    }
    const size_t fit = (budget - kHeader - act) / slot;
    if (fit < 3) continue;
    f.nrb = (int)((d + f.rows_d - 1) / f.rows_d);
    f.gu = gu;
    f.mt = (int)M;
    f.stage_bytes = (int)slot;
    f.stages = (int)std::min<size_t>(kMaxStages, fit);
    f.smem = kHeader + act + (size_t)f.stages * slot;
    return f;
  }
  return FusedPlan();
}

template <int MT>
cudaError_t launch_fused_mt(const FusedPlan& f, const DeviceInfo& dev, cudaStream_t stream,
                            const FusedParams& p) {
  auto kernel = fused_decode<MT>;
  cudaError_t e = allow_max_smem(kernel, dev);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)f.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = f.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kernel, p);
  if (e == cudaSuccess) note_launches(1);
  return e;
}

}  // namespace

bool fused_decode_supported(int64_t M, int64_t d, int64_t I, const DeviceInfo& dev) {
  return make_fused_plan(M, d, I, dev).mt != 0;
}

cudaError_t launch_fused_decode(const void* x, int64_t M, const void* gamma, float eps,
                                const void* P, int T, const void* W_down, int64_t d, int64_t I,
                                const void* residual, float* out, void* out_bf16,
                                uint32_t* ticket, uint32_t* inited, uint32_t* done,
                                uint32_t* status, const DeviceInfo& dev, cudaStream_t stream) {
  const FusedPlan f = make_fused_plan(M, d, I, dev);
  if (f.mt == 0) return cudaErrorInvalidConfiguration;
  FusedParams p;
  memset(&p, 0, sizeof(p));
  cudaError_t e = encode_tmap_2d_bf16(&p.wd_map, W_down, (uint64_t)d, (uint64_t)I,
                                      (uint64_t)I * 2, (uint32_t)f.rows_d, (uint32_t)f.swbox,
                                      CU_TENSOR_MAP_SWIZZLE_NONE);
  if (e != cudaSuccess) return e;
  p.x = (const __nv_bfloat16*)x;
  p.gamma = (const __nv_bfloat16*)gamma;
  p.residual = (const __nv_bfloat16*)residual;
  p.out = out;
  p.out_bf16 = (__nv_bfloat16*)out_bf16;
  p.ticket = ticket;
  p.inited = inited;
  p.done = done;
  p.n_init = std::min(f.grid, 4);
  p.ctl.status = status;
  p.ctl.wait_ns = wait_timeout_ns();
  p.ctl.drop_last = fault_injection();
  p.gu = GateUpGeom{(const __nv_bfloat16*)P, T, (int)d, (int)I, f.gu.kc, f.gu.nchunks};
  p.eps = eps;
  p.M = (int)M;
  p.d = (int)d;
  p.I = (int)I;
  p.units = f.units;
  p.swbox = f.swbox;
  p.rows_d = f.rows_d;
  p.nrb = f.nrb;
  p.stages = f.stages;
  p.stage_bytes = f.stage_bytes;
  switch (f.mt) {
    case 1: return launch_fused_mt<1>(f, dev, stream, p);
    case 2: return launch_fused_mt<2>(f, dev, stream, p);
    case 3: return launch_fused_mt<3>(f, dev, stream, p);
    default: return launch_fused_mt<4>(f, dev, stream, p);
  }
}

}  // namespace fmlp
