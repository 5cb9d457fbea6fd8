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
//   * four consumer warps share every stage: warp w owns gate/up pair w (or
//     W_down row w) of the group, dots it with the activations held in shared
//     memory, and arrives on the stage's "empty" mbarrier;
//   * fused_decode runs both steps in one persistent launch, the "Fusion MLP"
//     of the pages: the producer streams the W_down rows right behind the
//     gate/up rows while the consumers finish the gate-up phase, meet at a
//     grid-wide barrier (every CTA needs all of the intermediate a), and go
//     on to the down projection, so HBM does not idle between the steps;
//   * launches use programmatic dependent launch: a kernel's producer starts
//     streaming weights before the previous kernel on the stream has
//     finished; only the consumers wait for its results.
// Every wait is bounded (global-timer deadline); on expiry the CTA sets the
// timeout bit of the workspace status word, lets its in-flight copies land
// and exits.
#include "common.cuh"
#include "internal.h"

#include <algorithm>
#include <mutex>
#include <set>

namespace fmlp {
namespace {

constexpr int kConsumers = 4;                     // consumer warps = rows (pairs) per group
constexpr int kThreads = (kConsumers + 1) * 32;   // warp 0 produces
constexpr int kMaxStages = 8;
constexpr int kHeader = 256;                      // full[8], empty[8] mbarriers
constexpr int64_t kMaxStageBytes = 64 * 1024;
constexpr uint64_t kDrainNs = 1000000000ull;      // in-flight copies land long before this
constexpr int kGateRows = 2 * kConsumers;         // rows per gate-up stage (4 gate + 4 up)
constexpr int kDownRows = kConsumers;             // rows per down stage

static_assert(2 * kMaxStages * 8 <= kHeader, "barrier block overflows its header");

__host__ __device__ constexpr size_t align128(size_t n) { return (n + 127) & ~size_t(127); }

// acc += w . s over 8 elements (w: 8 bf16; s: 8 floats)
__device__ __forceinline__ float dot8(const uint4& w, const float4& s0, const float4& s1,
                                      float acc) {
  acc = fmaf(bf16lo(w.x), s0.x, acc); acc = fmaf(bf16hi(w.x), s0.y, acc);
  acc = fmaf(bf16lo(w.y), s0.z, acc); acc = fmaf(bf16hi(w.y), s0.w, acc);
  acc = fmaf(bf16lo(w.z), s1.x, acc); acc = fmaf(bf16hi(w.z), s1.y, acc);
  acc = fmaf(bf16lo(w.w), s1.z, acc); acc = fmaf(bf16hi(w.w), s1.w, acc);
  return acc;
}

// acc += w . v over 8 elements (both bf16)
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

// Groups [first, first + count) of `total`, split as evenly as possible over
// `parts`; the remainder goes to the first parts, or to the last ones if
// `from_end` (so two phases split this way balance each other).
__device__ __forceinline__ void split_groups(int total, int part, int parts, bool from_end,
                                             int& first, int& count) {
  const int per = total / parts, rem = total % parts;
  const int q = from_end ? parts - 1 - part : part;
  const int f = q * per + min(q, rem);
  count = per + (q < rem ? 1 : 0);
  first = from_end ? total - f - count : f;
}

// ---------------------------------------------------------------------------
// Stage ring.  Every consumer warp processes every stage in order, so stage k
// lives in slot k % S with phase parity (k / S) & 1 on both barriers.
// ---------------------------------------------------------------------------
struct Ring {
  uint64_t* full;   // producer arrival + copied bytes
  uint64_t* empty;  // one arrival per consumer warp
  uint8_t* stage0;
  int stages;
  int stage_bytes;
  __device__ __forceinline__ uint8_t* buf(int slot) const {
    return stage0 + (size_t)slot * stage_bytes;
  }
};

struct CtaState {
  int abort;
  int issued;  // stages issued by the producer
};

__device__ __forceinline__ void init_ring(const Ring& r, CtaState& st) {
  for (int j = 0; j < r.stages; ++j) {
    mbar_init(&r.full[j], 1);
    mbar_init(&r.empty[j], kConsumers);
  }
  st.abort = 0;
  st.issued = 0;
  fence_barrier_init();
}

// After a timeout: let every copy the producer issued land before the CTA
// exits (its shared memory must outlive the copies).  Thread 0 only.  Only
// the last `stages` stages can still be in flight: each earlier one was
// waited on by all consumers before its slot was reissued.
__device__ void drain_ring(const Ring& r, int issued) {
  for (int k = max(0, issued - r.stages); k < issued; ++k)
    mbar_wait_bounded(&r.full[k % r.stages], (uint32_t)((k / r.stages) & 1), kDrainNs,
                      nullptr);
}

__device__ __forceinline__ void flag_timeout(CtaState* st, uint32_t* status) {
  st->abort = 1;
  atomicOr(status, kStatusTimeout);
}

// Common per-launch settings of the producers and consumers.
struct Control {
  uint32_t* status;    // workspace status word
  uint64_t wait_ns;    // deadline of every bounded wait
  int drop_last;       // testing: withhold each CTA's last stage (fmlp_set_fault_injection)
};

struct Producer {
  Ring ring;
  CtaState* st;
  Control ctl;
  uint64_t pol;
  int total;           // stages this CTA will issue (all phases)
  int k = 0;           // next stage index
  bool dep_waited = false;

  // Claim the slot for stage k; false (and abort) on timeout or injected drop.
  __device__ __forceinline__ bool acquire() {
    if (ctl.drop_last && k == total - 1) return false;
    if (k < ring.stages) return true;
    if (!dep_waited) {  // start the clock only once the previous kernel is done
      grid_dependency_wait();
      dep_waited = true;
    }
    if (mbar_wait_bounded(&ring.empty[k % ring.stages], (uint32_t)(((k / ring.stages) - 1) & 1),
                          ctl.wait_ns, &st->abort))
      return true;
    flag_timeout(st, ctl.status);
    return false;
  }
};

struct Consumer {
  Ring ring;
  CtaState* st;
  Control ctl;
  int k = 0;  // next stage index
  int lane;

  __device__ __forceinline__ const uint8_t* wait_full() {
    const int slot = k % ring.stages;
    if (!mbar_wait_bounded(&ring.full[slot], (uint32_t)((k / ring.stages) & 1), ctl.wait_ns,
                           &st->abort)) {
      if (lane == 0) flag_timeout(st, ctl.status);
      return nullptr;
    }
    return ring.buf(slot);
  }
  __device__ __forceinline__ void release() {
    __syncwarp();
    if (lane == 0) mbar_arrive(&ring.empty[k % ring.stages]);
    ++k;
  }
};

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
    const __nv_bfloat16* pg = g.P + gate_row((g0 + j) * kConsumers, g.T) * g.d;
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
        const uint32_t run = (uint32_t)(kConsumers * g.d * 2);
        bulk_copy_g2s(buf, pg, run, bar, pr.pol);
        bulk_copy_g2s(buf + run, pu, run, bar, pr.pol);
      } else {
        for (int r = 0; r < kGateRows; ++r) {
          const __nv_bfloat16* row =
              r < kConsumers ? pg + (int64_t)r * g.d : pu + (int64_t)(r - kConsumers) * g.d;
          bulk_copy_g2s(buf + (size_t)r * g.kc * 2, row + k0, (uint32_t)len * 2u, bar, pr.pol);
        }
      }
      ++pr.k;
    }
  }
  return true;
}

// s = x * gamma (exact in f32) for the CTA's token rows, and r = 1/sqrt(mean x^2 + eps).
template <int MT>
__device__ void stage_x_gamma(const __nv_bfloat16* x, const __nv_bfloat16* gamma, float eps,
                              int d, int m0, int mt, float* s, float (*red)[MT], float* rinv) {
  const int lane = threadIdx.x & 31, c = (threadIdx.x >> 5) - 1, ct = threadIdx.x - 32;
  float ss[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) ss[m] = 0.f;
  for (int v = ct; v < d / 8; v += kConsumers * 32) {
    const uint4 gv = ld_keep(gamma + (int64_t)v * 8);
    const float gf[8] = {bf16lo(gv.x), bf16hi(gv.x), bf16lo(gv.y), bf16hi(gv.y),
                         bf16lo(gv.z), bf16hi(gv.z), bf16lo(gv.w), bf16hi(gv.w)};
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      uint4 xv = make_uint4(0, 0, 0, 0);
      if (m < mt) xv = ld_keep(x + (int64_t)(m0 + m) * d + (int64_t)v * 8);
      const float xf[8] = {bf16lo(xv.x), bf16hi(xv.x), bf16lo(xv.y), bf16hi(xv.y),
                           bf16lo(xv.z), bf16hi(xv.z), bf16lo(xv.w), bf16hi(xv.w)};
#pragma unroll
      for (int e = 0; e < 8; ++e) ss[m] = fmaf(xf[e], xf[e], ss[m]);
      float4* dst = reinterpret_cast<float4*>(s + (int64_t)m * d + (int64_t)v * 8);
      dst[0] = make_float4(xf[0] * gf[0], xf[1] * gf[1], xf[2] * gf[2], xf[3] * gf[3]);
      dst[1] = make_float4(xf[4] * gf[4], xf[5] * gf[5], xf[6] * gf[6], xf[7] * gf[7]);
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const float t = warp_sum(ss[m]);
    if (lane == 0) red[c][m] = t;
  }
  named_barrier_sync(1, kConsumers * 32);
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) t += red[w][m];
    rinv[m] = 1.0f / sqrtf(t / (float)d + eps);
  }
}

// Consumer warp c: pair c of every group; writes a[m, i] for its pairs.
template <int MT>
__device__ bool consume_gateup(Consumer& cs, const GateUpGeom& g, int g0, int n_groups,
                               const float* s, const float* rinv, __nv_bfloat16* a, int m0,
                               int mt) {
  const int c = (threadIdx.x >> 5) - 1, lane = cs.lane;
  for (int j = 0; j < n_groups; ++j) {
    float ag[2][MT], au[2][MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) ag[0][m] = ag[1][m] = au[0][m] = au[1][m] = 0.f;
    for (int ch = 0; ch < g.nchunks; ++ch) {
      const uint8_t* buf = cs.wait_full();
      if (!buf) return false;
      const int k0 = ch * g.kc;
      const int nv = min(g.kc, g.d - k0) / 8;
      const uint8_t* bg = buf + (size_t)c * g.kc * 2;
      const uint8_t* bu = buf + (size_t)(kConsumers + c) * g.kc * 2;
      const float* sk = s + k0;
      int v = lane;
      for (; v + 32 < nv; v += 64) {  // two independent accumulator sets
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int vv = v + 32 * h;
          const uint4 wg = lds128(bg + 16 * vv);
          const uint4 wu = lds128(bu + 16 * vv);
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const float4* sp = reinterpret_cast<const float4*>(sk + (int64_t)m * g.d + 8 * vv);
            const float4 s0 = sp[0], s1 = sp[1];
            ag[h][m] = dot8(wg, s0, s1, ag[h][m]);
            au[h][m] = dot8(wu, s0, s1, au[h][m]);
          }
        }
      }
      if (v < nv) {
        const uint4 wg = lds128(bg + 16 * v);
        const uint4 wu = lds128(bu + 16 * v);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const float4* sp = reinterpret_cast<const float4*>(sk + (int64_t)m * g.d + 8 * v);
          const float4 s0 = sp[0], s1 = sp[1];
          ag[0][m] = dot8(wg, s0, s1, ag[0][m]);
          au[0][m] = dot8(wu, s0, s1, au[0][m]);
        }
      }
      cs.release();
    }
    const int item = (g0 + j) * kConsumers + c;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float gs = warp_sum(ag[0][m] + ag[1][m]);
      const float us = warp_sum(au[0][m] + au[1][m]);
      if (lane == m && m < mt)
        a[(int64_t)(m0 + m) * g.I + item] =
            __float2bfloat16_rn(silu_mul(gs * rinv[m], us * rinv[m]));
    }
  }
  return true;
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
  named_barrier_sync(1, kConsumers * 32);
}

template <int MT>
__device__ bool consume_down(Consumer& cs, const DownGeom& g, int g0, int n_groups,
                             const uint8_t* act, const __nv_bfloat16* residual, float* out,
                             int m0, int mt) {
  const int c = (threadIdx.x >> 5) - 1, lane = cs.lane;
  for (int j = 0; j < n_groups; ++j) {
    float acc[2][MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[0][m] = acc[1][m] = 0.f;
    for (int ch = 0; ch < g.nchunks; ++ch) {
      const uint8_t* buf = cs.wait_full();
      if (!buf) return false;
      const int k0 = ch * g.kc;
      const int nv = min(g.kc, g.I - k0) / 8;
      const uint8_t* bw = buf + (size_t)c * g.kc * 2;
      const uint8_t* ak = act + (size_t)k0 * 2;
      int v = lane;
      for (; v + 32 < nv; v += 64) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int vv = v + 32 * h;
          const uint4 w = lds128(bw + 16 * vv);
#pragma unroll
          for (int m = 0; m < MT; ++m)
            acc[h][m] = dot8bf(w, lds128(ak + ((size_t)m * g.I + 8 * vv) * 2), acc[h][m]);
        }
      }
      if (v < nv) {
        const uint4 w = lds128(bw + 16 * v);
#pragma unroll
        for (int m = 0; m < MT; ++m)
          acc[0][m] = dot8bf(w, lds128(ak + ((size_t)m * g.I + 8 * v) * 2), acc[0][m]);
      }
      cs.release();
    }
    const int n = (g0 + j) * kDownRows + c;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float t = warp_sum(acc[0][m] + acc[1][m]);
      if (lane == m && m < mt) {
        float o = t;
        if (residual) o += __bfloat162float(residual[(int64_t)(m0 + m) * g.d + n]);
        out[(int64_t)(m0 + m) * g.d + n] = o;
      }
    }
  }
  return true;
}

// Grid-wide barrier between the two phases of fused_decode, run by one thread
// per CTA.  `count` returns to zero after every use; `gen` is a free-running
// generation counter.  Bounded: gives up after wait_ns.
__device__ bool grid_barrier(uint32_t* count, uint32_t* gen, uint32_t nblocks,
                             uint64_t wait_ns) {
  const uint32_t g = ld_acquire_gpu(gen);
  __threadfence();
  if (atomicAdd(count, 1u) == nblocks - 1) {
    atomicExch(count, 0u);
    __threadfence();
    atomicAdd(gen, 1u);
    return true;
  }
  const uint64_t t0 = globaltimer_ns();
  while (ld_acquire_gpu(gen) == g) {
    __nanosleep(64);
    if (globaltimer_ns() - t0 > wait_ns) return false;
  }
  __threadfence();
  return true;
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
  uint32_t* barrier;     // fused: [0] arrival count, [32] generation (separate lines)
  Control ctl;
  GateUpGeom gu;
  DownGeom dn;
  float eps;
  int M;
  int stages, stage_bytes;
};

template <int MT, bool GATE, bool DOWN>
__device__ __forceinline__ void stream_body(const StreamParams& p, size_t act_bytes) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ float red[kConsumers][MT];
  __shared__ CtaState st;

  Ring ring;
  ring.full = reinterpret_cast<uint64_t*>(smem);
  ring.empty = ring.full + kMaxStages;
  uint8_t* act = smem + kHeader;
  ring.stage0 = smem + kHeader + act_bytes;
  ring.stages = p.stages;
  ring.stage_bytes = p.stage_bytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * MT;
  const int mt = min(MT, p.M - m0);
  int ga0 = 0, nga = 0, gd0 = 0, ngd = 0;
  if (GATE) split_groups(p.gu.I / kConsumers, blockIdx.x, gridDim.x, false, ga0, nga);
  if (DOWN) split_groups(p.dn.d / kDownRows, blockIdx.x, gridDim.x, GATE, gd0, ngd);

  if (threadIdx.x == 0) init_ring(ring, st);
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
  } else {
    grid_dependency_wait();  // inputs may be written by the previous kernel
    Consumer cs{ring, &st, p.ctl, 0, lane};
    bool ok = true;
    if (GATE) {
      float rinv[MT];
      stage_x_gamma<MT>(p.x, p.gamma, p.eps, p.gu.d, m0, mt, reinterpret_cast<float*>(act),
                        red, rinv);
      ok = consume_gateup<MT>(cs, p.gu, ga0, nga, reinterpret_cast<const float*>(act), rinv,
                              p.a, m0, mt);
    }
    if (GATE && DOWN) {
      // every CTA needs all of a: grid-wide barrier (act is then reused for a)
      named_barrier_sync(1, kConsumers * 32);
      if (threadIdx.x == 32 && !grid_barrier(p.barrier, p.barrier + 32, gridDim.x,
                                             p.ctl.wait_ns))
        flag_timeout(&st, p.ctl.status);
      named_barrier_sync(1, kConsumers * 32);
      ok = ok && !st.abort;
    }
    if (DOWN && ok) {
      stage_a<MT>(p.a, p.dn.I, m0, mt, act);
      consume_down<MT>(cs, p.dn, gd0, ngd, act, p.residual, p.out, m0, mt);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && st.abort) drain_ring(ring, st.issued);
}

template <int MT>
__global__ void __launch_bounds__(kThreads, 1) gateup_stream(const StreamParams p) {
  stream_body<MT, true, false>(p, align128((size_t)MT * p.gu.d * sizeof(float)));
}

template <int MT>
__global__ void __launch_bounds__(kThreads, 1) down_stream(const StreamParams p) {
  stream_body<MT, false, true>(p, align128((size_t)MT * p.dn.I * 2));
}

template <int MT>
__global__ void __launch_bounds__(kThreads, 1) fused_decode(const StreamParams p) {
  const size_t act_g = align128((size_t)MT * p.gu.d * sizeof(float));
  const size_t act_d = align128((size_t)MT * p.dn.I * 2);
  stream_body<MT, true, true>(p, act_g > act_d ? act_g : act_d);
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
      size_t act = 0;
      if (gate) act = std::max(act, align128((size_t)mt * d * sizeof(float)));
      if (down) act = std::max(act, align128((size_t)mt * I * 2));
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
                         void* a, const void* residual, float* out, uint32_t* status,
                         uint32_t* barrier) {
  StreamParams p = {};
  p.x = (const __nv_bfloat16*)x;
  p.gamma = (const __nv_bfloat16*)gamma;
  p.residual = (const __nv_bfloat16*)residual;
  p.a = (__nv_bfloat16*)a;
  p.out = out;
  p.barrier = barrier;
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
FMLP_KERNEL_TAG(fused_decode)
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
                                     nullptr, status, nullptr);
  const dim3 grid((unsigned)std::min<int64_t>(I / kConsumers, dev.sm_count),
                  (unsigned)((M + pl.mt - 1) / pl.mt));
  return launch_mt<gateup_stream_tag>(pl.mt, grid, pl, dev, stream, p);
}

cudaError_t launch_down_stream(const void* a, int64_t M, const void* W_down, int64_t d,
                               int64_t I, const void* residual, float* out, uint32_t* status,
                               const DeviceInfo& dev, cudaStream_t stream) {
  const Plan pl = make_plan(M, d, I, false, true, dev);
  if (pl.mt == 0) return cudaErrorInvalidConfiguration;
  const StreamParams p = make_params(pl, nullptr, M, nullptr, 0.f, nullptr, 0, W_down, d, I,
                                     const_cast<void*>(a), residual, out, status, nullptr);
  const dim3 grid((unsigned)std::min<int64_t>(d / kDownRows, dev.sm_count),
                  (unsigned)((M + pl.mt - 1) / pl.mt));
  return launch_mt<down_stream_tag>(pl.mt, grid, pl, dev, stream, p);
}

bool fused_decode_supported(int64_t M, int64_t d, int64_t I, const DeviceInfo& dev) {
  const Plan pl = make_plan(M, d, I, true, true, dev);
  return pl.mt != 0 && pl.mt >= M;  // one pass over the weights: all rows in one CTA row
}

cudaError_t launch_fused_decode(const void* x, int64_t M, const void* gamma, float eps,
                                const void* P, int T, const void* W_down, int64_t d, int64_t I,
                                void* a, const void* residual, float* out, uint32_t* status,
                                uint32_t* barrier, const DeviceInfo& dev, cudaStream_t stream) {
  const Plan pl = make_plan(M, d, I, true, true, dev);
  if (pl.mt == 0 || pl.mt < M) return cudaErrorInvalidConfiguration;
  const StreamParams p = make_params(pl, x, M, gamma, eps, P, T, W_down, d, I, a, residual, out,
                                     status, barrier);
  // one CTA per SM at most, so every CTA is resident for the grid barrier
  const int groups = (int)std::min<int64_t>(I / kConsumers, d / kDownRows);
  const dim3 grid((unsigned)std::min(groups, dev.sm_count), 1);
  return launch_mt<fused_decode_tag>(pl.mt, grid, pl, dev, stream, p);
}

}  // namespace fmlp
