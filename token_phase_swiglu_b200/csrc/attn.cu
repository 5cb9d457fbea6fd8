// Token-phase attention step: the GKVC and TPSFLAT components of "FastTPS:
// An Optimized Method for LLM Token Phase for AI Accelerators" (xllm-io paper
// review), section 三, components 1-2, Figure 3 and Eq(2).
//
// For each of B sequences one new token arrives with q [H x D] and k, v
// [H_kv x D].  The step
//   * rotates q and k by RoPE at the token's position p (rotate-half pairs
//     (i, i + D/2), angle_i = p theta^(-2i/D), angles in binary64);
//   * appends the rotated k (rounded to bf16) and v to the cache in place, at
//     the Eq(2) address: row p of KV head g's region of N_max rows (GKVC: no
//     Concat rebuilds the cache);
//   * attends each query head h (KV head g = h / (H / H_kv)) over rows 0..p:
//     o_h = softmax(q'_h K_g^T / sqrt(D)) V_g, with RoPE, QK^T, the softmax and
//     PV fused in one pass over tiles of the cache (TPSFLAT).
//
// B200 mapping.  The work is the KV rows of every (sequence, KV head) segment,
// cut into units of 64 rows and split evenly over one CTA per SM (stream-K:
// a CTA's range may end inside one segment and start inside another).  Warp
// 0's elected lane streams each unit's K and V tiles into a ring of shared-
// memory stages with two 3-D TMA copies (swizzled column blocks, so that
// lanes reading their own rows meet no bank conflict; see AttnTile).  Eight
// consumer warps take the stages two at a time, 32 rows each: QK^T with one
// row per lane (the G query heads of the KV head at once, q held in shared
// memory, packed f32x2 FMAs), an online softmax in base 2 (scores carry
// log2(e)/sqrt(D)), and PV with the head's dimensions spread over the lanes.
// At the end of a segment's piece the warps' states are merged; the CTA that
// holds the new row folds it in from registers and writes it to the cache; a
// segment split over several CTAs is merged by the last to finish (arrival
// counter, no waiting on another CTA).
#include "common.cuh"
#include "internal.h"
#include "ring.cuh"
#include "tmap.h"

#include <math_constants.h>

#include <algorithm>
#include <cmath>
#include <cstddef>
#include <mutex>
#include <set>

namespace fmlp {
namespace {

constexpr int kAttnWarps = 8;                                   // consumer warps
constexpr int kAttnWarpsPerStage = 2;                           // 32 rows each
constexpr int kAttnGroups = kAttnWarps / kAttnWarpsPerStage;    // stages in work at once
constexpr int kAttnRows = 32 * kAttnWarpsPerStage;              // rows per unit (stage)
constexpr int kAttnThreads = (kAttnWarps + 1) * 32;             // warp 0 produces
constexpr int kAttnConsumerThreads = kAttnWarps * 32;
constexpr int kAttnBar = 1;                                     // consumer-only named barrier
constexpr int kAttnMaxCtas = 256;
constexpr int kAttnTileBytesPerBlock = kAttnRows * 64;          // per 32 columns of a tile
// Head dimensions that are multiples of 64 are copied in 64-column blocks with
// the 128-byte swizzle (128-byte pieces per row), the others (96) in
// 32-column blocks with the 64-byte swizzle.
constexpr bool kAttnWideBlocks = true;
// Consumer warps waiting for their next stage sleep between polls instead of
// taking issue slots from the warps that are computing.
constexpr bool kAttnBackoff = true;

template <int DC>
struct AttnTile {
  static constexpr bool wide = kAttnWideBlocks && DC % 2 == 0;
  static constexpr int block_cols = wide ? 64 : 32;
  static constexpr int row_bytes = block_cols * 2;           // of one block
  static constexpr int block_bytes = kAttnRows * row_bytes;
  // byte offset of element (row, column d) in a tile
  __device__ static __forceinline__ int offset(int row, int d) {
    const int zb = d / block_cols, col = d % block_cols;
    const int sw = wide ? (row & 7) : ((row >> 1) & 3);
    return zb * block_bytes + row * row_bytes + ((((col >> 3) ^ sw)) << 4) + (col & 7) * 2;
  }
};

__device__ __forceinline__ bool attn_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                          volatile int* abort) {
  if (!kAttnBackoff) return mbar_wait_bounded(bar, parity, limit_ns, abort);
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    __nanosleep(64);
    if (mbar_test(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

struct AttnParams {
  CUtensorMap k_map;        // cache as [B H_kv N_max rows x D] bf16: 32-column blocks, 64-B swizzle
  CUtensorMap v_map;
  const __nv_bfloat16* q;   // [B x H x D]
  const __nv_bfloat16* k_new;  // [B x H_kv x D]
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_cache;   // [B x H_kv x N_max x D]
  __nv_bfloat16* v_cache;
  const int32_t* pos;       // [B]
  float* out;               // [B x H x D]
  float* partials;          // [ctas + segments - 1][G][2 + D]: m, l, acc of a CTA's piece
  uint32_t* counters;       // [segments]: pieces merged (zero between calls)
  Control ctl;
  int B, H, H_kv, D, G;
  int64_t n_max;            // rows of a head's region (N_p + N_r)
  int n_ctx;                // every position < n_ctx
  int useg;                 // units per segment: ceil(n_ctx / 64)
  int64_t units;            // segments x useg
  float qscale;             // log2(e) / sqrt(D)
  double inv_freq[64];      // theta^(-2i/D), i < D/2 (binary64, from the host)
  int stages, stage_bytes;
};

// Shared-memory block after the ring barriers (floats unless noted).  q and
// p are read as float4, so they lead, 16-byte aligned.
template <int DC, int G>
struct AttnSmem {
  static constexpr int D = 32 * DC;
  alignas(16) float q[G * D];            // rotated q of the segment's G heads, times qscale
  alignas(16) float p[kAttnWarps * G * 32];  // per-warp weights of the 32 rows in work
  float wacc[kAttnWarps * G * D];        // per-warp softmax state: accumulators,
  float wm[kAttnWarps * G], wl[kAttnWarps * G];  // running maxima and sums
  float cs[D / 2], sn[D / 2];            // cos, sin of the RoPE angles at the token's position
  float kr[D], vn[D];                    // the new row: rotated k (bf16 value) and v
  float s_new[G];                        // its scores
  int last;                              // this CTA merges the segment
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
// bf16 pair as two f32 lanes
__device__ __forceinline__ uint64_t bf16x2_f32x2(uint32_t w) { return pk2(bf16lo(w), bf16hi(w)); }

__host__ __device__ inline int64_t unit_begin(int c, int ctas, int64_t units) {
  return (int64_t)c * units / ctas;
}
// The CTA whose unit range holds unit u (ranges [unit_begin(c), unit_begin(c + 1))).
__device__ __forceinline__ int cta_of_unit(int64_t u, int ctas, int64_t units) {
  return (int)(((u + 1) * ctas - 1) / units);
}

// Rows of unit j of a segment whose new row is p: the held rows [64 j, p).
__device__ __forceinline__ int unit_rows(int j, int p) {
  return min(max(p - j * kAttnRows, 0), kAttnRows);
}

// A position the call does not take: flagged, and its segments skipped by every CTA.
__device__ __forceinline__ bool bad_position(int p, int n_ctx) { return p < 0 || p >= n_ctx; }

template <int DC, int G>
__global__ void __launch_bounds__(kAttnThreads, 1) attn_decode(const __grid_constant__ AttnParams p) {
  constexpr int D = 32 * DC;
  using Sm = AttnSmem<DC, G>;
  static_assert(offsetof(Sm, q) % 16 == 0 && offsetof(Sm, p) % 16 == 0,
                "float4 reads need 16-byte alignment");
  static_assert(kHeader % 16 == 0, "the block starts 16-byte aligned");
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ CtaState st;
  AttnSmem<DC, G>& sh = *reinterpret_cast<AttnSmem<DC, G>*>(smem + kHeader);

  Ring ring;
  ring.full = reinterpret_cast<uint64_t*>(smem);
  ring.empty = ring.full + kMaxStages;
  ring.stage0 = smem + ((kHeader + sizeof(AttnSmem<DC, G>) + 1023) & ~size_t(1023));
  ring.stages = p.stages;
  ring.stage_bytes = p.stage_bytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ctas = gridDim.x, c = blockIdx.x;
  const int64_t u0 = unit_begin(c, ctas, p.units), u1 = unit_begin(c + 1, ctas, p.units);
  const int64_t seg0 = u0 / p.useg, seg1 = (u1 - 1) / p.useg;  // segments this CTA touches

  if (threadIdx.x == 0) init_ring(ring, st, kAttnWarpsPerStage);
  __syncthreads();
  grid_launch_dependents();
  grid_dependency_wait();  // the cache and the positions may come from the previous kernel

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      // every unit of the range, whatever the positions (the consumers mask the
      // rows at and past a sequence's position), so the first copies need no
      // read of the positions
      const int total = (int)(u1 - u0);
      Producer pr{ring, &st, p.ctl, evict_first_policy(), total};
      const uint32_t tile = (uint32_t)(DC * kAttnTileBytesPerBlock);
      bool ok = true;
      for (int64_t s = seg0; s <= seg1 && ok; ++s) {
        for (int64_t u = max(u0, s * p.useg); u < min(u1, (s + 1) * p.useg); ++u) {
          const int j = (int)(u - s * p.useg);
          if (!pr.acquire()) {
            ok = false;
            break;
          }
          const int slot = pr.k % ring.stages;
          uint8_t* buf = ring.buf(slot);
          uint64_t* bar = &ring.full[slot];
          mbar_arrive_expect_tx(bar, 2 * tile);  // boxes land whole (zeros past the tensor's end)
          const int row0 = (int)(s * p.n_max + (int64_t)j * kAttnRows);
          tma_load_3d(buf, &p.k_map, 0, row0, 0, bar, pr.pol);
          tma_load_3d(buf + tile, &p.v_map, 0, row0, 0, bar, pr.pol);
          ++pr.k;
        }
      }
      st.issued = pr.k;
    }
    __syncwarp();
  } else {
    // ---------------- consumers ----------------
    const int w = warp - 1, half = w % kAttnWarpsPerStage, grp = w / kAttnWarpsPerStage;
    const int ct = threadIdx.x - 32;
    int k = 0;  // stages consumed by the CTA so far (every warp counts all of them)
    bool ok = true;
    for (int64_t s = seg0; s <= seg1; ++s) {
      const int b = (int)(s / p.H_kv), g = (int)(s % p.H_kv);
      const int pb = __ldg(p.pos + b);
      if (bad_position(pb, p.n_ctx)) {
        if (ct == 0) atomicOr(p.ctl.status, kStatusBadInput);
        // its stages arrive all the same: take them and give them back
        for (int64_t u = max(u0, s * p.useg); u < min(u1, (s + 1) * p.useg) && ok; ++u, ++k) {
          if (k % kAttnGroups != grp) continue;
          const int slot = k % ring.stages;
          if (!attn_wait(&ring.full[slot], (uint32_t)((k / ring.stages) & 1), p.ctl.wait_ns,
                         &st.abort)) {
            if (lane == 0) flag_timeout(&st, p.ctl.status);
            ok = false;
            break;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&ring.empty[slot]);
        }
        if (consumer_barrier_any<kAttnConsumerThreads>(kAttnBar, !ok)) break;
        continue;
      }
      const int64_t sa = max(u0, s * p.useg), se = min(u1, (s + 1) * p.useg);
      const int64_t jnew = s * p.useg + pb / kAttnRows;  // unit holding the new row
      const bool owner = jnew >= sa && jnew < se;

      // RoPE at position pb: angles in binary64, then the rotated q (and, in
      // the owner, the new k and v, which it also appends to the cache).
      for (int i = ct; i < D / 2; i += kAttnConsumerThreads) {
        const double a = (double)pb * p.inv_freq[i];
        double sd, cd;
        sincos(a, &sd, &cd);
        sh.cs[i] = (float)cd;
        sh.sn[i] = (float)sd;
      }
      named_barrier_sync(kAttnBar, kAttnConsumerThreads);
      for (int t = ct; t < G * (D / 2); t += kAttnConsumerThreads) {
        const int h = t / (D / 2), i = t % (D / 2);
        const __nv_bfloat16* qh = p.q + ((int64_t)b * p.H + (int64_t)g * G + h) * D;
        const float x0 = __bfloat162float(qh[i]), x1 = __bfloat162float(qh[i + D / 2]);
        sh.q[h * D + i] = (x0 * sh.cs[i] - x1 * sh.sn[i]) * p.qscale;
        sh.q[h * D + i + D / 2] = (x0 * sh.sn[i] + x1 * sh.cs[i]) * p.qscale;
      }
      if (owner) {
        const int64_t src = ((int64_t)b * p.H_kv + g) * D;
        const int64_t dst = (s * p.n_max + pb) * D;  // Eq(2), offset by the segment's region
        for (int i = ct; i < D / 2; i += kAttnConsumerThreads) {
          const float x0 = __bfloat162float(p.k_new[src + i]);
          const float x1 = __bfloat162float(p.k_new[src + i + D / 2]);
          const __nv_bfloat16 r0 = __float2bfloat16_rn(x0 * sh.cs[i] - x1 * sh.sn[i]);
          const __nv_bfloat16 r1 = __float2bfloat16_rn(x0 * sh.sn[i] + x1 * sh.cs[i]);
          sh.kr[i] = __bfloat162float(r0);
          sh.kr[i + D / 2] = __bfloat162float(r1);
          p.k_cache[dst + i] = r0;
          p.k_cache[dst + i + D / 2] = r1;
        }
        for (int i = ct; i < D; i += kAttnConsumerThreads) {
          const __nv_bfloat16 v = p.v_new[src + i];
          sh.vn[i] = __bfloat162float(v);
          p.v_cache[dst + i] = v;
        }
      }
      named_barrier_sync(kAttnBar, kAttnConsumerThreads);
      if (owner && w < G) {  // score of the new row for head w
        float t = 0.f;
        for (int i = lane; i < D; i += 32) t = fmaf(sh.q[w * D + i], sh.kr[i], t);
        t = warp_sum(t);
        if (lane == 0) sh.s_new[w] = t;
      }

      // this warp's share of the piece's stages
      float m[G], l[G], acc[G][DC];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m[h] = -CUDART_INF_F;
        l[h] = 0.f;
#pragma unroll
        for (int i = 0; i < DC; ++i) acc[h][i] = 0.f;
      }
      for (int64_t u = sa; u < se && ok; ++u) {
        const int rows = unit_rows((int)(u - s * p.useg), pb);  // 0 past the position
        if (k % kAttnGroups == grp) {
          const int slot = k % ring.stages;
          if (!attn_wait(&ring.full[slot], (uint32_t)((k / ring.stages) & 1), p.ctl.wait_ns,
                         &st.abort)) {
            if (lane == 0) flag_timeout(&st, p.ctl.status);
            ok = false;
            break;
          }
          const uint8_t* kt = ring.buf(slot);
          const uint8_t* vt = kt + DC * kAttnTileBytesPerBlock;
          // QK^T: one row per lane
          const int r = half * 32 + lane;
          const bool valid = r < rows;
          uint64_t sacc[G];
#pragma unroll
          for (int h = 0; h < G; ++h) sacc[h] = 0ull;
#pragma unroll
          for (int z = 0; z < DC; ++z) {
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const uint4 kv = lds128(kt + AttnTile<DC>::offset(r, z * 32 + cc * 8));
              const uint64_t k0 = bf16x2_f32x2(kv.x), k1 = bf16x2_f32x2(kv.y);
              const uint64_t k2 = bf16x2_f32x2(kv.z), k3 = bf16x2_f32x2(kv.w);
#pragma unroll
              for (int h = 0; h < G; ++h) {
                const float4 qa = *reinterpret_cast<const float4*>(&sh.q[h * D + z * 32 + cc * 8]);
                const float4 qb = *reinterpret_cast<const float4*>(&sh.q[h * D + z * 32 + cc * 8 + 4]);
                sacc[h] = ffma2(k0, pk2(qa.x, qa.y), sacc[h]);
                sacc[h] = ffma2(k1, pk2(qa.z, qa.w), sacc[h]);
                sacc[h] = ffma2(k2, pk2(qb.x, qb.y), sacc[h]);
                sacc[h] = ffma2(k3, pk2(qb.z, qb.w), sacc[h]);
              }
            }
          }
          // online softmax (base 2)
          float* pw = &sh.p[w * G * 32];
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float sv = valid ? hsum2(sacc[h]) : -CUDART_INF_F;
            const float mnew = fmaxf(m[h], warp_max(sv));
            float pv = 0.f;
            if (mnew != -CUDART_INF_F) {
              const float alpha = exp2f(m[h] - mnew);  // 0 while m is -inf
              pv = valid ? exp2f(sv - mnew) : 0.f;
              l[h] = l[h] * alpha + pv;
#pragma unroll
              for (int i = 0; i < DC; ++i) acc[h][i] *= alpha;
              m[h] = mnew;
            }
            pw[h * 32 + lane] = pv;
          }
          __syncwarp();
          // PV: lane owns dimensions lane + 32 i
          const int nr = min(max(rows - half * 32, 0), 32);
          int rr = 0;
          for (; rr + 4 <= nr; rr += 4) {
            float4 pp[G];
#pragma unroll
            for (int h = 0; h < G; ++h) pp[h] = *reinterpret_cast<const float4*>(&pw[h * 32 + rr]);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const int row = half * 32 + rr + q4;
              float v[DC];
#pragma unroll
              for (int i = 0; i < DC; ++i)
                v[i] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                    vt + AttnTile<DC>::offset(row, lane + 32 * i)));
#pragma unroll
              for (int h = 0; h < G; ++h) {
                const float ph = q4 == 0 ? pp[h].x : q4 == 1 ? pp[h].y : q4 == 2 ? pp[h].z : pp[h].w;
#pragma unroll
                for (int i = 0; i < DC; ++i) acc[h][i] = fmaf(ph, v[i], acc[h][i]);
              }
            }
          }
          for (; rr < nr; ++rr) {
            const int row = half * 32 + rr;
#pragma unroll
            for (int i = 0; i < DC; ++i) {
              const float v = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                  vt + AttnTile<DC>::offset(row, lane + 32 * i)));
#pragma unroll
              for (int h = 0; h < G; ++h) acc[h][i] = fmaf(pw[h * 32 + rr], v, acc[h][i]);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&ring.empty[slot]);
        }
        ++k;
      }
      // this warp's state into shared memory
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float ls = warp_sum(l[h]);
        if (lane == 0) {
          sh.wm[w * G + h] = m[h];
          sh.wl[w * G + h] = ls;
        }
#pragma unroll
        for (int i = 0; i < DC; ++i) sh.wacc[(w * G + h) * D + lane + 32 * i] = acc[h][i];
      }
      if (consumer_barrier_any<kAttnConsumerThreads>(kAttnBar, !ok)) break;

      // merge the warps (and the new row) into this CTA's piece of the segment
      const int cf = cta_of_unit(s * p.useg, ctas, p.units);
      const int cl = cta_of_unit((s + 1) * p.useg - 1, ctas, p.units);
      float* piece = p.partials + (size_t)(c + s) * G * (2 + D);
      for (int t = ct; t < G * D; t += kAttnConsumerThreads) {
        const int h = t / D, d = t % D;
        float M = -CUDART_INF_F;
#pragma unroll
        for (int ww = 0; ww < kAttnWarps; ++ww) M = fmaxf(M, sh.wm[ww * G + h]);
        if (owner) M = fmaxf(M, sh.s_new[h]);
        float A = 0.f, L = 0.f;
        if (M != -CUDART_INF_F) {
#pragma unroll
          for (int ww = 0; ww < kAttnWarps; ++ww) {
            const float f = exp2f(sh.wm[ww * G + h] - M);
            A = fmaf(f, sh.wacc[(ww * G + h) * D + d], A);
            L = fmaf(f, sh.wl[ww * G + h], L);
          }
          if (owner) {
            const float f = exp2f(sh.s_new[h] - M);
            A = fmaf(f, sh.vn[d], A);
            L += f;
          }
        }
        if (cf == cl) {
          p.out[((int64_t)b * p.H + (int64_t)g * G + h) * D + d] = A / L;
        } else {
          piece[h * (2 + D) + 2 + d] = A;
          if (d == 0) {
            piece[h * (2 + D)] = M;
            piece[h * (2 + D) + 1] = L;
          }
        }
      }
      if (cf != cl) {
        __threadfence();
        named_barrier_sync(kAttnBar, kAttnConsumerThreads);
        if (ct == 0) sh.last = atomicAdd(p.counters + s, 1u) == (uint32_t)(cl - cf);
        named_barrier_sync(kAttnBar, kAttnConsumerThreads);
        if (sh.last) {
          __threadfence();
          for (int t = ct; t < G * D; t += kAttnConsumerThreads) {
            const int h = t / D, d = t % D;
            // the pieces' loads are independent: unrolled so that they overlap
            // (an L2 round trip each otherwise); an empty piece has m = -inf,
            // weight exp2(-inf) = 0 and zero sums
            float M = -CUDART_INF_F;
#pragma unroll 4
            for (int cc = cf; cc <= cl; ++cc)
              M = fmaxf(M, __ldcg(p.partials + (size_t)(cc + s) * G * (2 + D) + h * (2 + D)));
            float A = 0.f, L = 0.f;
#pragma unroll 4
            for (int cc = cf; cc <= cl; ++cc) {
              const float* pc = p.partials + (size_t)(cc + s) * G * (2 + D) + h * (2 + D);
              const float mc = __ldcg(pc), lc = __ldcg(pc + 1), ac = __ldcg(pc + 2 + d);
              const float f = exp2f(mc - M);
              A = fmaf(f, ac, A);
              L = fmaf(f, lc, L);
            }
            p.out[((int64_t)b * p.H + (int64_t)g * G + h) * D + d] = A / L;
          }
          if (ct == 0) atomicExch(p.counters + s, 0u);
        }
      }
      named_barrier_sync(kAttnBar, kAttnConsumerThreads);  // shared memory reused next
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && st.abort) drain_ring(ring, st.issued);
}

template <int DC, int G>
size_t attn_fixed_smem() {
  return (kHeader + sizeof(AttnSmem<DC, G>) + 1023) & ~size_t(1023);
}

struct AttnPlan {
  int ctas = 0, stages = 0, stage_bytes = 0, useg = 0;
  int64_t units = 0;
  size_t smem = 0;
};

template <int DC, int G>
AttnPlan attn_plan(int64_t B, int H_kv, int n_ctx, const DeviceInfo& dev) {
  AttnPlan pl;
  pl.useg = (n_ctx + kAttnRows - 1) / kAttnRows;
  pl.units = B * H_kv * (int64_t)pl.useg;
  pl.ctas = (int)std::min<int64_t>(std::min(dev.sm_count, kAttnMaxCtas), pl.units);
  pl.stage_bytes = 2 * DC * kAttnTileBytesPerBlock;
  const size_t budget = (size_t)dev.max_smem_optin - 1024;  // static shared memory + slack
  const size_t fixed = attn_fixed_smem<DC, G>();
  if (fixed >= budget) return AttnPlan();
  pl.stages = (int)std::min<size_t>(kMaxStages, (budget - fixed) / pl.stage_bytes);
  if (pl.stages < 2) return AttnPlan();
  pl.smem = fixed + (size_t)pl.stages * pl.stage_bytes;
  return pl;
}

template <typename Kernel>
cudaError_t allow_attn_smem(Kernel k, const DeviceInfo& dev) {
  static std::mutex mu;
  static std::set<std::pair<int, const void*>> done;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(dev.device, (const void*)k);
  if (done.count(key)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       dev.max_smem_optin - 1024);
  if (e == cudaSuccess) done.insert(key);
  return e;
}

template <int DC, int G>
cudaError_t launch_attn_t(AttnParams& p, const DeviceInfo& dev, cudaStream_t stream) {
  const AttnPlan pl = attn_plan<DC, G>(p.B, p.H_kv, p.n_ctx, dev);
  if (pl.ctas == 0) return cudaErrorInvalidValue;
  auto kern = attn_decode<DC, G>;
  cudaError_t e = allow_attn_smem(kern, dev);
  if (e != cudaSuccess) return e;
  p.useg = pl.useg;
  p.units = pl.units;
  p.stages = pl.stages;
  p.stage_bytes = pl.stage_bytes;
  const uint64_t rows = (uint64_t)p.B * p.H_kv * (uint64_t)p.n_max;
  using Tile = AttnTile<DC>;
  const CUtensorMapSwizzle sw = Tile::wide ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const uint32_t blocks = (uint32_t)(p.D / Tile::block_cols);
  e = encode_tmap_blocks_bf16(&p.k_map, p.k_cache, rows, (uint64_t)p.D, (uint64_t)p.D * 2,
                              Tile::block_cols, kAttnRows, blocks, sw);
  if (e == cudaSuccess)
    e = encode_tmap_blocks_bf16(&p.v_map, p.v_cache, rows, (uint64_t)p.D, (uint64_t)p.D * 2,
                                Tile::block_cols, kAttnRows, blocks, sw);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)pl.ctas);
  cfg.blockDim = dim3(kAttnThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e == cudaSuccess) note_launches(1);
  return e;
}

template <int DC>
cudaError_t launch_attn_g(AttnParams& p, const DeviceInfo& dev, cudaStream_t stream) {
  switch (p.G) {
    case 1: return launch_attn_t<DC, 1>(p, dev, stream);
    case 2: return launch_attn_t<DC, 2>(p, dev, stream);
    case 4: return launch_attn_t<DC, 4>(p, dev, stream);
    case 8: return launch_attn_t<DC, 8>(p, dev, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool attn_shape_ok(int H, int H_kv, int D) {
  if (H < 1 || H_kv < 1 || H % H_kv != 0) return false;
  const int G = H / H_kv;
  return (D == 64 || D == 96 || D == 128) && (G == 1 || G == 2 || G == 4 || G == 8);
}

AttnLayout attn_layout(int64_t B, int H, int H_kv, int D) {
  AttnLayout z;
  const int64_t segs = B * H_kv;
  const int G = H / H_kv;
  z.counters = 256;
  z.partials = (z.counters + (size_t)segs * 4 + 255) / 256 * 256;
  z.total = z.partials + (size_t)(kAttnMaxCtas + segs) * G * (2 + D) * sizeof(float);
  return z;
}

cudaError_t launch_attn_decode(const void* q, const void* k_new, const void* v_new, void* k_cache,
                               void* v_cache, const int32_t* pos, int64_t B, int H, int H_kv,
                               int D, int64_t n_max, int n_ctx, float theta, float* out,
                               void* workspace, const DeviceInfo& dev, cudaStream_t stream) {
  const AttnLayout z = attn_layout(B, H, H_kv, D);
  AttnParams p = {};
  p.q = (const __nv_bfloat16*)q;
  p.k_new = (const __nv_bfloat16*)k_new;
  p.v_new = (const __nv_bfloat16*)v_new;
  p.k_cache = (__nv_bfloat16*)k_cache;
  p.v_cache = (__nv_bfloat16*)v_cache;
  p.pos = pos;
  p.out = out;
  p.counters = (uint32_t*)((char*)workspace + z.counters);
  p.partials = (float*)((char*)workspace + z.partials);
  p.ctl.status = (uint32_t*)workspace;
  p.ctl.wait_ns = wait_timeout_ns();
  p.ctl.drop_last = fault_injection();
  p.B = (int)B;
  p.H = H;
  p.H_kv = H_kv;
  p.D = D;
  p.G = H / H_kv;
  p.n_max = n_max;
  p.n_ctx = n_ctx;
  for (int i = 0; i < D / 2; ++i) p.inv_freq[i] = std::pow((double)theta, -2.0 * i / D);
  p.qscale = (float)(1.4426950408889634 / std::sqrt((double)D));  // log2(e) / sqrt(D)
  switch (D) {
    case 64: return launch_attn_g<2>(p, dev, stream);
    case 96: return launch_attn_g<3>(p, dev, stream);
    case 128: return launch_attn_g<4>(p, dev, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fmlp
