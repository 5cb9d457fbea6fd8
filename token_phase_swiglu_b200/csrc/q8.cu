// int8 weight streaming for decode batches (1..4 token rows): the MLP block
// on weights stored as int8 with one binary32 scale per group of 64
// consecutive elements of a row (this library's own format: the pages name
// quantized weight streaming over interleaved gate/up rows -- the llama.cpp
// PR #29948 paragraph of "CUDAカーネル融合で推論が最大10%高速化",
// blog.cecily.jp -- but give no block format).  A weight stands for q * s.
//
//   quantize_q8   W bf16 [rows x K] -> q int8 [rows x K], s f32 [rows x K/64]:
//                 s = fl32(max|w| / 127), q = clamp(rint(fl32(w / s)), +-127)
//   q8_stream<GATE = true>   a[m, i] = bf16(SiLU(r g) * r u), g and u the dot
//                 products of x*gamma (f32, exact) with the dequantized gate
//                 and up rows of the packed matrix (interleaved like fmlp_pack's)
//   q8_stream<GATE = false>  out[m, n] = residual + sum_i Wd[n, i] a[m, i]
//
// Both products are HBM-bound GEMVs on the CUDA cores, built like the bf16
// streaming kernels: one CTA per SM, whose producer lane streams groups of
// whole rows (int8 values, then their scales) into a ring of shared-memory
// stages with bulk copies, and 16 consumer warps that share every stage --
// each takes a few of the stage's rows over one column part, so that one
// activation load serves several rows -- and leave their warp-reduced sums
// in shared memory, so no consumer waits for
// another until the phase ends; then each row's parts are summed in a fixed
// order (the result does not depend on timing).  The activations sit in
// shared memory as f32 in a chunk-interleaved order -- element e of 16-byte
// weight chunk c of a 512-element block at [e/4][c][e%4] -- so a lane's 16
// activations are four conflict-free 16-byte loads.  A chunk's dot product is
// taken on the dequantized int8 values with packed f32x2 FMAs and scaled once.
#include "common.cuh"
#include "internal.h"
#include "ring.cuh"

#include <algorithm>
#include <mutex>
#include <set>

namespace fmlp {
namespace {

constexpr int kQ8Group = 64;                         // elements per scale
constexpr int kQ8Consumers = 16;                     // consumer warps
constexpr int kQ8Threads = (kQ8Consumers + 1) * 32;  // warp 0 produces
constexpr int kQ8BarConsumers = 1;                   // named barrier: consumer-only sync
constexpr size_t kQ8MaxStageBytes = 72 * 1024;  // 16 rows of 4096 with their scales
constexpr int kQ8StaticSlack = 2048;                 // static shared memory of the kernels and slack

// Index of element k in the chunk-interleaved activation layout.
__device__ __forceinline__ int act_index(int k) {
  const int blk = k >> 9, c = (k >> 4) & 31, e = k & 15;
  return (blk << 9) + ((e >> 2) << 7) + (c << 2) + (e & 3);
}

__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// The 16 int8 weights of a 16-byte chunk as eight exact f32 pairs, without
// integer-to-float conversion instructions (a quarter-rate pipe): the byte
// q + 128 (0..255) is placed in the low mantissa bits of the binary32 number
// 2^23, whose unit in the last place is 1, so the word reads 2^23 + q + 128
// exactly, and subtracting 2^23 + 128 (also exact) leaves q.  One byte
// permute per weight and one packed add per pair.
__device__ __forceinline__ void dequant16(const uint4& q, uint64_t w[8]) {
  const uint32_t v[4] = {q.x, q.y, q.z, q.w};
  const uint64_t bias = pk2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t u = v[j] ^ 0x80808080u;  // each byte now q + 128
    const float f0 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540u));
    const float f1 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541u));
    const float f2 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542u));
    const float f3 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543u));
    w[2 * j] = fadd2(pk2(f0, f1), bias);
    w[2 * j + 1] = fadd2(pk2(f2, f3), bias);
  }
}

// ---------------------------------------------------------------------------
// quantization
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quantize_q8_kernel(const __nv_bfloat16* __restrict__ W,
                                                          int64_t groups,
                                                          int8_t* __restrict__ q,
                                                          float* __restrict__ s) {
  grid_launch_dependents();
  grid_dependency_wait();
  const int sub = threadIdx.x & 7;  // 8 lanes per group of 64 (8 bf16 each)
  const int64_t team0 = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 3;
  const int64_t teams = ((int64_t)gridDim.x * blockDim.x) >> 3;
  for (int64_t g = team0; g < groups; g += teams) {
    const uint4 v = ld_keep(W + g * kQ8Group + sub * 8);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    float w[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      w[2 * e] = bf16lo(wv[e]);
      w[2 * e + 1] = bf16hi(wv[e]);
    }
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(w[e]));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float sc = __fdiv_rn(m, 127.0f);
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      int qi = 0;
      if (sc > 0.f) qi = min(127, max(-127, __float2int_rn(__fdiv_rn(w[e], sc))));
      packed[e >> 2] |= ((uint32_t)(qi & 0xff)) << ((e & 3) * 8);
    }
    reinterpret_cast<uint2*>(q + g * kQ8Group)[sub] = make_uint2(packed[0], packed[1]);
    if (sub == 0) s[g] = sc;
  }
}

// ---------------------------------------------------------------------------
// streaming GEMVs
// ---------------------------------------------------------------------------
struct Q8Params {
  const __nv_bfloat16* x;
  const __nv_bfloat16* gamma;
  const __nv_bfloat16* residual;
  __nv_bfloat16* a;         // [M x I] intermediate
  float* out;               // [M x d]
  __nv_bfloat16* out_bf16;  // [M x d] or null
  const int8_t* q;          // the phase's int8 rows: packed gate/up [2I x d], or W_down [d x I]
  const float* s;           // their scales, K/64 per row
  Control ctl;
  float eps;
  int M, d, I, T;
  int K;                    // row length: d (gate-up) or I (down)
  int R;                    // rows per stage: gate-up G gate rows then their G up rows (R = 2G)
  int rw;                   // rows of a stage per consumer warp (divides R, <= q8_rows_per_warp)
  int groups;               // stages in the phase: I / G (gate-up) or d / R (down)
  int stages, stage_bytes;
};

// Stage layout: R rows of K int8, then R rows of K/64 scales.
__host__ __device__ constexpr size_t q8_stage_bytes(int R, int K) {
  return align128((size_t)R * K + (size_t)R * (K / kQ8Group) * sizeof(float));
}


template <bool GATE>
__device__ void q8_produce(Producer& pr, const Q8Params& p, int g0, int ng) {
  const int K = p.K, gpr = K / kQ8Group, R = p.R;
  for (int j = 0; j < ng; ++j) {
    if (!pr.acquire()) return;
    const int slot = pr.k % pr.ring.stages;
    uint8_t* buf = pr.ring.buf(slot);
    uint8_t* sbuf = buf + (size_t)R * K;
    uint64_t* bar = &pr.ring.full[slot];
    mbar_arrive_expect_tx(bar, (uint32_t)((size_t)R * K + (size_t)R * gpr * 4));
    if (GATE) {
      const int G = R / 2;
      const int64_t gr = gate_row((g0 + j) * G, p.T), ur = gr + p.T;
      const uint32_t rb = (uint32_t)(G * K), sb = (uint32_t)(G * gpr * 4);
      bulk_copy_g2s(buf, p.q + gr * K, rb, bar, pr.pol);
      bulk_copy_g2s(buf + rb, p.q + ur * K, rb, bar, pr.pol);
      bulk_copy_g2s(sbuf, p.s + gr * gpr, sb, bar, pr.pol);
      bulk_copy_g2s(sbuf + sb, p.s + ur * gpr, sb, bar, pr.pol);
    } else {
      const int64_t n = (int64_t)(g0 + j) * R;
      bulk_copy_g2s(buf, p.q + n * K, (uint32_t)(R * K), bar, pr.pol);
      bulk_copy_g2s(sbuf, p.s + n * gpr, (uint32_t)(R * gpr * 4), bar, pr.pol);
    }
    ++pr.k;
  }
}

// Rows of a stage that one consumer warp takes at the same columns: each
// activation load from shared memory then serves that many rows (2 for 3-4
// token rows, whose activations and accumulators take more registers).
template <int MT>
__host__ __device__ constexpr int q8_rows_per_warp() { return MT <= 2 ? 4 : 2; }
static_assert(q8_rows_per_warp<1>() == 4 && q8_rows_per_warp<3>() == 2, "q8_part_bytes agrees");

// Column parts per row of a stage of R rows: the kQ8Consumers warps take rw
// rows each, so R / rw warps span the rows once and each row is split
// kQ8Consumers rw / R ways.
__host__ __device__ constexpr int q8_parts(int R, int rw) { return kQ8Consumers * rw / R; }
// Bytes of the consumers' sums per CTA: every warp leaves rw <= RW row sums
// per token row per stage.
__host__ __device__ constexpr size_t q8_part_bytes(int max_groups, int mt) {
  return align128((size_t)max_groups * kQ8Consumers * (mt <= 2 ? 4 : 2) * mt * sizeof(float));
}

// Consumer warp c takes rows [r0, r0 + rw) of every stage (rw <= RW),
// r0 = rw (c % (R / rw)), and chunks [c0, c1) of them: part c / (R / rw) of
// the rows' kQ8Consumers rw / R column parts.  Leaves each stage's sums in
// part[((j R + r) parts + part) MT + m].
template <int MT>
__device__ bool q8_consume(Consumer& cs, const Q8Params& p, int ng, const float* act,
                           float* part) {
  constexpr int RW = q8_rows_per_warp<MT>();
  const int c = (threadIdx.x >> 5) - 1, lane = cs.lane;
  const int R = p.R, rw = p.rw, groups_r = R / rw, parts = q8_parts(R, rw);
  const int r0 = rw * (c % groups_r), pt = c / groups_r;
  const int K = p.K, nc = K / 16, gpr = K / kQ8Group;
  const int c0 = pt * nc / parts, c1 = (pt + 1) * nc / parts;
  for (int j = 0; j < ng; ++j) {
    const uint8_t* buf = cs.wait_full();
    if (!buf) return false;
    const uint8_t* wrow = buf + (size_t)r0 * K;
    const float* srow = reinterpret_cast<const float*>(buf + (size_t)R * K) + r0 * gpr;
    uint64_t acc[RW][MT];
#pragma unroll
    for (int rr = 0; rr < RW; ++rr)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[rr][m] = 0ull;
    for (int ch = c0 + lane; ch < c1; ch += 32) {
      const float* ab = act + ((ch >> 5) << 9) + ((ch & 31) << 2);
      if constexpr (MT <= 2) {
        // activations of every token row first, then one row's weights at a time
        float4 a4[MT][4];
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            a4[m][jj] = *reinterpret_cast<const float4*>(ab + m * K + (jj << 7));
#pragma unroll
        for (int rr = 0; rr < RW; ++rr) {
          if (rr < rw) {
            uint64_t w[8];
            dequant16(lds128(wrow + (size_t)rr * K + 16 * ch), w);
            const float sc = srow[rr * gpr + (ch >> 2)];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              uint64_t t = 0ull;
#pragma unroll
              for (int jj = 0; jj < 4; ++jj) {
                t = ffma2(w[2 * jj], pk2(a4[m][jj].x, a4[m][jj].y), t);
                t = ffma2(w[2 * jj + 1], pk2(a4[m][jj].z, a4[m][jj].w), t);
              }
              acc[rr][m] = ffma2(t, pk2(sc, sc), acc[rr][m]);
            }
          }
        }
      } else {
        // the rows' weights first, then one token row's activations at a time
        uint64_t w[RW][8];
        float sc[RW];
#pragma unroll
        for (int rr = 0; rr < RW; ++rr) {
          if (rr < rw) {
            dequant16(lds128(wrow + (size_t)rr * K + 16 * ch), w[rr]);
            sc[rr] = srow[rr * gpr + (ch >> 2)];
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          float4 a4[4];
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            a4[jj] = *reinterpret_cast<const float4*>(ab + m * K + (jj << 7));
#pragma unroll
          for (int rr = 0; rr < RW; ++rr) {
            if (rr < rw) {
              uint64_t t = 0ull;
#pragma unroll
              for (int jj = 0; jj < 4; ++jj) {
                t = ffma2(w[rr][2 * jj], pk2(a4[jj].x, a4[jj].y), t);
                t = ffma2(w[rr][2 * jj + 1], pk2(a4[jj].z, a4[jj].w), t);
              }
              acc[rr][m] = ffma2(t, pk2(sc[rr], sc[rr]), acc[rr][m]);
            }
          }
        }
      }
    }
    cs.release();
#pragma unroll
    for (int rr = 0; rr < RW; ++rr) {
      if (rr < rw) {
        float* dst = part + ((j * R + r0 + rr) * parts + pt) * MT;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const float v = warp_sum(hsum2(acc[rr][m]));
          if (lane == 0) dst[m] = v;
        }
      }
    }
  }
  return true;
}

// x * gamma (exact in f32) for the token rows into the interleaved layout,
// rows >= mt zero; returns 1/RMS of each row.  Consumer threads.
template <int MT>
__device__ void q8_stage_x(const Q8Params& p, int mt, float* act, float (*red)[MT],
                           float* rinv) {
  const int d = p.d, ct = threadIdx.x - 32, lane = threadIdx.x & 31, c = (threadIdx.x >> 5) - 1;
  float ss[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) ss[m] = 0.f;
  for (int v = ct; v < d / 8; v += kQ8Consumers * 32) {
    const uint4 gv = ld_keep(p.gamma + (int64_t)v * 8);
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      uint4 xv = make_uint4(0, 0, 0, 0);
      if (m < mt) xv = ld_keep(p.x + (int64_t)m * d + (int64_t)v * 8);
      const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = bf16lo(xw[e]), x1 = bf16hi(xw[e]);
        ss[m] = fmaf(x0, x0, ss[m]);
        ss[m] = fmaf(x1, x1, ss[m]);
        act[m * d + act_index(v * 8 + 2 * e)] = x0 * bf16lo(gw[e]);
        act[m * d + act_index(v * 8 + 2 * e + 1)] = x1 * bf16hi(gw[e]);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const float t = warp_sum(ss[m]);
    if (lane == 0) red[c][m] = t;
  }
  named_barrier_sync(kQ8BarConsumers, kQ8Consumers * 32);
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kQ8Consumers; ++w) t += red[w][m];
    rinv[m] = 1.0f / sqrtf(t / (float)d + p.eps);
  }
}

// a (bf16) as f32 into the interleaved layout, rows >= mt zero.  Consumer
// threads; each issues the loads of several vectors before storing any.
template <int MT>
__device__ void q8_stage_a(const Q8Params& p, int mt, float* act) {
  constexpr int V = MT <= 2 ? 4 : 2;
  const int I = p.I, ct = threadIdx.x - 32, nv = I / 8;
  for (int v0 = ct; v0 < nv; v0 += V * kQ8Consumers * 32) {
    uint4 av[V][MT];
#pragma unroll
    for (int u = 0; u < V; ++u)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const int v = v0 + u * kQ8Consumers * 32;
        av[u][m] = make_uint4(0, 0, 0, 0);
        if (v < nv && m < mt) av[u][m] = ld_keep(p.a + (int64_t)m * I + (int64_t)v * 8);
      }
#pragma unroll
    for (int u = 0; u < V; ++u) {
      const int v = v0 + u * kQ8Consumers * 32;
      if (v >= nv) break;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const uint32_t aw[4] = {av[u][m].x, av[u][m].y, av[u][m].z, av[u][m].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          act[m * I + act_index(v * 8 + 2 * e)] = bf16lo(aw[e]);
          act[m * I + act_index(v * 8 + 2 * e + 1)] = bf16hi(aw[e]);
        }
      }
    }
  }
  named_barrier_sync(kQ8BarConsumers, kQ8Consumers * 32);
}

template <int MT, bool GATE>
__global__ void __launch_bounds__(kQ8Threads, 1) q8_stream(const __grid_constant__ Q8Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ float red[kQ8Consumers][MT];
  __shared__ CtaState st;

  const int mt = min(MT, p.M);
  const size_t act_bytes = align128((size_t)MT * p.K * sizeof(float));
  const int max_groups = (p.groups + gridDim.x - 1) / gridDim.x;
  Ring ring;
  ring.full = reinterpret_cast<uint64_t*>(smem);
  ring.empty = ring.full + kMaxStages;
  float* act = reinterpret_cast<float*>(smem + kHeader);
  float* part = reinterpret_cast<float*>(smem + kHeader + act_bytes);
  ring.stage0 = smem + kHeader + act_bytes + q8_part_bytes(max_groups, MT);
  ring.stages = p.stages;
  ring.stage_bytes = p.stage_bytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int g0 = 0, ng = 0;
  split_groups(p.groups, blockIdx.x, gridDim.x, false, g0, ng);

  if (threadIdx.x == 0) init_ring(ring, st, kQ8Consumers);
  __syncthreads();
  grid_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      Producer pr{ring, &st, p.ctl, evict_first_policy(), ng};
      q8_produce<GATE>(pr, p, g0, ng);
      st.issued = pr.k;
    }
    __syncwarp();
  } else {
    grid_dependency_wait();  // x or a may be written by the previous kernel
    Consumer cs{ring, &st, p.ctl, 0, lane};
    const int ct = threadIdx.x - 32;
    if (GATE) {
      float rinv[MT];
      q8_stage_x<MT>(p, mt, act, red, rinv);
      const bool ok = q8_consume<MT>(cs, p, ng, act, part);
      if (!consumer_barrier_any<kQ8Consumers * 32>(kQ8BarConsumers, !ok)) {
        const int G = p.R / 2, parts = q8_parts(p.R, p.rw);
        for (int i = ct; i < ng * G; i += kQ8Consumers * 32) {
          const int j = i / G, gp = i - j * G;
          const float* pg = part + ((j * p.R + gp) * parts) * MT;
          const float* pu = part + ((j * p.R + G + gp) * parts) * MT;
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            if (m >= mt) continue;
            float g = 0.f, u = 0.f;
            for (int q = 0; q < parts; ++q) {
              g += pg[q * MT + m];
              u += pu[q * MT + m];
            }
            p.a[(int64_t)m * p.I + (int64_t)g0 * G + i] =
                __float2bfloat16_rn(silu_mul(g * rinv[m], u * rinv[m]));
          }
        }
      }
    } else {
      q8_stage_a<MT>(p, mt, act);
      const bool ok = q8_consume<MT>(cs, p, ng, act, part);
      if (!consumer_barrier_any<kQ8Consumers * 32>(kQ8BarConsumers, !ok)) {
        const int parts = q8_parts(p.R, p.rw);
        for (int i = ct; i < ng * p.R; i += kQ8Consumers * 32) {
          const int64_t n = (int64_t)g0 * p.R + i;
          const float* pr = part + (i * parts) * MT;
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            if (m >= mt) continue;
            float o = 0.f;
            for (int q = 0; q < parts; ++q) o += pr[q * MT + m];
            if (p.residual) o += __bfloat162float(p.residual[(int64_t)m * p.d + n]);
            if (p.out_bf16) p.out_bf16[(int64_t)m * p.d + n] = __float2bfloat16_rn(o);
            else p.out[(int64_t)m * p.d + n] = o;
          }
        }
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && st.abort) drain_ring(ring, st.issued);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct Q8Plan {
  int R = 0, rw = 0, stages = 0, groups = 0;
  size_t stage_bytes = 0, smem = 0;
};

// Rows of a stage per consumer warp: the largest rw <= rw_max (each
// activation load then serves rw rows) among those that keep the most lanes
// busy -- a row of nc 16-byte chunks is split into 16 rw / R parts, one
// chunk per lane at a time, so a part of 48 chunks leaves a quarter of the
// lanes idle on its second pass.
int q8_choose_rw(int R, int nc, int rw_max) {
  int best = 1;
  double best_eff = -1.0;
  for (int rw = std::min(rw_max, R); rw >= 1; rw /= 2) {
    const int parts = q8_parts(R, rw);
    const int longest = (nc + parts - 1) / parts;
    const double eff = (double)nc / parts / (32.0 * ((longest + 31) / 32));
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = rw;
    }
  }
  return best;
}

// Rows per stage and ring depth for one phase: the largest stage (at most
// 72 KB; the number of copies, more than their bytes, limits a bulk-copy
// ring) that leaves a ring of at least three stages beside the activations
// and the consumers' sums.
Q8Plan q8_plan(int64_t M, int64_t d, int64_t I, int T, bool gate, const DeviceInfo& dev) {
  const size_t budget = (size_t)dev.max_smem_optin - kQ8StaticSlack;
  const int K = (int)(gate ? d : I);
  const int sms = std::max(1, dev.sm_count);
  for (int R = 16; R >= (gate ? 2 : 1); R /= 2) {
    if (gate ? (T % (R / 2) != 0) : (d % R != 0)) continue;
    Q8Plan pl;
    pl.R = R;
    pl.groups = (int)(gate ? I / (R / 2) : d / R);
    pl.stage_bytes = q8_stage_bytes(R, K);
    if (pl.stage_bytes > kQ8MaxStageBytes) continue;
    const int grid = std::min(pl.groups, sms);
    const size_t fixed = kHeader + align128((size_t)M * K * sizeof(float)) +
                         q8_part_bytes((pl.groups + grid - 1) / grid, (int)M);
    if (fixed >= budget) return Q8Plan();
    const size_t fit = (budget - fixed) / pl.stage_bytes;
    if (fit < 3) continue;
    pl.stages = (int)std::min<size_t>(kMaxStages, fit);
    pl.smem = fixed + (size_t)pl.stages * pl.stage_bytes;
    pl.rw = q8_choose_rw(R, K / 16, M <= 2 ? 4 : 2);
    return pl;
  }
  return Q8Plan();
}

template <typename Kernel>
cudaError_t allow_q8_smem(Kernel k, const DeviceInfo& dev) {
  static std::mutex mu;
  static std::set<std::pair<int, const void*>> done;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(dev.device, (const void*)k);
  if (done.count(key)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       dev.max_smem_optin - kQ8StaticSlack);
  if (e == cudaSuccess) done.insert(key);
  return e;
}

template <int MT, bool GATE>
cudaError_t launch_phase(Q8Params p, const Q8Plan& pl, const DeviceInfo& dev,
                         cudaStream_t stream) {
  auto k = q8_stream<MT, GATE>;
  cudaError_t e = allow_q8_smem(k, dev);
  if (e != cudaSuccess) return e;
  p.R = pl.R;
  p.rw = pl.rw;
  p.groups = pl.groups;
  p.stages = pl.stages;
  p.stage_bytes = (int)pl.stage_bytes;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::min(pl.groups, dev.sm_count));
  cfg.blockDim = dim3(kQ8Threads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, k, p);
  if (e == cudaSuccess) note_launches(1);
  return e;
}

template <int MT>
cudaError_t launch_both(Q8Params p, const Q8Plan& pg, const Q8Plan& pd, const void* Pq,
                        const float* Ps, const void* Wdq, const float* Wds,
                        const DeviceInfo& dev, cudaStream_t stream) {
  p.q = (const int8_t*)Pq;
  p.s = Ps;
  p.K = p.d;
  cudaError_t e = launch_phase<MT, true>(p, pg, dev, stream);
  if (e != cudaSuccess) return e;
  p.q = (const int8_t*)Wdq;
  p.s = Wds;
  p.K = p.I;
  return launch_phase<MT, false>(p, pd, dev, stream);
}

}  // namespace

bool q8_supported(int64_t M, int64_t d, int64_t I, int T, const DeviceInfo& dev) {
  if (M < 1 || M > 4 || d % 512 != 0 || I % 512 != 0 || T <= 0 || T % 8 != 0 || I % T != 0)
    return false;
  return q8_plan(M, d, I, T, true, dev).R > 0 && q8_plan(M, d, I, T, false, dev).R > 0;
}

cudaError_t launch_quantize_q8(const void* W, int64_t rows, int64_t K, void* q, float* s,
                               const DeviceInfo& dev, cudaStream_t stream) {
  const int64_t groups = rows * K / kQ8Group;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::max<int64_t>(
      1, std::min<int64_t>((groups * 8 + 255) / 256, 8 * dev.sm_count)));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaError_t e = cudaLaunchKernelEx(&cfg, quantize_q8_kernel, (const __nv_bfloat16*)W, groups,
                                     (int8_t*)q, s);
  if (e == cudaSuccess) note_launches(1);
  return e;
}

cudaError_t launch_forward_q8(const void* x, int64_t M, const void* gamma, float eps,
                              const void* Pq, const float* Ps, int T, const void* Wdq,
                              const float* Wds, int64_t d, int64_t I, const void* residual,
                              float* out, void* out_bf16, void* a, uint32_t* status,
                              const DeviceInfo& dev, cudaStream_t stream) {
  const Q8Plan pg = q8_plan(M, d, I, T, true, dev), pd = q8_plan(M, d, I, T, false, dev);
  if (!pg.R || !pd.R) return cudaErrorInvalidValue;
  Q8Params p = {};
  p.x = (const __nv_bfloat16*)x;
  p.gamma = (const __nv_bfloat16*)gamma;
  p.residual = (const __nv_bfloat16*)residual;
  p.a = (__nv_bfloat16*)a;
  p.out = out;
  p.out_bf16 = (__nv_bfloat16*)out_bf16;
  p.ctl.status = status;
  p.ctl.wait_ns = wait_timeout_ns();
  p.ctl.drop_last = fault_injection();
  p.eps = eps;
  p.M = (int)M;
  p.d = (int)d;
  p.I = (int)I;
  p.T = T;
  switch (M) {
    case 1: return launch_both<1>(p, pg, pd, Pq, Ps, Wdq, Wds, dev, stream);
    case 2: return launch_both<2>(p, pg, pd, Pq, Ps, Wdq, Wds, dev, stream);
    case 3: return launch_both<3>(p, pg, pd, Pq, Ps, Wdq, Wds, dev, stream);
    default: return launch_both<4>(p, pg, pd, Pq, Ps, Wdq, Wds, dev, stream);
  }
}

}  // namespace fmlp
