// Tensor-core path (tcgen05 / TMEM) for token counts above the decode range.
//
// The gate-up contraction and the down projection of the MLP block
// ("FastTPS: An Optimized Method for LLM Token Phase for AI Accelerators",
// xllm-io review, section 三 Eq(1), Figure 4) as swap-AB GEMMs:
//
//     D[r, n] = sum_k A[r, k] B[n, k]
//
// with the weights as A (128 rows per MMA tile, M of the MMA) and the token
// rows as B (N of the MMA, 16..256).  For the gate-up step B holds, per token
// tile of Mt tokens, the rows hi(x*gamma) then lo(x*gamma): x*gamma has at
// most 16 significant bits, so hi + lo (two bf16) is exact and the MMA sees
// the activations at f32 precision; the epilogue adds the two halves of D.
// r = 1/RMS is applied in the epilogue, as in the CUDA-core path.
//
// Per CTA (one per SM, 192 threads):
//   warp 0     TMA producer: one 16 KB A box + one B box per 64-wide k-block
//              into a ring of shared-memory stages (128-byte swizzle);
//   warp 1     TMEM owner and MMA issuer (tcgen05.mma kind::f16, f32
//              accumulators double-buffered in TMEM, tcgen05.commit frees
//              stages and publishes accumulators);
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//              lanes 32*(w%4)..+31), SwiGLU and stores of a (gate-up), or
//              red.add of the tile into out (down).
// Work is split in data-parallel rounds of whole tiles and a "stream-K"
// remainder (see the schedule below).  A gate-up tile shared by several CTAs
// is finished by the last contributor from the others' partials (SwiGLU is
// not linear); down-projection shares are simply added into out, which the
// prologue set to the residual or zero.  Nobody waits on another CTA.
// Every mbarrier wait is bounded; on expiry the CTA flags the status word,
// waits for its own copies and MMAs, frees its TMEM and returns.
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

constexpr int kTcThreads = 192;
constexpr int kMaxStages = 12;
constexpr uint64_t kDrainNs = 1000000000ull;
// Pair kernel teardown: a stage one CTA issued but the leader never armed
// never completes; its copies land within microseconds, so a short limit.
constexpr uint64_t kPairDrainNs = 2000000ull;

enum Epi { kEpiSwiGLU = 0, kEpiDown = 1 };

// ---------------------------------------------------------------------------
// Schedule (Sched in tcgen05.cuh): data-parallel rounds, then stream-K.
// ---------------------------------------------------------------------------
// Segment s of this CTA's work: tile t, stages [kb0, kb1).  Segments
// 0..dp-1 are the whole tiles of the data-parallel rounds; then the
// stream-K range [u0, u1).  With a split schedule, segment s is item
// s * ctas + this CTA.  Returns false past the end.
__device__ __forceinline__ bool segment(const Sched& S, int64_t u0, int64_t u1, int s, int& t,
                                        int& kb0, int& kb1) {
  if (S.split) return s < S.dp && S.split_item(s * S.ctas + (int)blockIdx.x, t, kb0, kb1);
  if (s < S.dp) {
    t = s * S.ctas + (int)blockIdx.x;
    kb0 = 0;
    kb1 = S.KB;
    return true;
  }
  s -= S.dp;
  if (u0 >= u1) return false;
  const int t0 = (int)(u0 / S.KB);
  const int tl = t0 + s;
  const int64_t tb = (int64_t)tl * S.KB;
  if (tb >= u1) return false;
  t = S.sk_tile0() + tl;
  kb0 = (int)(max(u0, tb) - tb);
  kb1 = (int)(min(u1, tb + S.KB) - tb);
  return true;
}

// ---------------------------------------------------------------------------
// Kernel
// ---------------------------------------------------------------------------
struct TcParams {
  CUtensorMap a_map;   // A [rows x K] bf16, box 64 x 128, 128-byte swizzle
  CUtensorMap b_map;   // B [token-tile rows x K] bf16, box 64 x N, 128-byte swizzle
  Sched sched;
  int epi;             // kEpiSwiGLU or kEpiDown
  int N;               // MMA N (columns of D)
  int Mt;              // tokens per token tile
  int M;               // tokens
  int rows;            // valid A rows (2I packed rows, or d)
  int T;               // interleave tile (SwiGLU)
  int I, d;
  int C;               // accumulator chains per tile: MMA k-slice j goes to chain j % C
  int KS;              // k-blocks per stage (one 3-D copy of A and one of B)
  int KBtot;           // k-blocks of K
  int stages, stage_bytes, a_bytes, b_bytes;
  uint32_t tmem_cols;  // allocated TMEM columns (2 x C x N rounded up to a power of two)
  const float* rinv;   // [M] 1/RMS per token (SwiGLU)
  __nv_bfloat16* a_out;             // SwiGLU output a [M x I]
  float* out;                       // down output [M x d] (accumulated into)
  float* partials;     // [ctas][2][N][128] f32
  uint32_t* counters;  // [tiles] arrivals (zero between calls)
  uint32_t* status;
  uint64_t wait_ns;
  int drop_last;
};

struct TcShared {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t mma_done;   // abort path: all issued MMAs have completed
  uint32_t tmem_base;
  int abort;
  int last;
  int head_done;       // the other contributor of this CTA's last gate-up tile has arrived
  int k_issued;        // stages issued by the producer
  float rinv_s[2][kBM];  // 1/RMS of the token tile of each accumulator buffer (SwiGLU)
};

__device__ __forceinline__ void tc_flag(TcShared* sh, uint32_t* status) {
  sh->abort = 1;
  atomicOr(status, kStatusTimeout);
}

// SiLU(g) * u with the hardware exp2 and reciprocal approximations.  Their
// relative error (a few 1e-7) is far below the bf16 rounding of a that
// follows (2^-9), and the exact rows (shared memory).
template <int CW>
__device__ __forceinline__ void epilogue_columns(const TcParams& p, int tt, int row,
                                                 const float (&vals)[CW], int col0,
                                                 const float* rv) {
  // SwiGLU: within a 2T-row interleave tile rows [0,T) are gate, [T,2T) up;
  // the partner row is lane ^ T (T in {8, 16}).  The gate lane finishes the
  // first half of the chunk's tokens, the up lane the second half.
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
  const int loc0 = col0 + (is_gate ? 0 : H), tok0 = tt * p.Mt + loc0;
  if (row < p.rows && pair < p.I) {
#pragma unroll
    for (int j = 0; j < H; ++j) {
      const int m = tok0 + j;
      if (m < p.M) {
        const float r = rv[loc0 + j];
        p.a_out[(int64_t)m * p.I + pair] = __float2bfloat16_rn(silu_mul_fast(g[j] * r, u[j] * r));
      }
    }
  }
}

// Load CW columns at `col` of the tile's accumulator: the sum of its C chains.
template <int CW>
__device__ __forceinline__ void tile_cols(const TcParams& p, uint32_t tb, int col, float (&v)[CW]) {
  uint32_t r[CW];
  tmem_ld<CW>(tb + col, r);
  tmem_wait();
#pragma unroll
  for (int j = 0; j < CW; ++j) v[j] = __uint_as_float(r[j]);
  for (int c = 1; c < p.C; ++c) {
    tmem_ld<CW>(tb + (uint32_t)(c * p.N) + col, r);
    tmem_wait();
#pragma unroll
    for (int j = 0; j < CW; ++j) v[j] += __uint_as_float(r[j]);
  }
}

// Finish a tile: its accumulator (hi + lo for SwiGLU) plus the other
// contributors' partials, CW logical columns at a time, then the epilogue.
template <int CW>
__device__ void finish_tile(const TcParams& p, int t, uint32_t tb, bool whole, int c_first,
                            int c_last, int r_local, const float* rv) {
  const int ncol = p.epi == kEpiSwiGLU ? p.Mt : p.N;
  const int rt = t / p.sched.ntok, tt = t % p.sched.ntok;
  const int row = rt * kBM + r_local;
  for (int c0 = 0; c0 < ncol; c0 += CW) {
    float vals[CW];
#pragma unroll
    for (int j = 0; j < CW; ++j) vals[j] = 0.f;
    if (!whole) {
      // the other contributors' partials first: their L2 round trip
      // overlaps the accumulator reads below
      for (int cc = c_first; cc <= c_last; ++cc) {
        if (cc == (int)blockIdx.x) continue;
        int64_t cu0, cu1;
        p.sched.range(cc, cu0, cu1);
        const int slot = (t == p.sched.sk_tile0() + (int)(cu0 / p.sched.KB)) ? 0 : 1;
        const float* part = p.partials + ((size_t)cc * 2 + slot) * (size_t)p.N * kBM;
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          vals[j] += __ldcg(part + (size_t)(c0 + j) * kBM + r_local);
          if (p.epi == kEpiSwiGLU) vals[j] += __ldcg(part + (size_t)(p.Mt + c0 + j) * kBM + r_local);
        }
      }
    }
    float acc[CW];
    tile_cols<CW>(p, tb, c0, acc);
#pragma unroll
    for (int j = 0; j < CW; ++j) vals[j] += acc[j];
    if (p.epi == kEpiSwiGLU) {
      tile_cols<CW>(p, tb, p.Mt + c0, acc);  // lo half of x*gamma
#pragma unroll
      for (int j = 0; j < CW; ++j) vals[j] += acc[j];
    }
    epilogue_columns<CW>(p, tt, row, vals, c0, rv);
  }
}

// Down GEMM: add this CTA's accumulator of tile t (all C chains) into out.
template <int CW>
__device__ void add_tile_to_out(const TcParams& p, int t, uint32_t tb, int r_local) {
  const int rt = t / p.sched.ntok, tt = t % p.sched.ntok;
  const int n = rt * kBM + r_local;
  for (int c0 = 0; c0 < p.N; c0 += CW) {
    float v[CW];
    tile_cols<CW>(p, tb, c0, v);
    if (n < p.d) {
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        const int m = tt * p.Mt + c0 + j;
        if (m < p.M) atomicAdd(p.out + (int64_t)m * p.d + n, v[j]);
      }
    }
  }
}

__global__ void __launch_bounds__(kTcThreads, 1) tc_gemm(const __grid_constant__ TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ TcShared sh;
  // stages start at a 1024-byte boundary (128-byte swizzle atoms)
  uint8_t* stage0 = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int64_t u0, u1;
  p.sched.range(blockIdx.x, u0, u1);
  int nseg = 0, nk = 0;
  {
    int t, a, b;
    while (segment(p.sched, u0, u1, nseg, t, a, b)) {
      nk += b - a;
      ++nseg;
    }
  }

  if (threadIdx.x == 0) {
    for (int j = 0; j < p.stages; ++j) {
      mbar_init(&sh.full[j], 1);
      mbar_init(&sh.empty[j], 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(&sh.acc_full[j], 1);
      mbar_init(&sh.acc_empty[j], 4);
    }
    mbar_init(&sh.mma_done, 1);
    sh.abort = 0;
    sh.k_issued = 0;
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
    // ---------------- TMA producer ----------------
    // The weights (A) do not depend on the previous kernel: the first ring's
    // worth of A tiles is requested before the dependency wait; the
    // activations (B) only after it.
    if (lane == 0) {
      const uint64_t pol_a = evict_first_policy();
      uint64_t pol_b;
      asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol_b));
      const int brow_mul = p.epi == kEpiSwiGLU ? 2 * p.Mt : p.Mt;
      int early_kb[kMaxStages], early_tt[kMaxStages];
      const int n_early = min(nk, p.stages) - (p.drop_last && nk <= p.stages ? 1 : 0);
      int k = 0;
      bool ok = true;
      for (int s = 0; s < nseg && ok && !*abort; ++s) {
        int t, kb0, kb1;
        segment(p.sched, u0, u1, s, t, kb0, kb1);
        const int rt = t / p.sched.ntok, tt = t % p.sched.ntok;
        for (int kb = kb0; kb < kb1; ++kb, ++k) {
          if (p.drop_last && k == nk - 1) {
            ok = false;
            break;
          }
          const int slot = k % p.stages;
          uint8_t* a_dst = stage0 + (size_t)slot * p.stage_bytes;
          uint8_t* b_dst = a_dst + p.a_bytes;
          if (k >= p.stages) {
            if (k == p.stages) {
              // activations of the early stages, now that they are written
              grid_dependency_wait();
              for (int e = 0; e < n_early; ++e)
                tma_load_3d(stage0 + (size_t)e * p.stage_bytes + p.a_bytes, &p.b_map, 0,
                            early_tt[e] * brow_mul, early_kb[e] * p.KS, &sh.full[e], pol_b);
            }
            if (!mbar_wait_bounded(&sh.empty[slot], (uint32_t)(((k / p.stages) - 1) & 1),
                                   p.wait_ns, abort)) {
              tc_flag(&sh, p.status);
              ok = false;
              break;
            }
          }
          mbar_arrive_expect_tx(&sh.full[slot], (uint32_t)(p.a_bytes + p.b_bytes));
          tma_load_3d(a_dst, &p.a_map, 0, rt * kBM, kb * p.KS, &sh.full[slot], pol_a);
          if (k < p.stages) {
            early_kb[k] = kb;
            early_tt[k] = tt;
          } else {
            tma_load_3d(b_dst, &p.b_map, 0, tt * brow_mul, kb * p.KS, &sh.full[slot], pol_b);
          }
          sh.k_issued = k + 1;
        }
      }
      if (k <= p.stages && k > 0) {
        // the whole range fit in the first ring: its activations are still owed
        grid_dependency_wait();
        for (int e = 0; e < k; ++e)
          tma_load_3d(stage0 + (size_t)e * p.stage_bytes + p.a_bytes, &p.b_map, 0,
                      early_tt[e] * brow_mul, early_kb[e] * p.KS, &sh.full[e], pol_b);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    grid_dependency_wait();  // B is written by the previous kernel
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(p.N);
      int k = 0;
      bool ok = true;
      for (int s = 0; s < nseg && ok; ++s) {
        int t, kb0, kb1;
        segment(p.sched, u0, u1, s, t, kb0, kb1);
        const int buf = s & 1;
        if (!mbar_wait_bounded(&sh.acc_empty[buf], (uint32_t)(((s >> 1) & 1) ^ 1), p.wait_ns,
                               abort)) {
          tc_flag(&sh, p.status);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(buf * p.C * p.N);
        for (int kb = kb0; kb < kb1; ++kb, ++k) {
          const int slot = k % p.stages;
          if (!mbar_wait_bounded(&sh.full[slot], (uint32_t)((k / p.stages) & 1), p.wait_ns,
                                 abort)) {
            tc_flag(&sh, p.status);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(stage0 + (size_t)slot * p.stage_bytes);
          const uint32_t b_addr = a_addr + p.a_bytes;
          const uint32_t b_kblock = (uint32_t)(p.N * kBK * 2);
          // the last stage of K may hold fewer than KS k-blocks (the rest is zero fill)
          const int nkb = min(p.KS, p.KBtot - kb * p.KS);
          for (int kbi = 0; kbi < nkb; ++kbi) {
            // k-slice kk accumulates into chain kk % C: C independent MMA chains
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const int c = kk % p.C;
              const bool first = kb == kb0 && kbi == 0 && kk < p.C;
              mma_bf16(d_tmem + (uint32_t)(c * p.N),
                       sw128_desc(a_addr + (uint32_t)(kbi * kATileBytes) + kk * 32),
                       sw128_desc(b_addr + (uint32_t)kbi * b_kblock + kk * 32), idesc,
                       first ? 0u : 1u);
            }
          }
          mma_commit(&sh.empty[slot]);  // stage reusable once these MMAs finish
        }
        if (ok) mma_commit(&sh.acc_full[buf]);
      }
      // every MMA issued so far has completed once this commit arrives
      mma_commit(&sh.mma_done);
      mbar_wait_bounded(&sh.mma_done, 0, kDrainNs, nullptr);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2-5) ----------------
    const int q = warp & 3;                  // TMEM lane quadrant of this warp
    const int r_local = 32 * q + lane;       // accumulator row = TMEM lane
    const int et = threadIdx.x - 64;         // 0..127
    const int ncol = p.epi == kEpiSwiGLU ? p.Mt : p.N;  // logical columns (hi + lo summed)
    grid_dependency_wait();  // 1/RMS and the initial out come from earlier kernels
    for (int s = 0; s < nseg; ++s) {
      int t, kb0, kb1;
      segment(p.sched, u0, u1, s, t, kb0, kb1);
      const int buf = s & 1;
      // A gate-up tile shared by two CTAs: the one holding its first
      // k-blocks reaches it at the end of its range, long after the other
      // (whose range starts inside it) has stored its partial.  Look at the
      // tile's counter while the MMAs still run: if the other contributor has
      // arrived, this CTA finishes the tile without storing a partial of its
      // own or taking part in the count (the other one has left it).
      bool head_only = false;
      if (p.epi == kEpiSwiGLU && !(kb0 == 0 && kb1 == p.sched.KB) && kb0 == 0) {
        const int64_t tu = (int64_t)(t - p.sched.sk_tile0()) * p.sched.KB;
        if (p.sched.cta_of(tu + p.sched.KB - 1) == (int)blockIdx.x + 1) {
          if (et == 0) sh.head_done = ld_acquire_gpu(p.counters + t) == 1u;
          head_only = true;
        }
      }
      if (p.epi == kEpiSwiGLU) {  // 1/RMS of the token tile, while the MMAs run
        const int tt = t % p.sched.ntok;
        for (int i = et; i < p.Mt; i += 128) {
          const int m = tt * p.Mt + i;
          sh.rinv_s[buf][i] = m < p.M ? __ldg(p.rinv + m) : 0.f;
        }
      }
      const bool got =
          mbar_wait_bounded(&sh.acc_full[buf], (uint32_t)((s >> 1) & 1), p.wait_ns, abort);
      if (!got && lane == 0) tc_flag(&sh, p.status);
      if (epilogue_barrier_any(!got)) break;  // also publishes sh.head_done and sh.rinv_s
      tc_fence_after();
      const uint32_t tb = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * p.C * p.N);
      if (p.epi == kEpiDown) {
        // Split-K by accumulation: out already holds the residual (or zero)
        // and every contributor of a tile adds its share; no partials, no
        // tile counters, nobody waits for the last contributor.
        if (p.N % 32 == 0) add_tile_to_out<32>(p, t, tb, r_local);
        else add_tile_to_out<16>(p, t, tb, r_local);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.acc_empty[buf]);
        continue;
      }
      const bool whole = kb0 == 0 && kb1 == p.sched.KB;
      const int64_t tu = (int64_t)(t - p.sched.sk_tile0()) * p.sched.KB;  // stream-K tiles only
      const int c_first = whole ? 0 : p.sched.cta_of(tu);
      const int c_last = whole ? 0 : p.sched.cta_of(tu + p.sched.KB - 1);
      bool finalize = whole;
      if (head_only && sh.head_done) {
        // the other contributor's partial is visible (acquire above)
        finalize = true;
      } else if (!whole) {
        // this CTA's partial (chains summed): slot 0 if the tile is where its
        // range starts, else 1.  N is a multiple of 16.
        const int slot = (t == p.sched.sk_tile0() + (int)(u0 / p.sched.KB)) ? 0 : 1;
        float* part = p.partials + ((size_t)blockIdx.x * 2 + slot) * (size_t)p.N * kBM;
        int c = 0;
        for (; c + 32 <= p.N; c += 32) {
          float v[32];
          tile_cols<32>(p, tb, c, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) __stcg(part + (size_t)(c + j) * kBM + r_local, v[j]);
        }
        if (c < p.N) {
          float v[16];
          tile_cols<16>(p, tb, c, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) __stcg(part + (size_t)(c + j) * kBM + r_local, v[j]);
        }
        __threadfence();
        named_barrier_sync(1, 128);
        if (et == 0) sh.last = atomicAdd(p.counters + t, 1u) == (uint32_t)(c_last - c_first);
        named_barrier_sync(1, 128);
        finalize = sh.last;
        if (finalize) __threadfence();
      }
      if (finalize) {
        // a chunk width that divides the logical columns (a multiple of 8)
        const float* rv = sh.rinv_s[buf];
        if (ncol % 32 == 0) finish_tile<32>(p, t, tb, whole, c_first, c_last, r_local, rv);
        else if (ncol % 16 == 0) finish_tile<16>(p, t, tb, whole, c_first, c_last, r_local, rv);
        else finish_tile<8>(p, t, tb, whole, c_first, c_last, r_local, rv);
        if (!whole && et == 0) atomicExch(p.counters + t, 0u);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.acc_empty[buf]);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && sh.abort) {
    for (int k = max(0, sh.k_issued - p.stages); k < sh.k_issued; ++k)
      mbar_wait_bounded(&sh.full[k % p.stages], (uint32_t)((k / p.stages) & 1), kDrainNs, nullptr);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

// ---------------------------------------------------------------------------
// Two-SM tiles (cta_group::2) for wide operands (N >= 128: verify, prefill).
//
// A cluster of two CTAs computes a 256-row tile: CTA r holds weight rows
// [128 r, 128 r + 128) of the tile and rows [N/2 r, N/2 r + N/2) of the B
// operand in its shared memory, and its TMEM holds the 128 x N accumulator
// of its rows.  Per k-block each CTA loads 16 KB of weights and N/2 x 128 B
// of activations instead of N x 128 B: half the activation traffic per
// weight byte of the one-SM kernel.  Both CTAs load their own halves and
// signal the leader's (rank 0) "full" barrier, which the leader's producer
// arms with both CTAs' bytes; the leader's MMA warp issues every MMA
// (tcgen05.mma.cta_group::2, M = 256) and its commits arrive on both CTAs'
// "empty" and "accumulator full" barriers; both epilogues release the
// accumulator on the leader's barrier.  Stream-K partials and tile counters
// are kept per (tile, rank).
// Teardown: both CTAs stop, meet at a cluster barrier, the leader waits for
// every stage either CTA issued (bounded) and for its MMAs, and a second
// cluster barrier precedes TMEM release and exit, so no copy, MMA or
// barrier arrive of one CTA can target a CTA that has left.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared variable in CTA `rank`
__device__ __forceinline__ uint32_t mapa_shared(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t ld_shared_cluster_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// 3-D TMA copy into this CTA's shared memory whose completion is counted on
// the pair leader's barrier (a shared::cluster address).
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const void* tmap, int x, int y, int z,
                                                 uint32_t leader_bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;"
      ::"r"(smem_u32(dst)), "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(leader_bar), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
// arrive (when the leader's MMAs issued so far complete) on the barrier at
// the same offset in the CTAs of `mask`
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)), "h"(mask)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Segment s of stream-K/data-parallel work unit `me` (a CTA, or a CTA pair).
__device__ __forceinline__ bool segment_of(const Sched& S, int me, int64_t u0, int64_t u1, int s,
                                           int& t, int& kb0, int& kb1) {
  if (S.split) return s < S.dp && S.split_item(s * S.ctas + me, t, kb0, kb1);
  if (s < S.dp) {
    t = s * S.ctas + me;
    kb0 = 0;
    kb1 = S.KB;
    return true;
  }
  s -= S.dp;
  if (u0 >= u1) return false;
  const int tl = (int)(u0 / S.KB) + s;
  const int64_t tb = (int64_t)tl * S.KB;
  if (tb >= u1) return false;
  t = S.sk_tile0() + tl;
  kb0 = (int)(max(u0, tb) - tb);
  kb1 = (int)(min(u1, tb + S.KB) - tb);
  return true;
}

// Finish this CTA's 128 rows of a gate-up tile in the pair kernel: its
// accumulator plus the other pairs' partials of the same rank.
template <int CW>
__device__ void finish_tile_pair(const TcParams& p, int t, int rank, uint32_t tb, bool whole,
                                 int c_first, int c_last, int me, int r_local, const float* rv) {
  const int ncol = p.Mt;
  const int rt = t / p.sched.ntok, tt = t % p.sched.ntok;
  const int row = rt * 2 * kBM + rank * kBM + r_local;
  for (int c0 = 0; c0 < ncol; c0 += CW) {
    float vals[CW];
    tile_cols<CW>(p, tb, c0, vals);
    float lo[CW];
    tile_cols<CW>(p, tb, p.Mt + c0, lo);  // lo half of x*gamma
#pragma unroll
    for (int j = 0; j < CW; ++j) vals[j] += lo[j];
    if (!whole) {
      for (int cc = c_first; cc <= c_last; ++cc) {
        if (cc == me) continue;
        int64_t cu0, cu1;
        p.sched.range(cc, cu0, cu1);
        const int slot = (t == p.sched.sk_tile0() + (int)(cu0 / p.sched.KB)) ? 0 : 1;
        const float* part =
            p.partials + ((size_t)(cc * 2 + rank) * 2 + slot) * (size_t)p.N * kBM;
#pragma unroll
        for (int j = 0; j < CW; ++j)
          vals[j] += __ldcg(part + (size_t)(c0 + j) * kBM + r_local) +
                     __ldcg(part + (size_t)(p.Mt + c0 + j) * kBM + r_local);
      }
    }
    epilogue_columns<CW>(p, tt, row, vals, c0, rv);
  }
}

template <int CW>
__device__ void add_tile_to_out_pair(const TcParams& p, int t, int rank, uint32_t tb,
                                     int r_local) {
  const int rt = t / p.sched.ntok, tt = t % p.sched.ntok;
  const int n = rt * 2 * kBM + rank * kBM + r_local;
  for (int c0 = 0; c0 < p.N; c0 += CW) {
    float v[CW];
    tile_cols<CW>(p, tb, c0, v);
    if (n < p.d) {
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        const int m = tt * p.Mt + c0 + j;
        if (m < p.M) atomicAdd(p.out + (int64_t)m * p.d + n, v[j]);
      }
    }
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTcThreads, 1)
    tc_gemm_pair(const __grid_constant__ TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ TcShared sh;
  uint8_t* stage0 = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = (int)cluster_ctarank();
  const bool leader = rank == 0;
  const int me = (int)blockIdx.x / 2;  // the pair's work index
  const int N = p.N, half_n = p.N / 2;
  int64_t u0, u1;
  p.sched.range(me, u0, u1);
  int nseg = 0, nk = 0;
  {
    int t, a, b;
    while (segment_of(p.sched, me, u0, u1, nseg, t, a, b)) {
      nk += b - a;
      ++nseg;
    }
  }

  if (threadIdx.x == 0) {
    for (int j = 0; j < p.stages; ++j) {
      mbar_init(&sh.full[j], 1);   // the leader's producer arms it (both CTAs' bytes)
      mbar_init(&sh.empty[j], 1);  // one multicast commit per stage
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(&sh.acc_full[j], 1);
      mbar_init(&sh.acc_empty[j], 8);  // four epilogue warps of each CTA (leader's is used)
    }
    mbar_init(&sh.mma_done, 1);
    sh.abort = 0;
    sh.k_issued = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc_pair(&sh.tmem_base, p.tmem_cols);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any copy or arrive targets them
  tc_fence_after();
  grid_launch_dependents();
  const uint32_t tmem = sh.tmem_base;
  volatile int* abort = &sh.abort;
  const uint32_t leader_full = mapa_shared(&sh.full[0], 0);
  const uint32_t leader_acc_empty = mapa_shared(&sh.acc_empty[0], 0);

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      const uint64_t pol_a = evict_first_policy();
      uint64_t pol_b;
      asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol_b));
      const int a_row0 = rank * kBM, b_row0 = rank * half_n;
      int early_kb[kMaxStages], early_tt[kMaxStages];
      const int n_early = min(nk, p.stages) - (p.drop_last && nk <= p.stages ? 1 : 0);
      int k = 0;
      bool ok = true;
      for (int s = 0; s < nseg && ok && !*abort; ++s) {
        int t, kb0, kb1;
        segment_of(p.sched, me, u0, u1, s, t, kb0, kb1);
        const int rt = t / p.sched.ntok, tt = t % p.sched.ntok;
        for (int kb = kb0; kb < kb1; ++kb, ++k) {
          if (p.drop_last && k == nk - 1) {
            ok = false;
            break;
          }
          const int slot = k % p.stages;
          uint8_t* a_dst = stage0 + (size_t)slot * p.stage_bytes;
          uint8_t* b_dst = a_dst + p.a_bytes;
          if (k >= p.stages) {
            if (k == p.stages) {
              grid_dependency_wait();  // activations of the early stages
              for (int e = 0; e < n_early; ++e)
                tma_load_3d_pair(stage0 + (size_t)e * p.stage_bytes + p.a_bytes, &p.b_map, 0,
                                 early_tt[e] * N + b_row0, early_kb[e] * p.KS,
                                 leader_full + 8u * e, pol_b);
            }
            if (!mbar_wait_bounded(&sh.empty[slot], (uint32_t)(((k / p.stages) - 1) & 1),
                                   p.wait_ns, abort)) {
              tc_flag(&sh, p.status);
              ok = false;
              break;
            }
          }
          if (leader)
            mbar_arrive_expect_tx(&sh.full[slot], (uint32_t)(2 * (p.a_bytes + p.b_bytes)));
          tma_load_3d_pair(a_dst, &p.a_map, 0, rt * 2 * kBM + a_row0, kb * p.KS,
                           leader_full + 8u * slot, pol_a);
          if (k < p.stages) {
            early_kb[k] = kb;
            early_tt[k] = tt;
          } else {
            tma_load_3d_pair(b_dst, &p.b_map, 0, tt * N + b_row0, kb * p.KS,
                             leader_full + 8u * slot, pol_b);
          }
          sh.k_issued = k + 1;
        }
      }
      if (k <= p.stages && k > 0) {
        grid_dependency_wait();
        for (int e = 0; e < k; ++e)
          tma_load_3d_pair(stage0 + (size_t)e * p.stage_bytes + p.a_bytes, &p.b_map, 0,
                           early_tt[e] * N + b_row0, early_kb[e] * p.KS, leader_full + 8u * e,
                           pol_b);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader only) ----------------
    if (leader && lane == 0) {
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
                             ((uint32_t)((2 * kBM) >> 4) << 24);
      int k = 0;
      bool ok = true;
      for (int s = 0; s < nseg && ok; ++s) {
        int t, kb0, kb1;
        segment_of(p.sched, me, u0, u1, s, t, kb0, kb1);
        const int buf = s & 1;
        if (!mbar_wait_bounded(&sh.acc_empty[buf], (uint32_t)(((s >> 1) & 1) ^ 1), p.wait_ns,
                               abort)) {
          tc_flag(&sh, p.status);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(buf * p.C * N);
        for (int kb = kb0; kb < kb1; ++kb, ++k) {
          const int slot = k % p.stages;
          if (!mbar_wait_bounded(&sh.full[slot], (uint32_t)((k / p.stages) & 1), p.wait_ns,
                                 abort)) {
            tc_flag(&sh, p.status);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(stage0 + (size_t)slot * p.stage_bytes);
          const uint32_t b_addr = a_addr + p.a_bytes;
          const uint32_t b_kblock = (uint32_t)(half_n * kBK * 2);
          const int nkb = min(p.KS, p.KBtot - kb * p.KS);
          for (int kbi = 0; kbi < nkb; ++kbi) {
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const int c = kk % p.C;
              const bool first = kb == kb0 && kbi == 0 && kk < p.C;
              mma_bf16_pair(d_tmem + (uint32_t)(c * N),
                            sw128_desc(a_addr + (uint32_t)(kbi * kATileBytes) + kk * 32),
                            sw128_desc(b_addr + (uint32_t)kbi * b_kblock + kk * 32), idesc,
                            first ? 0u : 1u);
            }
          }
          mma_commit_pair(&sh.empty[slot], (uint16_t)3);  // both CTAs' slot reusable
        }
        if (ok) mma_commit_pair(&sh.acc_full[buf], (uint16_t)3);
      }
      mma_commit_pair(&sh.mma_done, (uint16_t)1);
      mbar_wait_bounded(&sh.mma_done, 0, kDrainNs, nullptr);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2-5, both CTAs) ----------------
    const int q = warp & 3;
    const int r_local = 32 * q + lane;
    const int et = threadIdx.x - 64;
    const int ncol = p.epi == kEpiSwiGLU ? p.Mt : N;
    grid_dependency_wait();  // 1/RMS and the initial out come from earlier kernels
    for (int s = 0; s < nseg; ++s) {
      int t, kb0, kb1;
      segment_of(p.sched, me, u0, u1, s, t, kb0, kb1);
      const int buf = s & 1;
      if (p.epi == kEpiSwiGLU) {  // 1/RMS of the token tile, while the MMAs run
        const int tt = t % p.sched.ntok;
        for (int i = et; i < p.Mt; i += 128) {
          const int m = tt * p.Mt + i;
          sh.rinv_s[buf][i] = m < p.M ? __ldg(p.rinv + m) : 0.f;
        }
      }
      const bool got =
          mbar_wait_bounded(&sh.acc_full[buf], (uint32_t)((s >> 1) & 1), p.wait_ns, abort);
      if (!got && lane == 0) tc_flag(&sh, p.status);
      if (epilogue_barrier_any(!got)) break;  // also publishes sh.rinv_s
      tc_fence_after();
      const uint32_t tb = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * p.C * N);
      if (p.epi == kEpiDown) {
        if (N % 32 == 0) add_tile_to_out_pair<32>(p, t, rank, tb, r_local);
        else add_tile_to_out_pair<16>(p, t, rank, tb, r_local);
      } else {
        const bool whole = kb0 == 0 && kb1 == p.sched.KB;
        const int64_t tu = (int64_t)(t - p.sched.sk_tile0()) * p.sched.KB;
        const int c_first = whole ? 0 : p.sched.cta_of(tu);
        const int c_last = whole ? 0 : p.sched.cta_of(tu + p.sched.KB - 1);
        bool finalize = whole;
        if (!whole) {
          const int slot = (t == p.sched.sk_tile0() + (int)(u0 / p.sched.KB)) ? 0 : 1;
          float* part = p.partials + ((size_t)blockIdx.x * 2 + slot) * (size_t)N * kBM;
          int c = 0;
          for (; c + 32 <= N; c += 32) {
            float v[32];
            tile_cols<32>(p, tb, c, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) __stcg(part + (size_t)(c + j) * kBM + r_local, v[j]);
          }
          if (c < N) {  // N is a multiple of 16
            float v[16];
            tile_cols<16>(p, tb, c, v);
#pragma unroll
            for (int j = 0; j < 16; ++j) __stcg(part + (size_t)(c + j) * kBM + r_local, v[j]);
          }
          __threadfence();
          named_barrier_sync(1, 128);
          if (et == 0)
            sh.last = atomicAdd(p.counters + 2 * t + rank, 1u) == (uint32_t)(c_last - c_first);
          named_barrier_sync(1, 128);
          finalize = sh.last;
          if (finalize) __threadfence();
        }
        if (finalize) {
          const float* rv = sh.rinv_s[buf];
          if (ncol % 32 == 0)
            finish_tile_pair<32>(p, t, rank, tb, whole, c_first, c_last, me, r_local, rv);
          else if (ncol % 16 == 0)
            finish_tile_pair<16>(p, t, rank, tb, whole, c_first, c_last, me, r_local, rv);
          else
            finish_tile_pair<8>(p, t, rank, tb, whole, c_first, c_last, me, r_local, rv);
          if (!whole && et == 0) atomicExch(p.counters + 2 * t + rank, 0u);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&sh.acc_empty[buf]);
        else mbar_arrive_cluster(leader_acc_empty + 8u * buf);
      }
    }
  }
  __syncthreads();
  cluster_sync();  // neither CTA issues anything any more
  if (leader && threadIdx.x == 0) {
    // Every stage either CTA issued counts its copies on this CTA's barriers:
    // wait for them (bounded) before either CTA may leave.
    const int mine = sh.k_issued;
    const int peer = (int)ld_shared_cluster_u32(mapa_shared(&sh.k_issued, 1));
    const int n = max(mine, peer);
    for (int k = max(0, n - p.stages); k < n; ++k)
      mbar_wait_bounded(&sh.full[k % p.stages], (uint32_t)((k / p.stages) & 1), kPairDrainNs,
                        nullptr);
  }
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, p.tmem_cols);
  }
}

// ---------------------------------------------------------------------------
// Prologue: B operand of the gate-up GEMM and 1/RMS per token.
// One CTA per token slot of the padded token tiles: rows [2Mt*j + i] = hi and
// [2Mt*j + Mt + i] = lo of token m = Mt*j + i (zeros for padding slots).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) act_split(const __nv_bfloat16* __restrict__ x,
                                                 const __nv_bfloat16* __restrict__ gamma,
                                                 float eps, int M, int d, int Mt,
                                                 __nv_bfloat16* __restrict__ b_hl,
                                                 float* __restrict__ rinv,
                                                 uint32_t* __restrict__ counters,
                                                 int ncounters, float* __restrict__ out,
                                                 const __nv_bfloat16* __restrict__ residual) {
  // The GEMM launched next may start (and prefetch its weights) right away;
  // it waits for this grid's completion before it reads what this writes.
  grid_launch_dependents();
  const int slot = blockIdx.x;
  const int j = slot / Mt, i = slot % Mt;
  const int m = slot;
  __nv_bfloat16* hi = b_hl + ((int64_t)2 * Mt * j + i) * d;
  __nv_bfloat16* lo = hi + (int64_t)Mt * d;
  __shared__ float red[8];
  float ss = 0.f;
  // x * gamma, split into hi + lo, and the sum of squares of the row, for 8
  // columns [8v, 8v + 8) given x and gamma there
  auto split8 = [&](int v, const uint4& xv, const uint4& gv) {
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float x0 = bf16lo(xw[e]), x1 = bf16hi(xw[e]);
      ss = fmaf(x0, x0, ss);
      ss = fmaf(x1, x1, ss);
      const float s0 = x0 * bf16lo(gw[e]), s1 = x1 * bf16hi(gw[e]);  // exact in f32
      const __nv_bfloat16 h0 = __float2bfloat16_rn(s0), h1 = __float2bfloat16_rn(s1);
      const __nv_bfloat16 l0 = __float2bfloat16_rn(s0 - __bfloat162float(h0));
      const __nv_bfloat16 l1 = __float2bfloat16_rn(s1 - __bfloat162float(h1));
      hw[e] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
      lw[e] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
    }
    reinterpret_cast<uint4*>(hi)[v] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    reinterpret_cast<uint4*>(lo)[v] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  };
  const int nv = d / 8;
  constexpr int kRegV = 4;  // vectors per thread held in registers (d <= 8192 at 256 threads)
  if (nv <= kRegV * (int)blockDim.x) {
    // gamma (a weight) before the dependency wait; every x load of the
    // thread in flight at once after it
    uint4 gv[kRegV], xv[kRegV];
#pragma unroll
    for (int q = 0; q < kRegV; ++q) {
      const int v = threadIdx.x + q * blockDim.x;
      gv[q] = v < nv ? ld_keep(gamma + (int64_t)v * 8) : make_uint4(0, 0, 0, 0);
    }
    grid_dependency_wait();
#pragma unroll
    for (int q = 0; q < kRegV; ++q) {
      const int v = threadIdx.x + q * blockDim.x;
      xv[q] = make_uint4(0, 0, 0, 0);
      if (m < M && v < nv) xv[q] = ld_keep(x + (int64_t)m * d + (int64_t)v * 8);
    }
#pragma unroll
    for (int q = 0; q < kRegV; ++q) {
      const int v = threadIdx.x + q * blockDim.x;
      if (v < nv) split8(v, xv[q], gv[q]);
    }
  } else {
    grid_dependency_wait();
    for (int v = threadIdx.x; v < nv; v += blockDim.x) {
      uint4 xv = make_uint4(0, 0, 0, 0);
      if (m < M) xv = ld_keep(x + (int64_t)m * d + (int64_t)v * 8);
      split8(v, xv, ld_keep(gamma + (int64_t)v * 8));
    }
  }
  // The stream-K arrival counters start every call at zero, whatever a
  // previous call (an aborted one, or one of another shape) left there.  The
  // previous call's kernels are complete once the wait above returns.
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < ncounters; c += gridDim.x * blockDim.x)
    counters[c] = 0u;
  // The down GEMM adds its split-K shares into out: start it at the residual
  // (or zero), one token row per CTA.
  if (out && m < M)
    for (int v = threadIdx.x; v < d / 4; v += blockDim.x) {
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (residual) {
        const uint2 r = __ldg(reinterpret_cast<const uint2*>(residual + (int64_t)m * d) + v);
        o = make_float4(bf16lo(r.x), bf16hi(r.x), bf16lo(r.y), bf16hi(r.y));
      }
      reinterpret_cast<float4*>(out + (int64_t)m * d)[v] = o;
    }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0 && m < M) {
    float t = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    rinv[m] = 1.0f / sqrtf(t / (float)d + eps);
  }
}

// dst = bf16(src), round to nearest even: the f32 sum of the block rounded to
// its bf16 output once the down projection has finished adding into it.
__global__ void __launch_bounds__(256) out_bf16_kernel(const float* __restrict__ src,
                                                       __nv_bfloat16* __restrict__ dst,
                                                       int64_t n4) {
  grid_launch_dependents();
  grid_dependency_wait();  // the sum is complete once the previous kernel is
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(src)[i];
    uint2 w;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w.x) : "f"(v.y), "f"(v.x));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w.y) : "f"(v.w), "f"(v.z));
    reinterpret_cast<uint2*>(dst)[i] = w;
  }
}

// out = residual (or zero), before a down GEMM that is not preceded by the
// gate-up prologue (fmlp_down_proj).
__global__ void __launch_bounds__(256) out_init(float* __restrict__ out,
                                                const __nv_bfloat16* __restrict__ residual,
                                                int64_t n4) {
  grid_launch_dependents();
  grid_dependency_wait();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    if (residual) {
      const uint2 r = __ldg(reinterpret_cast<const uint2*>(residual) + i);
      o = make_float4(bf16lo(r.x), bf16hi(r.x), bf16lo(r.y), bf16hi(r.y));
    }
    reinterpret_cast<float4*>(out)[i] = o;
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
struct TcPlan {
  int N = 0, Mt = 0, ntok = 0, C = 0, KS = 1, stages = 0, stage_bytes = 0, a_bytes = 0,
      b_bytes = 0;
  bool pair = false;   // two-SM tiles (tc_gemm_pair)
  uint32_t tmem_cols = 0;
  size_t smem = 0;
};


uint32_t pow2_at_least(uint32_t n) {
  uint32_t c = 32;
  while (c < n) c <<= 1;
  return c;
}

// Tile shape of one GEMM: token tile Mt (N = 2 Mt for the hi/lo gate-up
// operand) and C accumulator chains (2 C N TMEM columns <= 512, double-buffered).
void tc_shape(int epi, int64_t M, int& Mt, int& N, int& C) {
  if (epi == kEpiSwiGLU) {
    Mt = (int)std::min<int64_t>(128, (M + 7) / 8 * 8);
    N = 2 * Mt;
  } else {
    Mt = (int)std::min<int64_t>(256, (M + 15) / 16 * 16);
    N = Mt;
  }
  C = 4 * N <= 256 ? 4 : (2 * N <= 256 ? 2 : 1);
}

constexpr int kTcMaxKs = 4;

// Stages of KS k-blocks.  On B200 one SM issues TMA copies at a few million
// per second whatever their size (measured: ~2 M stages/s of two copies),
// so a stage moves KS k-blocks of A and of B in one copy each.  KS is the
// largest that still leaves a ring of min_stages stages: 3 for narrow B
// operands (decode batches: 8B M = 8 went from 3.2 to 5.4 TB/s, M = 32
// gains 4% from 3 stages of 3 k-blocks over 2 of 4) and 2 or 3 for wide ones
// (below).
TcPlan make_tc_plan(int epi, int64_t M, int64_t K, const DeviceInfo& dev) {
  TcPlan pl;
  tc_shape(epi, M, pl.Mt, pl.N, pl.C);
  pl.ntok = (int)((M + pl.Mt - 1) / pl.Mt);
  const size_t budget = (size_t)dev.max_smem_optin - 2048 - 1024;  // static + alignment slack
  const int kb_total = (int)(K / kBK);
  // Two-SM tiles for wide operands (measured: pairing narrower ones, the
  // M = 32 decode batch, was 4% slower).  Ring depth, measured per shape:
  // streaming weights read once (one token tile: verify) want 3 stages of 2
  // k-blocks; weight tiles reused from L2 (prefill) want 2 stages of 3.
  pl.pair = pl.N >= 128;
  const int b_rows = pl.pair ? pl.N / 2 : pl.N;  // per CTA: a pair holds half the B rows
  const int min_stages = pl.pair ? (pl.ntok > 1 ? 2 : 3) : (pl.N < 128 ? 3 : 2);
  for (int ks = kTcMaxKs; ks >= 1; --ks) {
    if (ks > 1 && ks > kb_total) continue;
    pl.KS = ks;
    pl.a_bytes = ks * kATileBytes;
    pl.b_bytes = ks * b_rows * kBK * 2;
    pl.stage_bytes = (pl.a_bytes + pl.b_bytes + 1023) / 1024 * 1024;
    pl.stages = (int)std::min<size_t>(kMaxStages, budget / pl.stage_bytes);
    if (pl.stages >= min_stages) break;
  }
  pl.smem = (size_t)pl.stages * pl.stage_bytes + 1024;
  pl.tmem_cols = pow2_at_least((uint32_t)(2 * pl.C * pl.N));
  return pl;
}

template <typename Kernel>
cudaError_t allow_tc_smem(Kernel kernel, const DeviceInfo& dev) {
  static std::mutex mu;
  static std::set<std::pair<int, const void*>> done;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(dev.device, (const void*)kernel);
  if (done.count(key)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       dev.max_smem_optin - 2048);
  if (e == cudaSuccess) done.insert(key);
  return e;
}

// CTA pairs of tc_gemm_pair that can be resident at once (cluster placement
// may leave some SMs unpaired), queried once per device.
int pair_slots(const DeviceInfo& dev, size_t smem) {
  static std::mutex mu;
  static std::set<std::pair<int, int>> done;
  static int slots[64] = {0};
  std::lock_guard<std::mutex> lock(mu);
  if (dev.device >= 0 && dev.device < 64 && slots[dev.device] > 0) return slots[dev.device];
  int n = 0;
  if (allow_tc_smem(tc_gemm_pair, dev) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(dev.sm_count & ~1));
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = smem;
    if (cudaOccupancyMaxActiveClusters(&n, tc_gemm_pair, &cfg) != cudaSuccess) n = 0;
  }
  if (n <= 0) n = dev.sm_count / 2;
  n = std::min(n, dev.sm_count / 2);
  if (dev.device >= 0 && dev.device < 64) slots[dev.device] = n;
  return n;
}

cudaError_t launch_tc(const TcParams& p, const TcPlan& pl, const DeviceInfo& dev,
                      cudaStream_t stream) {
  cudaError_t e = pl.pair ? allow_tc_smem(tc_gemm_pair, dev) : allow_tc_smem(tc_gemm, dev);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(pl.pair ? 2 * p.sched.ctas : p.sched.ctas));
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = pl.pair ? cudaLaunchKernelEx(&cfg, tc_gemm_pair, p) : cudaLaunchKernelEx(&cfg, tc_gemm, p);
  if (e == cudaSuccess) note_launches(1);
  return e;
}

void fill_common(TcParams& p, const TcPlan& pl, int epi, int64_t M, int rows, int K,
                 const TcWorkspace& ws, const DeviceInfo& dev) {
  (void)epi;
  p.epi = epi;
  p.N = pl.N;
  p.Mt = pl.Mt;
  p.M = (int)M;
  p.rows = rows;
  p.C = pl.C;
  p.KS = pl.KS;
  p.KBtot = K / kBK;
  p.stages = pl.stages;
  p.stage_bytes = pl.stage_bytes;
  p.a_bytes = pl.a_bytes;
  p.b_bytes = pl.b_bytes;
  p.tmem_cols = pl.tmem_cols;
  p.sched.KB = (K / kBK + pl.KS - 1) / pl.KS;
  p.sched.ntok = pl.ntok;
  // work units are CTAs, or CTA pairs with 256-row tiles
  const int tile_rows = pl.pair ? 2 * kBM : kBM;
  p.sched.tiles = ((rows + tile_rows - 1) / tile_rows) * pl.ntok;
  const int64_t units_max = pl.pair ? pair_slots(dev, pl.smem) : std::min(dev.sm_count, kTcMaxCtas);
  p.sched.ctas = (int)std::min<int64_t>((int64_t)p.sched.tiles * p.sched.KB, units_max);
  // With one token tile no weight tile is reused, so plain stream-K balances
  // best.  Otherwise whole waves run data-parallel, and the stream-K rest is
  // kept at half a wave or more (folding one wave into it if needed) so that
  // a stream-K tile has only a few contributors.
  const int waves = p.sched.tiles / p.sched.ctas, rest = p.sched.tiles % p.sched.ctas;
  p.sched.dp = pl.ntok == 1 ? 0 : (2 * rest >= p.sched.ctas ? waves : std::max(0, waves - 1));
  p.sched.split = 0;
  if (epi == kEpiDown && pl.ntok > 1) {
    // The down GEMM adds every share into out, so it can run all of its work
    // as data-parallel (tile, k-part) items: the CTAs of a round then share
    // each weight stage across the token tiles, where a stream-K remainder
    // read a weight tile once per token tile (8B prefill: 598 MB of DRAM
    // reads against 176 MB).  The k-part count fills the rounds best.
    const int max_split = std::max(1, std::min(8, p.sched.KB / 4));
    double best = -1.0;
    for (int sp = 1; sp <= max_split; ++sp) {
      const int64_t items = (int64_t)p.sched.tiles * sp;
      const int64_t rounds = (items + p.sched.ctas - 1) / p.sched.ctas;
      const double eff = (double)items / (double)(rounds * p.sched.ctas);
      if (eff > best + 1e-3) {
        best = eff;
        p.sched.split = sp;
        p.sched.dp = (int)rounds;
      }
    }
  }
  p.partials = ws.partials;
  p.counters = ws.counters;
  p.status = ws.status;
  p.wait_ns = wait_timeout_ns();
  p.drop_last = fault_injection();
}

}  // namespace

TcSizes tc_sizes(int64_t M, int64_t d, int64_t I, int sm_count) {
  if (M < 1) return TcSizes();
  TcSizes z;
  int Mt_g, N_g, C_g, Mt_d, N_d, C_d;
  tc_shape(kEpiSwiGLU, M, Mt_g, N_g, C_g);
  tc_shape(kEpiDown, M, Mt_d, N_d, C_d);
  const int64_t ntok_g = (M + Mt_g - 1) / Mt_g, ntok_d = (M + Mt_d - 1) / Mt_d;
  z.b_hl = (size_t)ntok_g * 2 * Mt_g * d * 2;
  z.rinv = (size_t)M * 4;
  z.partials = (size_t)sm_count * 2 * std::max(N_g, N_d) * kBM * 4;
  const int64_t tiles_g = ((2 * I + kBM - 1) / kBM) * ntok_g;
  const int64_t tiles_d = ((d + kBM - 1) / kBM) * ntok_d;
  // one counter per 128-row tile (per (256-row tile, rank) in the pair kernel)
  z.counters = (size_t)(std::max(tiles_g, tiles_d) + 2) * 4;
  return z;
}

bool tc_supported(int64_t M, int64_t d, int64_t I, int T) {
  return M >= 1 && d % 64 == 0 && I % 64 == 0 && (T == 8 || T == 16);
}

cudaError_t launch_tc_gateup(const void* x, int64_t M, const void* gamma, float eps,
                             const void* P, int T, int64_t d, int64_t I, void* a,
                             float* out_init, const void* residual, const TcWorkspace& ws,
                             const DeviceInfo& dev, cudaStream_t stream) {
  const TcPlan pl = make_tc_plan(kEpiSwiGLU, M, d, dev);
  // prologue: hi/lo split of x * gamma into the token-tiled B operand, and 1/RMS
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(pl.ntok * pl.Mt));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, act_split, (const __nv_bfloat16*)x,
                                       (const __nv_bfloat16*)gamma, eps, (int)M, (int)d, pl.Mt,
                                       (__nv_bfloat16*)ws.b_hl, ws.rinv, ws.counters,
                                       ws.ncounters, out_init, (const __nv_bfloat16*)residual);
    if (e != cudaSuccess) return e;
    note_launches(1);
  }
  TcParams p;
  memset(&p, 0, sizeof(p));
  const int rows = (int)(2 * I);
  cudaError_t e = encode_tmap_kblocks_bf16(&p.a_map, P, (uint64_t)rows, (uint64_t)d,
                                           (uint64_t)d * 2, kBM, (uint32_t)pl.KS);
  if (e == cudaSuccess)
    e = encode_tmap_kblocks_bf16(&p.b_map, ws.b_hl, (uint64_t)pl.ntok * 2 * pl.Mt, (uint64_t)d,
                                 (uint64_t)d * 2, (uint32_t)(pl.pair ? pl.N / 2 : pl.N),
                                 (uint32_t)pl.KS);
  if (e != cudaSuccess) return e;
  fill_common(p, pl, kEpiSwiGLU, M, rows, (int)d, ws, dev);
  p.T = T;
  p.I = (int)I;
  p.d = (int)d;
  p.rinv = ws.rinv;
  p.a_out = (__nv_bfloat16*)a;
  return launch_tc(p, pl, dev, stream);
}

cudaError_t launch_out_bf16(const float* src, void* dst, int64_t M, int64_t d,
                            const DeviceInfo& dev, cudaStream_t stream) {
  const int64_t n4 = M * d / 4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>((n4 + 255) / 256,
                                                                       4 * dev.sm_count)));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, out_bf16_kernel, src, (__nv_bfloat16*)dst, n4);
  if (e == cudaSuccess) note_launches(1);
  return e;
}

cudaError_t launch_out_init(float* out, const void* residual, int64_t M, int64_t d,
                            const DeviceInfo& dev, cudaStream_t stream) {
  const int64_t n4 = M * d / 4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>((n4 + 255) / 256,
                                                                       4 * dev.sm_count)));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, out_init, out, (const __nv_bfloat16*)residual, n4);
  if (e == cudaSuccess) note_launches(1);
  return e;
}

cudaError_t launch_tc_down(const void* a, int64_t M, const void* W_down, int64_t d, int64_t I,
                           float* out, const TcWorkspace& ws, const DeviceInfo& dev,
                           cudaStream_t stream) {
  const TcPlan pl = make_tc_plan(kEpiDown, M, I, dev);
  TcParams p;
  memset(&p, 0, sizeof(p));
  cudaError_t e = encode_tmap_kblocks_bf16(&p.a_map, W_down, (uint64_t)d, (uint64_t)I,
                                           (uint64_t)I * 2, kBM, (uint32_t)pl.KS);
  if (e == cudaSuccess)
    e = encode_tmap_kblocks_bf16(&p.b_map, a, (uint64_t)M, (uint64_t)I, (uint64_t)I * 2,
                                 (uint32_t)(pl.pair ? pl.N / 2 : pl.N), (uint32_t)pl.KS);
  if (e != cudaSuccess) return e;
  fill_common(p, pl, kEpiDown, M, (int)d, (int)I, ws, dev);
  p.I = (int)I;
  p.d = (int)d;
  p.out = out;
  return launch_tc(p, pl, dev, stream);
}

}  // namespace fmlp
