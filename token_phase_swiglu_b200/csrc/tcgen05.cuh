// tcgen05 (5th-generation tensor core) primitives shared by the tensor-core
// kernels (sm_100a only): shared-memory matrix and instruction descriptors,
// MMA issue and commit, TMEM allocation and loads, and the stream-K schedule.
#pragma once

#include "common.cuh"

namespace fmlp {

constexpr int kBM = 128;        // A rows per tile (MMA M)
constexpr int kBK = 64;         // k-block: one 128-byte swizzle atom of bf16
constexpr int kATileBytes = kBM * kBK * 2;

// ---------------------------------------------------------------------------
// tcgen05 wrappers
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor: K-major tile of rows x 128 bytes with the
// 128-byte swizzle (8-row atoms of 1024 bytes, stride 1024 bytes between atoms).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address (16-byte units)
  d |= (uint64_t)1 << 16;                    // leading offset: unused for swizzled K-major
  d |= (uint64_t)(1024 >> 4) << 32;          // stride offset between 8-row atoms
  d |= (uint64_t)1 << 46;                    // descriptor version
  d |= (uint64_t)2 << 61;                    // 128-byte swizzle
  return d;
}

// Instruction descriptor: bf16 x bf16 -> f32, A and B K-major, M = 128, N.
__host__ __device__ constexpr uint32_t idesc_bf16(int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(kBM >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::
                   "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// 32 lanes x W consecutive 32-bit columns (W = 8, 16, 32); thread i of the
// warp gets lane (32 * (warp % 4) + i), columns col..col+W-1.  No wait:
// several loads may be in flight; tmem_wait() before using the values.
template <int W>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[W]);
template <>
__device__ __forceinline__ void tmem_ld<8>(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld<16>(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld<32>(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Barrier of the four epilogue warps that also ORs a failure flag, so that a
// timeout in any of them makes all of them leave together.
__device__ __forceinline__ bool epilogue_barrier_any(bool failed) {
  uint32_t any;
  asm volatile(
      "{\n .reg .pred q, r;\n setp.ne.u32 q, %1, 0;\n"
      " bar.red.or.pred r, 2, 128, q;\n selp.u32 %0, 1, 0, r;\n}"
      : "=r"(any)
      : "r"((uint32_t)failed)
      : "memory");
  return any != 0;
}

// ---------------------------------------------------------------------------
// Schedule: data-parallel rounds, then stream-K over the remainder.
//
// Tiles are numbered t = row_tile * ntok + token_tile.  In round r < dp
// work unit c (a CTA, or a CTA pair) computes tile r * ctas + c whole, so the
// units running at the same time share each weight row tile across all token
// tiles and it crosses HBM once (L2 serves the other token tiles).  The last
// one to two waves of tiles are cut "stream-K": their (tile, stage) units are
// split evenly over the work units, so a tile may be shared by a few of them;
// each writes its partial accumulator to the workspace and the last one to
// arrive (tile counter) sums them and runs the epilogue.
// ---------------------------------------------------------------------------
struct Sched {
  int KB;      // stages (groups of KS k-blocks) per tile
  int tiles;   // row tiles x token tiles
  int ntok;    // token tiles (tile index = row_tile * ntok + token_tile)
  int ctas;    // grid size
  int dp;      // data-parallel rounds (whole tiles per CTA, or split items)
  int split = 0;  // > 0: every round is data-parallel over (tile, k-part) items, `split`
                  // k-parts per tile, ordered so that a round's items share weight k-parts
                  // (down GEMM only: its shares are added into out); no stream-K part
  __device__ __forceinline__ int sk_tile0() const { return dp * ctas; }
  __device__ __forceinline__ int64_t units() const {
    return split ? 0 : (int64_t)(tiles - sk_tile0()) * KB;
  }
  // Item i of the split schedule: tile t, stages [kb0, kb1).  Items run in
  // the order (row tile, k-part, token tile), so the CTAs of one round that
  // take the token tiles of a row tile read the same weight stages together.
  __device__ __forceinline__ bool split_item(int i, int& t, int& kb0, int& kb1) const {
    if (i >= tiles * split) return false;
    const int tt = i % ntok, rest = i / ntok, kp = rest % split, rt = rest / split;
    t = rt * ntok + tt;
    kb0 = (int)((int64_t)KB * kp / split);
    kb1 = (int)((int64_t)KB * (kp + 1) / split);
    return true;
  }
  // stream-K unit range of CTA c (units counted from the first stream-K tile)
  __device__ __forceinline__ void range(int c, int64_t& u0, int64_t& u1) const {
    const int64_t U = units(), per = U / ctas, rem = U % ctas;
    u0 = c * per + (c < rem ? (int64_t)c : rem);
    u1 = u0 + per + (c < rem ? 1 : 0);
  }
  __device__ __forceinline__ int cta_of(int64_t u) const {
    const int64_t U = units(), per = U / ctas, rem = U % ctas;
    const int64_t big = rem * (per + 1);
    return u < big ? (int)(u / (per + 1)) : (int)(rem + (u - big) / per);
  }
};


// SiLU(g) * u with the hardware exp2 and reciprocal approximations.  Their
// relative error (a few 1e-7) is far below the bf16 rounding of a that
// follows (2^-9), and the exact form's limits hold: for g << 0, exp(-g) is
// +inf, its reciprocal 0 and the result -0 * u; for g >> 0 it is g * u.  The
// epilogue runs one warp per scheduler, so the exact division and exp would
// sit on the tail of every gate-up GEMM.
__device__ __forceinline__ float silu_mul_fast(float g, float u) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + __expf(-g)));
  return g * r * u;
}

}  // namespace fmlp
