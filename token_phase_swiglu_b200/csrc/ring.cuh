// Stage ring of the weight-streaming kernels: one producer lane fills
// shared-memory stages with bulk copies (TMA engine), consumer warps read
// them in order.  Every wait is bounded by a global-timer deadline; on expiry
// the CTA sets the timeout bit of the workspace status word, lets its copies
// in flight land and exits.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace fmlp {

constexpr int kMaxStages = 8;
constexpr int kHeader = 256;                      // full[8], empty[8] mbarriers
constexpr uint64_t kDrainNs = 1000000000ull;      // in-flight copies land long before this
static_assert(2 * kMaxStages * 8 <= kHeader, "barrier block overflows its header");

__host__ __device__ constexpr size_t align128(size_t n) { return (n + 127) & ~size_t(127); }

// Two f32 lanes in one 64-bit register, for the packed FMA of sm_100.
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float hsum2(uint64_t v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return lo + hi;
}
// Barrier `id` of the kConsumerThreads consumer threads; returns true if any
// of them failed.
template <int kConsumerThreads>
__device__ __forceinline__ bool consumer_barrier_any(int id, bool failed) {
  uint32_t any;
  asm volatile(
      "{\n .reg .pred q, r;\n setp.ne.u32 q, %1, 0;\n"
      " bar.red.or.pred r, %2, %3, q;\n selp.u32 %0, 1, 0, r;\n}"
      : "=r"(any)
      : "r"((uint32_t)failed), "r"(id), "n"(kConsumerThreads)
      : "memory");
  return any != 0;
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
  int issued;     // stages issued by the producer
  int out_ready;  // fused_decode: 0 until every share of out is set, then 1 (-1: gave up)
  int last;       // fused_decode: this CTA was the last to finish
};

__device__ __forceinline__ void init_ring(const Ring& r, CtaState& st, int consumers) {
  for (int j = 0; j < r.stages; ++j) {
    mbar_init(&r.full[j], 1);
    mbar_init(&r.empty[j], (uint32_t)consumers);
  }
  st.abort = 0;
  st.issued = 0;
  st.out_ready = 0;
  fence_barrier_init();
}

// After a timeout: let every copy the producer issued land before the CTA
// exits (its shared memory must outlive the copies).  Thread 0 only.  Only
// the last `stages` stages can still be in flight: each earlier one was
// waited on by all consumers before its slot was reissued.
__device__ inline void drain_ring(const Ring& r, int issued) {
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

}  // namespace fmlp
