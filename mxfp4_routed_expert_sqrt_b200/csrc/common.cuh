// Shared device helpers of libmoe: error word, mbarriers, 1-D bulk copies,
// element conversions.  sm_100a only.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "moe.h"

namespace moe {

// Device error codes written to g_error (first writer wins).
enum : int32_t {
  kErrNone = 0,
  kErrBadExpert = 0x201,    // an expert id outside [0, E) reached moe_permute
  kErrWaitTc = 0x301,       // tensor-core kernel gave up waiting on an mbarrier
  kErrSpanFlush = 0x302,    // a weight row's E8M0 bytes span > 36 octaves: the lowest groups were flushed
  kErrF16Range = 0x303,     // an activation beyond the f16 range reached the dequantising expert path
  kErrF16Small = 0x304,     // dequantising path: every h of a unit's 32 rows fell below f16's normal range
  kErrWaitSelftest = 0x401, // moe_selftest_wait: its wait ran out, as it should
  kErrBadIndex = 0x501,     // debug build: a pair index (perm / inv) outside [0, T * top_k)
  kErrBadOffsets = 0x502,   // debug build: group offsets not non-decreasing from 0 to T * top_k
};

// The debug build (-DMOE_DEBUG) checks the indices the kernels otherwise
// trust -- the grouped pair ids, the group offsets, the combine's slots --
// records kErrBadIndex / kErrBadOffsets and skips the access instead.
#ifdef MOE_DEBUG
constexpr bool kDebug = true;
#else
constexpr bool kDebug = false;
#endif

__device__ int32_t g_error;

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may begin while its predecessor in the stream is finishing;
// griddep_wait() returns once every prerequisite grid has completed and its
// memory is visible, so each kernel calls it before its first global read or
// write.  griddep_launch() lets the stream's next kernel begin launching (its
// CTAs then wait in their own griddep_wait()).  Without the launch attribute
// both are no-ops.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void set_error(int32_t code) { atomicCAS(&g_error, 0, code); }

// Upper bound on the time a kernel waits for one mbarrier phase before it
// gives up (a copy that has not landed by then never will), and on the number
// of polls (try_wait itself may suspend the thread for a while).
constexpr uint64_t kMaxWaitNs = 2000000000ull;  // 2 s
constexpr uint32_t kMaxPolls = 1u << 26;

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete: false after
// max_ns of %globaltimer time (or kMaxPolls polls).
__device__ __forceinline__ bool mbar_wait_ns(uint64_t* bar, uint32_t parity, uint64_t max_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 0; i < kMaxPolls; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (i >= 32) {
      __nanosleep(64);
      if ((i & 255) == 0 && global_ns() - t0 > max_ns) return false;
    }
  }
  return false;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  return mbar_wait_ns(bar, parity, kMaxWaitNs);
}

// The bounded-wait path on its own: waits for a phase of a fresh mbarrier
// that nothing arrives on, gives up after max_ns, records kErrWaitSelftest
// and returns (what every pipeline kernel does when a copy never lands).
__global__ void selftest_wait_kernel(uint64_t max_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait_ns(&bar, 0, max_ns)) set_error(kErrWaitSelftest);
  }
}

// 1-D bulk copy global -> shared (async proxy), completion counted in bytes
// on `bar`, with an L2 evict-first hint (streamed expert weights are read
// once).  Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s_stream(void* smem_dst, const void* gmem_src,
                                                uint32_t bytes, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], "
      "%2, [%3], %4;" ::"r"(smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Two E2M1 codes (one byte, low nibble first) -> f16x2 (low half = low nibble).
// Exact: every E2M1 value is an f16.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte_in_low8) {
  uint32_t out;
  asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %1;\n"
      " cvt.rn.f16x2.e2m1x2 %0, b0;\n}\n"
      : "=r"(out)
      : "r"(byte_in_low8));
  return out;
}

// Four bytes (8 codes) -> 4 f16x2.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t (&o)[4]) {
  asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}\n"
      : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
      : "r"(w));
}

// bf16x2 -> f16x2 (exact for |v| in [2^-17, 65504]; the activations here are
// N(0,1)-scale, far inside that range).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  float lo = __uint_as_float(v << 16), hi = __uint_as_float(v & 0xFFFF0000u);
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ float silu_clamped_swiglu(float g, float u, float limit) {
  g = fminf(g, limit);
  u = fminf(fmaxf(u, -limit), limit);
  return g / (1.0f + expf(-g)) * u;
}

}  // namespace moe
