// Grouped expert GEMM on the 5th-generation tensor cores (tcgen05) with the
// weights dequantised in software: moe_expert_gemm's path for calls with more
// than 24 pairs per expert on average (prefill), and the bf16 GEMMs of the
// router and the shared expert above 64 tokens.
//
// Per unit = (expert e, token chunk of <= n_chunk grouped pairs, row tile):
//   MODE 0 (gate/up):  acc0 = Wg[rows] x^T, acc1 = Wu[rows] x^T over K = hidden;
//                      epilogue h = silu(min(acc0, L)) * clamp(acc1, -L, L),
//                      stored in f16 (|h| <= L^2; 11 mantissa bits)
//   MODE 1 (down):     acc0/acc1 = Wd[2 x 128 rows] h^T over K = inter, fp32 out
// MXFP4 operands run as f16 x f16 MMAs (fp32 accumulation): activations come
// in f16 and each weight is dequantised exactly to f16 as v * 2^(e - 127 -
// c_r), c_r = e_max(row) - 140 (signed), with 2^c_r applied to the fp32
// accumulator row in the epilogue.  That is exact for every group within 36
// octaves of its row's largest (any E8M0 byte otherwise); groups further below
// are flushed to zero and the call records device error 0x302.  Two
// instructions per pair of codes (cvt + multiply).  bf16 weights (shared expert, router) are copied as
// they are.
// ("Model techniques map", row "SwiGLU feed-forward": the clamped SwiGLU;
// "ElytronAI / DeepSeek-v4-Flash", Sizes/Layout: MXFP4 weights, expert xid at
// base + xid * expert_bytes.)
//
// Swap-AB: the weight rows are the MMA's M = 128 dimension and the expert's
// tokens its N dimension (a multiple of 16, <= n_chunk), so a unit needs no
// token padding beyond 16.  The token operand is read from a matrix already in
// unit order (activations gathered per pair beforehand, or h), so it arrives
// by plain 2-D TMA boxes.
//
// Pipeline stage = 2 k-blocks of 64 (K = 128): the A producers write both
// k-blocks' values to TMEM, the token loader both k-blocks' token tiles, and
// the MMA issuer runs 16 MMAs and ONE tcgen05.commit per stage.  On B200 every
// producer/consumer handshake around the tensor pipe costs a few hundred
// cycles that do not overlap the MMAs, so stages are made as long as TMEM
// allows.
//
// Roles (480 or 608 threads, one CTA per SM, persistent over units):
//   warps 0-3 (and 15-18 when EPI = 8)  epilogue: tcgen05.ld of the two
//               accumulators (TMEM lane quadrant = warp mod 4; with 8 warps
//               the two warps of a quadrant take alternate 16-column chunks,
//               so a wide accumulator is released twice as soon), SwiGLU or
//               copy, global stores.  8 epilogue warps pay off for 128-token
//               chunks (prefill); for small chunks the 480-thread launch
//               leaves the A producers more registers;
//   warps 4-11  A producers: thread = one weight row of one of the two tiles;
//               reads its row's bytes from the weight ring (conflict-free: the
//               ring holds swizzled TMA boxes), converts them exactly and writes
//               them into TMEM with tcgen05.st: the MMA takes A from TMEM.
//               Each thread fetches its row's E8M0 bytes for the NEXT unit with
//               cp.async into a thread-major buffer;
//   warp 12     token loader: 2-D TMA boxes of 16 token rows x 64 columns;
//   warp 13     TMEM owner and MMA issuer (the whole warp runs the loop, an
//               elected lane issues each MMA and commit);
//   warp 14     weight loader (one thread): 3-D TMA boxes (128 rows x <= 128
//               bytes per tile, expert index as the third coordinate) into the
//               weight ring, running ahead across unit boundaries.
// TMEM (512 columns): acc0 [0, acc), acc1 [acc, 2 acc), stages of 128 columns
// (2 k-blocks x 2 tiles x 32) from 2 acc.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace moe {

// Threads of a launch with EPI epilogue warps (4: warps 0-3; 8: also 15-18).
__host__ __device__ constexpr int tc_threads(int epi) { return (11 + epi) * 32; }
constexpr int kTcKB = 64;      // k per k-block (one 128-byte swizzle atom of 16-bit values)
constexpr int kTcKG = 2;       // k-blocks per pipeline stage
constexpr int kTcStageK = kTcKB * kTcKG;
constexpr int kTcNMax = 128;   // tokens per unit
constexpr int kTcTmemCols = 512;
constexpr int kTcStageCols = 64 * kTcKG;  // TMEM columns of one stage
constexpr int kTcMaxStages = 8;  // upper bound of every ring's depth
constexpr int kTcAThreads = 256; // A producer threads (8 warps)
constexpr int kTcBoxRows = 16;   // token rows per TMA box
constexpr int kCrowRing = 8;     // units of per-row offsets kept for the epilogue
constexpr int kScaleRowMax = 128;  // E8M0 bytes per weight row (cols <= 4096)
// Dynamic shared memory one CTA may use (the opt-in maximum minus the static
// arrays and the alignment slack).
constexpr int kTcSmemMax = 227 * 1024 - 6 * 1024;

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async8(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---- tcgen05 / TMA primitives --------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]^T.  Called by all 32 lanes of a
// converged warp with the same operands; one lane, chosen by elect.sync,
// issues.  A lone thread in a lane-0 branch issues an MMA only every ~80
// cycles whatever its N (its operands are not warp-uniform); a warp with an
// elected lane every ~45 (measured on a B200).
__device__ __forceinline__ void umma_tmem_a_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                 uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p, e;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// tcgen05.commit from one elected lane of a converged warp.
__device__ __forceinline__ void umma_commit_warp(uint64_t* bar) {
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
        "=r"(v[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 B apart (the layout TMA writes with CU_TENSOR_MAP_SWIZZLE_128B).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;            // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset: next 8-row group
  d |= (uint64_t)1 << 46;            // descriptor version
  d |= (uint64_t)2 << 61;            // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16: bf16 (or f16) A and B, both K-major, fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Box {x, y, z} of a 3-D tensor map into shared memory, L2 hint `policy`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], "
      "[%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Box {x, y} of a 2-D tensor map into shared memory.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Copies issued from a warp that runs the loader loop as a whole: every lane
// calls with the same operands and only the lane whose `leader` is nonzero
// (chosen once with elect.sync) issues, which keeps the operands warp-uniform.
__device__ __forceinline__ uint32_t elect_leader() {
  uint32_t r;
  asm volatile("{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n selp.u32 %0, 1, 0, e;\n}\n" : "=r"(r));
  return r;
}
__device__ __forceinline__ void mbar_arrive_expect_tx_if(uint32_t leader, uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n .reg .pred e;\n setp.ne.b32 e, %0, 0;\n @e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%1], %2;\n}\n" ::"r"(
                   leader),
               "r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void tma_load_3d_if(uint32_t leader, void* dst, const CUtensorMap* map, int x, int y, int z,
                                               uint64_t* bar, uint64_t policy) {
  asm volatile(
      "{\n .reg .pred e;\n setp.ne.b32 e, %0, 0;\n"
      " @e cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%1], [%2, "
      "{%3, %4, %5}], [%6], %7;\n}\n" ::"r"(leader),
      "r"(smem_u32(dst)), "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d_if(uint32_t leader, void* dst, const CUtensorMap* map, int x, int y,
                                               uint64_t* bar) {
  asm volatile(
      "{\n .reg .pred e;\n setp.ne.b32 e, %0, 0;\n"
      " @e cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%1], [%2, {%3, %4}], "
      "[%5];\n}\n" ::"r"(leader),
      "r"(smem_u32(dst)), "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// f16x2 with 2^k in both halves, k in [-24, 15] (subnormal f16 below -14).
__device__ __forceinline__ uint32_t pow2_f16x2(int k) {
  const float f = __uint_as_float((uint32_t)(k + 127) << 23);
  return f32x2_to_f16x2(f, f);
}

// Octaves below a row's largest E8M0 group that still dequantise exactly: a
// code v in {0.5, ..., 6} times 2^k is an f16 value (subnormals included) for
// k in [-23, 13].
constexpr int kF16Span = 36;

// Dequantisation factor of one group, k = e - 127 - c_r <= 13: 2^k as f16x2,
// or 0 (the group flushed) below the exact range.
__device__ __forceinline__ uint32_t group_factor_f16x2(int k) { return k >= -23 ? pow2_f16x2(k) : 0u; }

// 2^k as fp32 for k in [-149, 127] (subnormal below -126).
__device__ __forceinline__ float pow2_f32(int k) {
  return k >= -126 ? __uint_as_float((uint32_t)(k + 127) << 23) : __uint_as_float(1u << (k + 149));
}

// Byte offset inside a TMA box written with the swizzle mode that matches its
// inner extent (128 B: SWIZZLE_128B, 64 B: SWIZZLE_64B): the 16-byte chunk
// bits [4, 4+b) are XORed with the row bits [7, 7+b), mask = 2^b - 1.
__device__ __forceinline__ uint32_t swz(uint32_t off, uint32_t mask) { return off ^ (((off >> 7) & mask) << 4); }

// Slot and phase of a ring of `n` stages.
struct TcRing {
  int s, n;
  uint32_t ph;
  __device__ explicit TcRing(int depth) : s(0), n(depth), ph(0) {}
  __device__ void next() {
    if (++s == n) {
      s = 0;
      ph ^= 1;
    }
  }
};

enum { kAMxfp4 = 0, kABf16 = 1 };

struct TcArgs {
  const uint8_t* w0;     // MODE 0: gate; MODE 1: down (or any bf16 [rows][a_cols] matrix)
  const uint8_t* w1;     // MODE 0: up
  int64_t expert_bytes;  // stride between experts (MXFP4); 0 for a single bf16 matrix
  int rows;              // rows of one projection (the MMA's M extent)
  int a_cols;            // columns of the weight matrix
  int k_total;           // reduction length: a multiple of a_cols (A column = k mod a_cols)
  int b_cols;            // columns of a token row (token column = k mod b_cols)
  const int32_t* offsets;  // [E+1] grouped rows; null: one group of n_single rows
  int E, n_single;
  int n_chunk;           // tokens per unit: multiple of 16, <= kTcNMax
  void* out;             // see the epilogue
  float limit;
  // pipeline shape, filled in by tc_plan()
  int acc_cols;      // TMEM columns per accumulator (>= n_chunk)
  int stages;        // pipeline stages (TMEM A of 2 k-blocks)
  int b_stages;      // token-tile ring (shared memory, 2 k-blocks each): may run ahead of the TMEM stages
  int w_slots;       // weight slots
  int w_inner;       // bytes of one weight row in one TMA box
  int w_slot_bytes;  // bytes of one weight slot (both tiles)
  int st_per_slot;   // pipeline stages per weight slot
  int sr;            // E8M0 bytes per weight row (MXFP4)
  int off_b, off_sc, off_prefix;  // shared-memory offsets from the 1024-aligned base
  int smem_bytes;                 // dynamic shared memory of the launch
};

// Ring depths and the shared-memory carve-up of one launch.  False when the
// shape is outside what the kernel implements.
inline bool tc_plan(TcArgs& a, int af) {
  const int nc = a.n_chunk;
  if (nc < 16 || nc > kTcNMax || nc % 16) return false;
  if (a.k_total % kTcStageK || a.a_cols % kTcKB || a.b_cols % kTcKB || a.k_total % a.a_cols) return false;
  a.acc_cols = nc <= 32 ? 32 : nc <= 64 ? 64 : 128;
  a.stages = (kTcTmemCols - 2 * a.acc_cols) / kTcStageCols;
  if (a.stages > kTcMaxStages) a.stages = kTcMaxStages;
  const int nst = a.k_total / kTcStageK;
  if (af == kAMxfp4) {
    if (a.a_cols % kTcStageK || a.a_cols / 32 > kScaleRowMax || a.k_total != a.a_cols) return false;
    a.w_inner = a.a_cols / 2 < 128 ? a.a_cols / 2 : 128;
    if ((a.a_cols / 2) % a.w_inner) return false;
    a.st_per_slot = a.w_inner / 64;  // 64 code bytes of a row per stage
    a.w_slot_bytes = 2 * 128 * a.w_inner;
    a.sr = a.a_cols / 32;
  } else {
    a.w_inner = 128;  // 64 bf16 columns per box, two boxes per tile and stage
    a.st_per_slot = 1;
    a.w_slot_bytes = 2 * kTcKG * 128 * 128;
    a.sr = 0;
  }
  if (nst % a.st_per_slot) return false;
  // the A producers run at most ceil(stages / nst) + 1 units ahead of the
  // epilogue, which reads their per-row offsets
  if ((a.stages + nst - 1) / nst + 1 >= kCrowRing) return false;
  const int bst = kTcKG * nc * 128;
  const int sc = af == kAMxfp4 ? 2 * kTcAThreads * a.sr : 0;
  const int groups = a.offsets != nullptr ? a.E : 1;
  const int pre = (2 * (groups + 1) * 4 + 127) / 128 * 128;  // unit prefix + group offsets
  const int budget = kTcSmemMax - 1024;  // 1024: alignment slack of the dynamic base
  auto weight_slots = [&](int b_stages) { return (budget - b_stages * bst - sc - pre) / a.w_slot_bytes; };
  // Token tiles one stage deeper than the TMEM stages, so a tile's copy is in
  // flight while the two TMEM stages turn over (its latency otherwise stalls
  // every stage): MXFP4 weights then come in 64-byte boxes (one stage per
  // slot) if 128-byte ones leave no room for it.  At least three weight stages
  // stay in flight.
  a.b_stages = a.stages;
  if (af == kAMxfp4 && a.stages + 1 <= kTcMaxStages) {
    const int b3 = a.stages + 1;
    if (weight_slots(b3) * a.st_per_slot >= 3 && weight_slots(b3) >= 2) {
      a.b_stages = b3;
    } else if (a.w_inner == 128 && (a.a_cols / 2) % 64 == 0) {
      const int keep_inner = a.w_inner, keep_sps = a.st_per_slot, keep_wsb = a.w_slot_bytes;
      a.w_inner = 64;
      a.st_per_slot = 1;
      a.w_slot_bytes = 2 * 128 * 64;
      if (weight_slots(b3) >= 3) {
        a.b_stages = b3;
      } else {
        a.w_inner = keep_inner;
        a.st_per_slot = keep_sps;
        a.w_slot_bytes = keep_wsb;
      }
    }
  }
  const int w = weight_slots(a.b_stages);
  a.w_slots = w < 6 ? w : 6;
  if (a.w_slots < 2) return false;
  a.off_b = a.w_slots * a.w_slot_bytes;
  a.off_sc = a.off_b + a.b_stages * bst;
  a.off_prefix = a.off_sc + sc;
  a.smem_bytes = a.off_prefix + pre + 1024;
  return a.smem_bytes <= kTcSmemMax;
}

template <int MODE, int AF, int EPI>
__global__ void __launch_bounds__(tc_threads(EPI), 1)
    tc_expert_kernel(const __grid_constant__ CUtensorMap bmap, const __grid_constant__ CUtensorMap wmap0,
                     const __grid_constant__ CUtensorMap wmap1, const TcArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kTcMaxStages], empty[kTcMaxStages];
  __shared__ __align__(8) uint64_t b_full[kTcMaxStages], b_empty[kTcMaxStages];
  __shared__ __align__(8) uint64_t w_full[kTcMaxStages], w_empty[kTcMaxStages];
  __shared__ __align__(8) uint64_t acc_full, acc_empty, mma_done;
  __shared__ uint32_t s_taddr;
  __shared__ int32_t s_abort;
  __shared__ int16_t s_crow[kCrowRing][2][128];  // per-row f16 offsets c_r, ring over units

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_w = smem;                  // weight ring
  uint8_t* s_b = smem + args.off_b;     // token tiles, ring of b_stages
  uint8_t* s_sc = smem + args.off_sc;   // E8M0 rows, two unit buffers, thread-major
  int32_t* s_prefix = reinterpret_cast<int32_t*>(smem + args.off_prefix);  // [E + 1] units before group e
  int32_t* s_off = s_prefix + (args.offsets != nullptr ? args.E : 1) + 1;  // [E + 1] copy of offsets

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool grouped = args.offsets != nullptr;
  const int E = grouped ? args.E : 1;
  const int MT = MODE == 0 ? args.rows / 128 : args.rows / 256;  // row tiles per group
  const int nst = args.k_total / kTcStageK;                       // stages per unit
  const int NC = args.n_chunk;
  const int tile_bytes = args.w_slot_bytes / 2;
  const int atom = NC * 128;         // one k-block of token rows (128-byte rows)
  const int bst = kTcKG * atom;      // token bytes of one stage
  const uint32_t a_base = 2 * args.acc_cols;

  // ---- unit table: units(e) = MT * ceil(n_e / NC), exclusive prefix ----------
  // The group offsets are read once, by all threads in parallel, into shared
  // memory: the scan and every unit lookup then stay on chip.
  griddep_wait();  // inputs come from earlier kernels of the stream
  if (grouped)
    for (int i = tid; i <= E; i += blockDim.x) s_off[i] = args.offsets[i];
  __syncthreads();
  if (kDebug && grouped) {  // offsets must not decrease (the pair count bounds them above)
    bool bad = false;
    for (int i = tid; i < E; i += blockDim.x) bad |= s_off[i] > s_off[i + 1];
    if (tid == 0) bad |= s_off[0] != 0;
    if (__syncthreads_or(bad ? 1 : 0)) {
      if (tid == 0) set_error(kErrBadOffsets);
      for (int i = tid; i <= E; i += blockDim.x) s_off[i] = 0;  // no units
      __syncthreads();
    }
  }
  if (warp == 0) {
    int run = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int c = 0;
      if (e < E) {
        const int n = grouped ? s_off[e + 1] - s_off[e] : args.n_single;
        c = MT * ((n + NC - 1) / NC);
      }
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (e < E) s_prefix[e] = run + incl - c;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_prefix[E] = run;
  }
  if (tid == 0) {
    for (int s = 0; s < kTcMaxStages; ++s) {
      mbar_init(&full[s], 8);  // one arrival per A-producer warp
      mbar_init(&empty[s], 1);
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
      mbar_init(&w_full[s], 1);
      mbar_init(&w_empty[s], 8);
    }
    mbar_init(&acc_full, 1);
    mbar_init(&acc_empty, EPI);
    mbar_init(&mma_done, 1);
    s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 13) {
    tmem_alloc(&s_taddr, kTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = s_taddr;
  const int n_units = s_prefix[E];
  // the next kernel may begin launching once every CTA has started its last unit
  if (tid == 0 && (int)blockIdx.x + (int)gridDim.x >= n_units) griddep_launch();

  // unit -> (group, row tile, first row of the token matrix, tokens)
  auto decode_unit = [&](int u, int& e, int& mt, int& pos0, int& n) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {  // last e with s_prefix[e] <= u
      const int mid = (lo + hi + 1) >> 1;
      if (s_prefix[mid] <= u) lo = mid; else hi = mid - 1;
    }
    e = lo;
    const int local = u - s_prefix[e];
    mt = local % MT;
    const int chunk = local / MT;
    const int start = grouped ? s_off[e] : 0;
    const int ne = grouped ? s_off[e + 1] - start : args.n_single;
    pos0 = start + chunk * NC;
    n = min(NC, ne - chunk * NC);
  };
  auto aborted = [&]() { return *reinterpret_cast<volatile int32_t*>(&s_abort) != 0; };
  auto give_up = [&]() {
    set_error(kErrWaitTc);
    *reinterpret_cast<volatile int32_t*>(&s_abort) = 1;
  };
  // bounded wait whose outcome is the same for the whole warp (the tcgen05
  // loads and stores that follow are taken by whole warps)
  auto warp_wait = [&](uint64_t* bar, uint32_t ph) {
    return __all_sync(0xffffffffu, mbar_wait(bar, ph) ? 1 : 0) != 0;
  };

  if (warp >= 4 && warp < 12) {
    // ------------------------------ A producers --------------------------------
    const int t = (warp - 4) >> 2, q = warp & 3, r = q * 32 + lane;
    const int tslot = (warp - 4) * 32 + lane;
    const uint32_t tl = tbase + ((uint32_t)(q * 32) << 16) + a_base + t * 32;
    const uint32_t mask = (uint32_t)args.w_inner / 16 - 1;
    TcRing rs(args.stages), rw(args.w_slots);
    int js = 0;  // stage within the current weight slot
    // publish stage rs.s (both k-blocks stored): one arrival per warp
    auto publish = [&]() {
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[rs.s]);
      rs.next();
      if (++js == args.st_per_slot) {  // slot fully read: hand it back to the loader
        js = 0;
        if (lane == 0) mbar_arrive(&w_empty[rw.s]);
        rw.next();
      }
    };
    auto wait_stage = [&]() -> bool {  // TMEM stage free (its MMAs done)
      if (!warp_wait(&empty[rs.s], rs.ph ^ 1)) return false;
      tc_fence_after();
      return true;
    };
    if (AF == kAMxfp4) {
      const int sr = args.sr, cs = sr < 16 ? sr : 16;
      const int64_t plane = (int64_t)args.rows * (args.a_cols / 2);
      // this thread's E8M0 row of unit u -> scale buffer `buf`, cs-byte pieces
      // at [piece][thread] (cp.async; committed by the caller)
      auto sc_issue = [&](int u, int buf) {
        int e, mt, pos0, n;
        decode_unit(u, e, mt, pos0, n);
        const int R = MODE == 0 ? mt * 128 + r : mt * 256 + t * 128 + r;
        const uint8_t* src =
            (MODE == 0 && t == 1 ? args.w1 : args.w0) + (int64_t)e * args.expert_bytes + plane + (int64_t)R * sr;
        uint8_t* dst = s_sc + buf * kTcAThreads * sr + tslot * cs;
        for (int c = 0; c < sr / cs; ++c) {
          uint8_t* d = dst + c * kTcAThreads * cs;
          if (cs == 16) cp_async16(d, src + c * 16);
          else if (cs == 8) cp_async8(d, src + c * 8);
          else cp_async4(d, src + c * 4);
        }
      };
      if ((int)blockIdx.x < n_units) sc_issue(blockIdx.x, 0);
      cp_async_commit();
      uint32_t un = 0;
      for (int u = blockIdx.x; u < n_units && !__any_sync(0xffffffffu, aborted() ? 1 : 0); u += gridDim.x, ++un) {
        if (u + (int)gridDim.x < n_units) sc_issue(u + gridDim.x, (un + 1) & 1);
        cp_async_commit();
        cp_async_wait<1>();  // this unit's E8M0 row has landed
        const uint8_t* scb = s_sc + (un & 1) * kTcAThreads * sr + tslot * cs;
        auto sc_word = [&](int w) {  // E8M0 bytes 4w .. 4w + 3 of the row
          const int b = 4 * w;
          return *reinterpret_cast<const uint32_t*>(scb + (b / cs) * kTcAThreads * cs + b % cs);
        };
        // per-row exponent offset c_r = e_max(row) - 140 (signed): every group
        // factor 2^(e-127-c_r) = 2^(e - e_max + 13) is at most 2^13, so the
        // largest code (6) stays inside f16, and groups down to 36 octaves
        // below the row's largest are exact f16 values
        uint32_t mx = 0, mn = 0xFFFFFFFFu;
        for (int w = 0; w < sr / 4; ++w) {
          const uint32_t v = sc_word(w);
          mx = __vmaxu4(mx, v);
          mn = __vminu4(mn, v);
        }
        mx = __vmaxu4(mx, mx >> 16);
        mx = __vmaxu4(mx, mx >> 8);
        mn = __vminu4(mn, mn >> 16);
        mn = __vminu4(mn, mn >> 8);
        const int crow = (int)(mx & 0xFFu) - 140;
        // a wider span cannot be exact in f16: those groups are flushed to
        // zero (their products are below 2^-36 of the row's largest group's)
        // and the call is flagged
        if ((int)(mx & 0xFFu) - (int)(mn & 0xFFu) > kF16Span) set_error(kErrSpanFlush);
        s_crow[un % kCrowRing][t][r] = (int16_t)crow;
        // k-block g of the current stage of this row -> 64 f16 values
        auto convert = [&](int g, uint32_t sw, uint32_t (&v)[32]) {
          const uint8_t* tile = s_w + rw.s * args.w_slot_bytes + t * tile_bytes;
          const uint32_t o = (uint32_t)(r * args.w_inner + 64 * js + 32 * g);
          const uint4 c0 = *reinterpret_cast<const uint4*>(tile + swz(o, mask));
          const uint4 c1 = *reinterpret_cast<const uint4*>(tile + swz(o + 16, mask));
          const int e0 = (int)((sw >> (16 * g)) & 0xFFu), e1 = (int)((sw >> (16 * g + 8)) & 0xFFu);
          const uint32_t wds[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
          const uint32_t f0 = group_factor_f16x2(e0 - 127 - crow);
          const uint32_t f1 = group_factor_f16x2(e1 - 127 - crow);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t hv[4];
            e2m1x8_to_f16x2(wds[c], hv);
#pragma unroll
            for (int b = 0; b < 4; ++b) v[4 * c + b] = hmul2(hv[b], c < 4 ? f0 : f1);
          }
        };
        bool ok = true;
        for (int st = 0; st < nst && ok; ++st) {
          if (js == 0 && !warp_wait(&w_full[rw.s], rw.ph)) {
            ok = false;
            break;
          }
          const uint32_t sw = sc_word(st);  // E8M0 of this stage's two k-blocks
          // both k-blocks converted while the stage is still in use: once it
          // frees, only the stores stand between it and the MMAs
          uint32_t v0[32], v1[32];
          convert(0, sw, v0);
          convert(1, sw, v1);
          if (!wait_stage()) {
            ok = false;
            break;
          }
          tmem_st32(tl + rs.s * kTcStageCols, v0);
          tmem_st32(tl + rs.s * kTcStageCols + 64, v1);
          publish();
        }
        if (!ok) {
          give_up();
          break;
        }
      }
      cp_async_wait<0>();
    } else {
      // bf16 rows, copied as they are (the loader picks column k mod a_cols)
      auto copy = [&](int g, uint32_t (&v)[32]) {
        const uint8_t* box = s_w + rw.s * args.w_slot_bytes + t * tile_bytes + g * 16384;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(box + swz((uint32_t)(r * 128 + 16 * c), 7));
          v[4 * c] = w.x;
          v[4 * c + 1] = w.y;
          v[4 * c + 2] = w.z;
          v[4 * c + 3] = w.w;
        }
      };
      for (int u = blockIdx.x; u < n_units && !__any_sync(0xffffffffu, aborted() ? 1 : 0); u += gridDim.x) {
        bool ok = true;
        for (int st = 0; st < nst && ok; ++st) {
          if (!warp_wait(&w_full[rw.s], rw.ph)) {
            ok = false;
            break;
          }
          uint32_t v0[32], v1[32];
          copy(0, v0);
          copy(1, v1);
          if (!wait_stage()) {
            ok = false;
            break;
          }
          tmem_st32(tl + rs.s * kTcStageCols, v0);
          tmem_st32(tl + rs.s * kTcStageCols + 64, v1);
          publish();
        }
        if (!ok) {
          give_up();
          break;
        }
      }
    }
  } else if (warp == 14) {
    // ------------------------------ weight loader ------------------------------
    // The whole warp runs the loop (wait outcomes agreed with __all_sync); one
    // elected lane issues every copy and barrier arrival.
    {
      const uint32_t leader = elect_leader();
      auto warp_aborted = [&]() { return __shfl_sync(0xffffffffu, aborted() ? 1 : 0, 0) != 0; };
      TcRing rw(args.w_slots);
      const uint64_t pol = policy_evict_first();
      const int n_slots = nst / args.st_per_slot;
      int issued = 0;
      for (int u = blockIdx.x; u < n_units && !warp_aborted(); u += gridDim.x) {
        if (u + (int)gridDim.x >= n_units) griddep_launch();  // this CTA's last unit
        int e, mt, pos0, n;
        decode_unit(u, e, mt, pos0, n);
        bool ok = true;
        const int y0 = MODE == 0 ? mt * 128 : mt * 256;
        const int y1 = MODE == 0 ? mt * 128 : mt * 256 + 128;
        for (int i = 0; i < n_slots; ++i) {
          if (!warp_wait(&w_empty[rw.s], rw.ph ^ 1)) {
            if (lane == 0) give_up();
            ok = false;
            break;
          }
          mbar_arrive_expect_tx_if(leader, &w_full[rw.s], (uint32_t)args.w_slot_bytes);
          uint8_t* dst = s_w + rw.s * args.w_slot_bytes;
          if (AF == kAMxfp4) {  // code bytes [i * w_inner, +w_inner) of 128 rows, expert e
            tma_load_3d_if(leader, dst, &wmap0, i * args.w_inner, y0, e, &w_full[rw.s], pol);
            tma_load_3d_if(leader, dst + tile_bytes, MODE == 0 ? &wmap1 : &wmap0, i * args.w_inner, y1, e,
                           &w_full[rw.s], pol);
          } else {  // bf16 columns (k mod a_cols) of the stage's two k-blocks
#pragma unroll
            for (int g = 0; g < kTcKG; ++g) {
              const int x = (i * kTcStageK + g * kTcKB) % args.a_cols;
              tma_load_3d_if(leader, dst + g * 16384, &wmap0, x, y0, 0, &w_full[rw.s], pol);
              tma_load_3d_if(leader, dst + tile_bytes + g * 16384, MODE == 0 ? &wmap1 : &wmap0, x, y1, 0,
                             &w_full[rw.s], pol);
            }
          }
          rw.next();
          ++issued;
        }
        if (!ok) break;
      }
      // the last fills must have landed before the CTA exits (on the normal
      // path the A producers have already waited for every one of them)
      for (int i = 0; i < min(issued, rw.n); ++i) {
        const int s = (rw.s - 1 - i + rw.n) % rw.n;
        if (!warp_wait(&w_full[s], s < rw.s ? rw.ph : rw.ph ^ 1) && lane == 0) set_error(kErrWaitTc);
      }
    }
    __syncwarp();
  } else if (warp == 12) {
    // ------------------------------ token loader -------------------------------
    // the whole warp runs the loop; one elected lane issues
    {
      const uint32_t leader = elect_leader();
      auto warp_aborted = [&]() { return __shfl_sync(0xffffffffu, aborted() ? 1 : 0, 0) != 0; };
      TcRing rb(args.b_stages);  // token tiles, released by the MMAs that read them
      int issued = 0;
      for (int u = blockIdx.x; u < n_units && !warp_aborted(); u += gridDim.x) {
        int e, mt, pos0, n;
        decode_unit(u, e, mt, pos0, n);
        bool ok = true;
        for (int st = 0; st < nst; ++st) {
          if (!warp_wait(&b_empty[rb.s], rb.ph ^ 1)) {
            if (lane == 0) give_up();
            ok = false;
            break;
          }
          // one box of n_chunk token rows per k-block (rows past the unit's
          // tokens are loaded but never stored)
          mbar_arrive_expect_tx_if(leader, &b_full[rb.s], (uint32_t)(kTcKG * NC * 128));
          uint8_t* dst = s_b + rb.s * bst;
#pragma unroll
          for (int g = 0; g < kTcKG; ++g) {
            const int col = (st * kTcStageK + g * kTcKB) % args.b_cols;
            tma_load_2d_if(leader, dst + g * atom, &bmap, col, pos0, &b_full[rb.s]);
          }
          rb.next();
          ++issued;
        }
        if (!ok) break;
      }
      for (int i = 0; i < min(issued, rb.n); ++i) {
        const int s = (rb.s - 1 - i + rb.n) % rb.n;
        if (!warp_wait(&b_full[s], s < rb.s ? rb.ph : rb.ph ^ 1) && lane == 0) set_error(kErrWaitTc);
      }
    }
    __syncwarp();
  } else if (warp == 13) {
    // ------------------------------ MMA issuer --------------------------------
    // The whole warp runs the loop (wait outcomes agreed with __all_sync, so
    // it stays converged); an elected lane issues each MMA and commit.
    // Descriptors are built once and advanced by byte offset / 16 (operands
    // lie below 256 KB: the 14-bit address field never carries).
    TcRing rs(args.stages), rb(args.b_stages);
    uint32_t un = 0;
    const uint64_t d_b = sdesc_sw128(smem_u32(s_b));
    auto warp_aborted = [&]() { return __shfl_sync(0xffffffffu, aborted() ? 1 : 0, 0) != 0; };
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && !warp_aborted(); u += gridDim.x, ++un) {
      int e, mt, pos0, n;
      decode_unit(u, e, mt, pos0, n);
      const int n16 = (n + 15) & ~15;
      // MXFP4 weights run as f16 x f16, bf16 weights as bf16 x bf16
      const uint32_t idesc = AF == kAMxfp4 ? idesc_f16_f32(128, n16) : idesc_bf16_f32(128, n16);
      if (!warp_wait(&acc_empty, (un & 1) ^ 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int st = 0; st < nst; ++st) {
        if (!warp_wait(&full[rs.s], rs.ph) || !warp_wait(&b_full[rb.s], rb.ph)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t bd0 = d_b + (uint64_t)((rb.s * bst) >> 4);
        const uint32_t a0 = tbase + a_base + rs.s * kTcStageCols;
        const uint32_t acc1 = tbase + args.acc_cols;
        const uint32_t first = st > 0 ? 1u : 0u;
#pragma unroll
        for (int g = 0; g < kTcKG; ++g) {
          const uint64_t bdg = bd0 + (uint64_t)((g * atom) >> 4);
#pragma unroll
          for (int ks = 0; ks < kTcKB / 16; ++ks) {
            const uint64_t bd = bdg + (uint64_t)(2 * ks);
            const uint32_t acc = (g > 0 || ks > 0) ? 1u : first;
            umma_tmem_a_warp(tbase, a0 + g * 64 + ks * 8, bd, idesc, acc);
            umma_tmem_a_warp(acc1, a0 + g * 64 + 32 + ks * 8, bd, idesc, acc);
          }
        }
        umma_commit_warp(&empty[rs.s]);
        umma_commit_warp(&b_empty[rb.s]);
        if (st == nst - 1) umma_commit_warp(&acc_full);
        rs.next();
        rb.next();
      }
      if (!ok) break;
    }
    if (!ok && lane == 0) give_up();
    // every MMA of this warp done before TMEM is released
    umma_commit_warp(&mma_done);
    if (!warp_wait(&mma_done, 0) && lane == 0) set_error(kErrWaitTc);
  } else if (warp < 4 || (EPI == 8 && warp >= 15)) {
    // ------------------------------ epilogue ----------------------------------
    // MODE 0, MXFP4: h = swiglu(gate, up) in f16 [pos][rows]
    // MODE 0, bf16:  h as a bf16 pair, hi at [pos][col], lo = h - hi at [pos][rows + col]
    // MODE 1:        fp32 [pos][rows], both row tiles
    const int q = warp & 3;             // TMEM lanes 32q..32q+31
    const int half = warp >= 15 ? 1 : 0;  // EPI = 8: the two warps of a quadrant take alternate 16-column chunks
    const int r = q * 32 + lane;
    uint32_t un = 0;
    for (int u = blockIdx.x; u < n_units && !__any_sync(0xffffffffu, aborted() ? 1 : 0); u += gridDim.x, ++un) {
      int e, mt, pos0, n;
      decode_unit(u, e, mt, pos0, n);
      if (!warp_wait(&acc_full, un & 1)) { give_up(); break; }
      tc_fence_after();
      const uint32_t lrow = (uint32_t)(q * 32) << 16;
      // MXFP4: undo the A producers' per-row offsets 2^c_r (rows of acc0 and
      // acc1), written before this unit's first stage
      float s0 = 1.f, s1 = 1.f;
      if (AF == kAMxfp4) {
        s0 = pow2_f32(s_crow[un % kCrowRing][0][r]);
        s1 = pow2_f32(s_crow[un % kCrowRing][1][r]);
      }
      float hmax = 0.f;  // MXFP4 gate/up: the largest |h| of this warp's rows in the unit
      // the accumulator is handed back to the MMA warp as soon as this warp's
      // last columns are in registers (before their SwiGLU and stores): the
      // next unit's MMAs overwrite it
      bool released = false;
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty);
        released = true;
      };
      for (int c0 = 16 * half; c0 < n; c0 += 16 * (EPI / 4)) {
        uint32_t g[16], h[16];
        tmem_ld16(tbase + lrow + c0, g);
        tmem_ld16(tbase + lrow + args.acc_cols + c0, h);
        tmem_ld_wait();
        if (c0 + 16 * (EPI / 4) >= n) release();
        if (MODE == 0) {
          const int col = mt * 128 + r;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < n) {
              const float hv =
                  silu_clamped_swiglu(__uint_as_float(g[j]) * s0, __uint_as_float(h[j]) * s1, args.limit);
              const int64_t o = (int64_t)(pos0 + c0 + j);
              if (AF == kAMxfp4) {
                static_cast<__half*>(args.out)[o * args.rows + col] = __float2half_rn(hv);
                hmax = fmaxf(hmax, fabsf(hv));
              } else {
                const __nv_bfloat16 hi = __float2bfloat16_rn(hv);
                __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.out) + o * 2 * args.rows;
                out[col] = hi;
                out[args.rows + col] = __float2bfloat16_rn(hv - __bfloat162float(hi));
              }
            }
        } else {
          float* out = static_cast<float*>(args.out);
          const int col = mt * 256 + r;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < n) {
              out[(int64_t)(pos0 + c0 + j) * args.rows + col] = __uint_as_float(g[j]) * s0;
              out[(int64_t)(pos0 + c0 + j) * args.rows + col + 128] = __uint_as_float(h[j]) * s1;
            }
        }
      }
      if (MODE == 0 && AF == kAMxfp4) {
        // h travels to the down GEMM in f16: if none of it reaches f16's
        // normal range (2^-14), it kept only subnormal precision -- flagged
        const float m = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(hmax)));
        if (lane == 0 && m > 0.f && m < 6.103515625e-05f) set_error(kErrF16Small);
      }
      if (!released) release();  // a warp with no columns in this unit
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tbase, kTcTmemCols);
  }
}

// True when either half of an f16x2 is infinite.
__device__ __forceinline__ bool f16x2_has_inf(uint32_t h) {
  return (h & 0x7FFFu) == 0x7C00u || ((h >> 16) & 0x7FFFu) == 0x7C00u;
}

// Activations in pair order for the gate/up GEMM: out[pos] = f16(x[perm[pos] /
// K]), rows of h8 groups of 8 values.  Exact for |x| in [2^-17, 65504] (f16
// subnormals carry bf16's 8 bits down to 2^-17); a value beyond 65504 becomes
// inf and the call records device error 0x303.
__global__ void gather_f16_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm, int K, int h8,
                                  int64_t rows, uint4* __restrict__ out) {
  griddep_wait();
  const int64_t n = rows * h8;
  bool inf = false;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / h8;
    const int c = (int)(i - row * h8);
    int64_t pid = perm[row];
    if (kDebug && (pid < 0 || pid >= rows)) {
      set_error(kErrBadIndex);
      pid = 0;
    }
    const uint4 v = x[(int64_t)(pid / K) * h8 + c];
    const uint4 o = make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z), bf16x2_to_f16x2(v.w));
    inf |= f16x2_has_inf(o.x) | f16x2_has_inf(o.y) | f16x2_has_inf(o.z) | f16x2_has_inf(o.w);
    out[i] = o;
  }
  if (inf) set_error(kErrF16Range);
}

// Router weight fp32 [n] -> three bf16 parts hi, mid, lo with w = hi + mid + lo
// (to within 2^-24 |w|): hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid);
// each difference is exact in fp32.  Laid out [rows][3 * cols]: hi | mid | lo.
__global__ void split3_bf16_kernel(const float* __restrict__ w, __nv_bfloat16* __restrict__ out, int rows,
                                   int cols) {
  griddep_wait();
  const int64_t n = (int64_t)rows * cols;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t rr = i / cols, c = i % cols;
    const float v = w[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    __nv_bfloat16* o = out + rr * 3 * cols;
    o[c] = hi;
    o[cols + c] = mid;
    o[2 * cols + c] = lo;
  }
}

}  // namespace moe
