// Grouped expert GEMM on the 5th-generation tensor cores (tcgen05), for the
// prefill / many-token regime.
//
// Per unit = (expert e, token chunk of <= 128 grouped pairs, 128-row tile):
//   MODE 0 (gate/up):  acc0 = Wg[rows] x^T, acc1 = Wu[rows] x^T over K = hidden;
//                      epilogue h = silu(min(acc0, L)) * clamp(acc1, -L, L),
//                      stored in f16 (|h| <= L^2; 11 mantissa bits)
//   MODE 1 (down):     acc0/acc1 = Wd[2 x 128 rows] h^T over K = inter, fp32 out
// MXFP4 operands run as f16 x f16 MMAs (fp32 accumulation): activations come
// in f16 and each weight is dequantised exactly to f16 as v * 2^(e - 127 -
// c_r), c_r = max(0, e_max(row) - 140), with 2^c_r applied to the fp32
// accumulator row in the epilogue.  That is exact whenever a row's E8M0
// exponents span at most 36 octaves, and costs two instructions per pair of
// codes (cvt + multiply), which keeps the tensor cores, not the dequant, the
// limit.  bf16 weights (shared expert, router) are copied as they are.
// ("Model techniques map", row "SwiGLU feed-forward": the clamped SwiGLU;
// "ElytronAI / DeepSeek-v4-Flash", Sizes/Layout: MXFP4 weights, expert xid at
// base + xid * expert_bytes.)
//
// Swap-AB: the weight rows are the MMA's M = 128 dimension and the expert's
// tokens its N dimension (a multiple of 16, <= 128), so a unit needs no token
// padding beyond 16.
//
// Roles (448 threads, one CTA per SM, persistent over units):
//   warps 0-3   epilogue: tcgen05.ld of the two accumulators (TMEM lane
//               quadrant = warp), SwiGLU or copy, global stores;
//   warps 4-11  A producer: thread = one weight row of one of the two tiles;
//               its raw k-blocks arrive through a private cp.async ring; per
//               64-column k-block it converts the 32 code bytes exactly (see
//               above) and writes the 64 values into TMEM with tcgen05.st: the
//               MMA takes its A operand from TMEM, so the weight tiles never
//               touch shared memory;
//   warp 12     token producer: TMA tile::gather4 of the unit's activation rows
//               (bf16, 128-byte swizzle) into a 4-stage shared-memory ring;
//   warp 13     TMEM owner and MMA issuer (one thread): 2 x 4 tcgen05.mma
//               (M=128, N=n16, K=16) per k-block, tcgen05.commit to free stages.
// TMEM (512 columns): acc0 [0,128), acc1 [128,256), A stages [256, 512).
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace moe {

constexpr int kTcThreads = 448;
constexpr int kTcStages = 4;
constexpr int kTcKB = 64;     // k per stage (one 128-byte swizzle atom of bf16)
constexpr int kTcNMax = 128;  // tokens per unit
constexpr int kTcBTile = kTcNMax * kTcKB * 2;  // 16 KB per stage
constexpr int kTcTmemCols = 512;
constexpr int kTcAccCols = 128;
constexpr int kTcAStage = 64;  // TMEM columns per stage: 2 tiles x 32
// Raw A staging: every A-producer thread copies its own weight row's next
// k-blocks with cp.async into a private ring, kRawStagesMx deep for MXFP4
// (32 code bytes per k-block; the row's whole E8M0 row is fetched once per
// unit) and kRawStagesBf deep for bf16 rows (128 bytes per k-block).  Code
// planes are [stage][16-byte chunk][thread], so a warp's 16-byte reads are
// contiguous.
constexpr int kTcAThreads = 256;
constexpr int kRawStagesMx = 6;
constexpr int kRawStagesBf = 3;
constexpr int kScaleRowMax = 128;  // E8M0 bytes per weight row held per producer thread (cols <= 4096)
constexpr int kRawMxBytes = kRawStagesMx * 2 * kTcAThreads * 16 + kTcAThreads * kScaleRowMax;  // 80 KB
constexpr int kRawBfBytes = kRawStagesBf * 8 * kTcAThreads * 16;                          // 96 KB
constexpr int kRawBytes = kRawMxBytes > kRawBfBytes ? kRawMxBytes : kRawBfBytes;
constexpr int kTcSmemUsed = kTcStages * kTcBTile + kRawBytes + 1024 /*align*/ + 8192 /*tables*/;
// requested dynamic shared memory: more than half an SM's, so one CTA per SM
// (each CTA owns all 512 TMEM columns)
constexpr int kTcSmem = kTcSmemUsed;
static_assert(kTcSmem > 114 * 1024 && kTcSmem <= 227 * 1024, "tc_expert shared memory");

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
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
// D[tmem] (+)= A[tmem] * B[smem desc]^T
__device__ __forceinline__ void umma_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
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

// Four rows (r0..r3), 64 bf16 columns from col, of a 2-D tensor map whose box
// is {64, 1} with 128-byte swizzle, into 512 contiguous bytes of shared memory.
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* map, int col, int r0, int r1, int r2,
                                            int r3, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes [%0], [%1, "
      "{%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(col), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(smem_u32(bar))
      : "memory");
}

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

// f16x2 with 2^k in both halves, k in [-24, 15] (subnormal f16 below -14).
__device__ __forceinline__ uint32_t pow2_f16x2(int k) {
  const float f = __uint_as_float((uint32_t)(k + 127) << 23);
  return f32x2_to_f16x2(f, f);
}

__device__ __forceinline__ uint32_t hmul2_bf16(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

enum { kAMxfp4 = 0, kABf16 = 1 };

struct TcArgs {
  const uint8_t* w0;     // MODE 0: gate; MODE 1: down (or any bf16 [rows][a_cols] matrix)
  const uint8_t* w1;     // MODE 0: up
  int64_t expert_bytes;  // stride between experts (MXFP4); 0 for a single bf16 matrix
  int rows;              // rows of one projection (the MMA's M extent)
  int a_cols;            // columns of the weight matrix
  int k_total;           // reduction length: a multiple of a_cols (A column = k mod a_cols)
  int b_cols;            // columns of a B row (B column = k mod b_cols)
  const int32_t* offsets;  // [E+1] grouped pairs; null: one group of n_single rows
  const int32_t* perm;     // B row of pos = perm[pos] / K; null: B row = pos
  int K, E, n_single;
  int n_chunk;           // tokens per unit: multiple of 16, <= kTcNMax
  void* out;             // see the epilogue
  float limit;
};

template <int MODE, int AF>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_expert_kernel(const __grid_constant__ CUtensorMap bmap, const TcArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t a_full[kTcStages], b_full[kTcStages], empty[kTcStages];
  __shared__ __align__(8) uint64_t acc_full, acc_empty;
  __shared__ uint32_t s_taddr;
  __shared__ int32_t s_abort;
  __shared__ int32_t s_rows[kTcNMax];
  __shared__ int16_t s_crow[4][2][128];  // per-row f16 offsets c_r, ring over units

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_raw = smem + kTcStages * kTcBTile;                                    // raw A ring
  int32_t* s_prefix = reinterpret_cast<int32_t*>(s_raw + kRawBytes);               // [E + 1]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool grouped = args.offsets != nullptr;
  const int E = grouped ? args.E : 1;
  const int MT = MODE == 0 ? args.rows / 128 : args.rows / 256;  // row tiles per group
  const int nkb = args.k_total / kTcKB;
  const int NC = args.n_chunk;

  // ---- unit table: units(e) = MT * ceil(n_e / NC), exclusive prefix ----------
  if (warp == 0) {
    int run = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int c = 0;
      if (e < E) {
        const int n = grouped ? args.offsets[e + 1] - args.offsets[e] : args.n_single;
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
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&a_full[s], 8);
      mbar_init(&b_full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&acc_full, 1);
    mbar_init(&acc_empty, 4);
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

  // unit -> (group, row tile, first position, tokens)
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
    const int start = grouped ? args.offsets[e] : 0;
    const int ne = grouped ? args.offsets[e + 1] - start : args.n_single;
    pos0 = start + chunk * NC;
    n = min(NC, ne - chunk * NC);
  };
  auto aborted = [&]() { return *reinterpret_cast<volatile int32_t*>(&s_abort) != 0; };
  auto give_up = [&]() {
    set_error(kErrWaitTc);
    *reinterpret_cast<volatile int32_t*>(&s_abort) = 1;
  };

  if (warp >= 4 && warp < 12) {
    // ------------------------------ A producer ---------------------------------
    const int t = (warp - 4) >> 2, q = warp & 3, r = q * 32 + lane;
    uint32_t it = 0, un_a = 0;
    for (int u = blockIdx.x; u < n_units && !aborted(); u += gridDim.x, ++un_a) {
      int e, mt, pos0, n;
      decode_unit(u, e, mt, pos0, n);
      const int R = MODE == 0 ? mt * 128 + r : mt * 256 + t * 128 + r;
      const uint8_t* blob = (MODE == 0 && t == 1 ? args.w1 : args.w0) + (int64_t)e * args.expert_bytes;
      const int tslot = (warp - 4) * 32 + lane;
      if (AF == kAMxfp4) {
        const uint8_t* nib = blob + (int64_t)R * (args.a_cols / 2);
        const int sr = args.a_cols / 32;  // scale bytes per row (multiple of 4, <= kScaleRowMax)
        const uint8_t* scl = blob + (int64_t)args.rows * (args.a_cols / 2) + (int64_t)R * sr;
        uint8_t* my_sc = s_raw + kRawStagesMx * 2 * kTcAThreads * 16 + tslot * kScaleRowMax;
        auto nib_at = [&](int st, int h) { return s_raw + ((st * 2 + h) * kTcAThreads + tslot) * 16; };
        auto issue = [&](int kb2) {
          cp_async16(nib_at(kb2 % kRawStagesMx, 0), nib + kb2 * 32);
          cp_async16(nib_at(kb2 % kRawStagesMx, 1), nib + kb2 * 32 + 16);
        };
        // the row's E8M0 bytes in one go (first group), then the ring prologue
        if (sr % 16 == 0) {
          for (int i = 0; i < sr; i += 16) cp_async16(my_sc + i, scl + i);
        } else {
          for (int i = 0; i < sr; i += 4)
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(my_sc + i)), "l"(scl + i)
                         : "memory");
        }
        cp_async_commit();
#pragma unroll
        for (int p = 0; p < kRawStagesMx - 1; ++p) {
          if (p < nkb) issue(p);
          cp_async_commit();
        }
        cp_async_wait<kRawStagesMx - 1>();  // the scale group has landed
        // per-row exponent offset keeping v * 2^(e-127-c_r) inside f16
        uint32_t mx = 0;
        for (int i = 0; i < sr; i += 4) mx = __vmaxu4(mx, *reinterpret_cast<const uint32_t*>(my_sc + i));
        mx = __vmaxu4(mx, mx >> 16);
        mx = __vmaxu4(mx, mx >> 8);
        const int crow = max(0, (int)(mx & 0xFFu) - 140);
        s_crow[un_a & 3][t][r] = (int16_t)crow;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          if (kb + kRawStagesMx - 1 < nkb) issue(kb + kRawStagesMx - 1);
          cp_async_commit();
          cp_async_wait<kRawStagesMx - 1>();
          const uint4 c0 = *reinterpret_cast<const uint4*>(nib_at(kb % kRawStagesMx, 0));
          const uint4 c1 = *reinterpret_cast<const uint4*>(nib_at(kb % kRawStagesMx, 1));
          const uint32_t sc = *reinterpret_cast<const uint16_t*>(my_sc + kb * 2);
          const uint32_t e0 = sc & 0xFFu, e1 = sc >> 8;
          uint32_t v[32];
          const uint32_t wds[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
          const uint32_t f0 = pow2_f16x2(max((int)e0 - 127 - crow, -24));
          const uint32_t f1 = pow2_f16x2(max((int)e1 - 127 - crow, -24));
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t hv[4];
            e2m1x8_to_f16x2(wds[c], hv);
#pragma unroll
            for (int b = 0; b < 4; ++b) v[4 * c + b] = hmul2(hv[b], c < 4 ? f0 : f1);
          }
          const int s = it % kTcStages;
          if (!mbar_wait(&empty[s], ((it / kTcStages) & 1) ^ 1)) { give_up(); break; }
          tc_fence_after();
          tmem_st32(tbase + ((uint32_t)(q * 32) << 16) + kTcTmemCols / 2 + s * kTcAStage + t * 32, v);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&a_full[s]);
        }
      } else {
        // bf16 rows, copied as they are; column = k mod a_cols
        const uint8_t* row = blob + (int64_t)R * args.a_cols * 2;
        auto chunk_at = [&](int st, int c) { return s_raw + ((st * 8 + c) * kTcAThreads + tslot) * 16; };
        auto issue = [&](int kb2) {
          const uint8_t* src = row + (int64_t)((kb2 * kTcKB) % args.a_cols) * 2;
#pragma unroll
          for (int c = 0; c < 8; ++c) cp_async16(chunk_at(kb2 % kRawStagesBf, c), src + c * 16);
        };
#pragma unroll
        for (int p = 0; p < kRawStagesBf - 1; ++p) {
          if (p < nkb) issue(p);
          cp_async_commit();
        }
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          if (kb + kRawStagesBf - 1 < nkb) issue(kb + kRawStagesBf - 1);
          cp_async_commit();
          cp_async_wait<kRawStagesBf - 1>();
          uint32_t v[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 w = *reinterpret_cast<const uint4*>(chunk_at(kb % kRawStagesBf, c));
            v[4 * c] = w.x; v[4 * c + 1] = w.y; v[4 * c + 2] = w.z; v[4 * c + 3] = w.w;
          }
          const int s = it % kTcStages;
          if (!mbar_wait(&empty[s], ((it / kTcStages) & 1) ^ 1)) { give_up(); break; }
          tc_fence_after();
          tmem_st32(tbase + ((uint32_t)(q * 32) << 16) + kTcTmemCols / 2 + s * kTcAStage + t * 32, v);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&a_full[s]);
        }
      }
      cp_async_wait<0>();
    }
  } else if (warp == 12) {
    // ------------------------------ token producer ---------------------------
    uint32_t it = 0;
    for (int u = blockIdx.x; u < n_units && !aborted(); u += gridDim.x) {
      int e, mt, pos0, n;
      decode_unit(u, e, mt, pos0, n);
      const int n16 = (n + 15) & ~15;
      for (int j = lane; j < n16; j += 32) {
        const int p = pos0 + min(j, n - 1);  // pad rows repeat the last token
        s_rows[j] = args.perm != nullptr ? args.perm[p] / args.K : p;
      }
      __syncwarp();
      for (int kb = 0; kb < nkb; ++kb, ++it) {
        const int s = it % kTcStages;
        if (lane == 0) {
          if (!mbar_wait(&empty[s], ((it / kTcStages) & 1) ^ 1)) { give_up(); }
          else {
            mbar_arrive_expect_tx(&b_full[s], (uint32_t)n16 * kTcKB * 2);
            uint8_t* dst = smem + s * kTcBTile;
            const int col = (kb * kTcKB) % args.b_cols;
            for (int j = 0; j < n16; j += 4)
              tma_gather4(dst + j * 128, &bmap, col, s_rows[j], s_rows[j + 1], s_rows[j + 2], s_rows[j + 3],
                          &b_full[s]);
          }
        }
        __syncwarp();
        if (aborted()) break;
      }
      __syncwarp();
    }
  } else if (warp == 13) {
    // ------------------------------ MMA issuer --------------------------------
    uint32_t it = 0, un = 0;
    for (int u = blockIdx.x; u < n_units && !aborted(); u += gridDim.x, ++un) {
      int e, mt, pos0, n;
      decode_unit(u, e, mt, pos0, n);
      const int n16 = (n + 15) & ~15;
      // MXFP4 weights run as f16 x f16, bf16 weights as bf16 x bf16
      const uint32_t idesc = AF == kAMxfp4 ? idesc_f16_f32(128, n16) : idesc_bf16_f32(128, n16);
      if (lane == 0) {
        if (!mbar_wait(&acc_empty, (un & 1) ^ 1)) give_up();
        tc_fence_after();
      }
      __syncwarp();
      for (int kb = 0; kb < nkb && !aborted(); ++kb, ++it) {
        const int s = it % kTcStages;
        if (lane == 0) {
          const uint32_t ph = (it / kTcStages) & 1;
          if (!mbar_wait(&a_full[s], ph) || !mbar_wait(&b_full[s], ph)) { give_up(); }
          else {
            tc_fence_after();
            const uint32_t bsa = smem_u32(smem + s * kTcBTile);
            const uint32_t a0 = tbase + kTcTmemCols / 2 + s * kTcAStage;
#pragma unroll
            for (int ks = 0; ks < kTcKB / 16; ++ks) {
              const uint64_t bd = sdesc_sw128(bsa + ks * 32);
              const uint32_t acc = (kb > 0 || ks > 0) ? 1u : 0u;
              umma_tmem_a(tbase, a0 + ks * 8, bd, idesc, acc);
              umma_tmem_a(tbase + kTcAccCols, a0 + 32 + ks * 8, bd, idesc, acc);
            }
            umma_commit(&empty[s]);
            if (kb == nkb - 1) umma_commit(&acc_full);
          }
        }
        __syncwarp();
      }
    }
  } else {
    // ------------------------------ epilogue ----------------------------------
    // MODE 0, MXFP4: h = swiglu(gate, up) in f16 [pos][rows]
    // MODE 0, bf16:  h as a bf16 pair, hi at [pos][col], lo = h - hi at [pos][rows + col]
    // MODE 1:        fp32 [pos][rows], both row tiles
    const int q = warp;  // TMEM lanes 32q..32q+31
    const int r = q * 32 + lane;
    uint32_t un = 0;
    for (int u = blockIdx.x; u < n_units && !aborted(); u += gridDim.x, ++un) {
      int e, mt, pos0, n;
      decode_unit(u, e, mt, pos0, n);
      if (!mbar_wait(&acc_full, un & 1)) { give_up(); break; }
      tc_fence_after();
      const uint32_t lrow = (uint32_t)(q * 32) << 16;
      // MXFP4: undo the A producer's per-row offsets 2^c_r (rows of acc0 and acc1).
      // The producer of a unit's rows wrote them before its first k-block,
      // which precedes acc_full; it cannot be four units ahead of this read.
      float s0 = 1.f, s1 = 1.f;
      if (AF == kAMxfp4) {
        s0 = __uint_as_float((uint32_t)(s_crow[un & 3][0][r] + 127) << 23);
        s1 = __uint_as_float((uint32_t)(s_crow[un & 3][1][r] + 127) << 23);
      }
      for (int c0 = 0; c0 < n; c0 += 16) {
        uint32_t g[16], h[16];
        tmem_ld16(tbase + lrow + c0, g);
        tmem_ld16(tbase + lrow + kTcAccCols + c0, h);
        tmem_ld_wait();
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
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tbase, kTcTmemCols);
  }
}

// Activations bf16 -> f16 (n8 groups of 8, 16-byte aligned): exact for
// |x| in [2^-14, 65504], f16 subnormals below; |x| > 65504 is out of range.
__global__ void bf16_to_f16_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, int64_t n8) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = in[i];
    out[i] = make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z), bf16x2_to_f16x2(v.w));
  }
}

// Router weight fp32 [n] -> three bf16 parts hi, mid, lo with w = hi + mid + lo
// (to within 2^-24 |w|): hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid);
// each difference is exact in fp32.  Laid out [rows][3 * cols]: hi | mid | lo.
__global__ void split3_bf16_kernel(const float* __restrict__ w, __nv_bfloat16* __restrict__ out, int rows,
                                   int cols) {
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
