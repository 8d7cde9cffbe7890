// Grouped MXFP4 expert GEMM on the block-scaled tensor cores
// (tcgen05.mma.kind::mxf8f6f4.block_scale): the path of moe_expert_gemm for
// calls with at most 24 pairs per expert on average (decode and small
// batches).
//
// The weights reach the MMA exactly as stored: E2M1 codes straight from HBM by
// TMA (CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, which widens every 8 bytes of
// packed codes to a 16-byte shared-memory chunk, the operand layout of the
// f8f6f4 kind) and their E8M0 group-32 scales into tensor memory, where the MMA
// applies them.  Nothing dequantises the weights in software.
// ("ElytronAI / DeepSeek-v4-Flash", Layout and Sizes: the E2M1 nibble plane,
// the E8M0 group-32 scale plane, expert xid at base + xid * expert_bytes;
// "Model techniques map", row "SwiGLU feed-forward": the clamped SwiGLU.)
//
// The token operand is E4M3 with its own E8M0 group-32 scales.  Each
// activation v is carried as a sum of `parts` E4M3 terms: term p encodes the
// residual r_p = v - (terms 0 .. p-1) with the block scale 2^(floor(log2(max
// |r_p| over the 32-value group)) - 7) and round-to-nearest-even.  Two terms
// carry a bf16 value exactly (8 significant bits in two 4-bit terms) unless
// the residual of an element falls below the E4M3 normal range of its group;
// h between the GEMMs (fp32 in the epilogue) keeps about 12 significant bits
// with three terms and about 8 with two.  The terms reach the tensor core in
// one of two ways (args.term_acc):
//   stacked  (0): along the MMA's N dimension (N = parts x tokens), summed in
//                 fp32 by the epilogue -- free while N stays small (an MMA of
//                 N <= 64 costs about what one of N 16 does), so decode
//                 batches use it;
//   summed   (1): one MMA per term into the same accumulator columns (the
//                 product is linear in the token operand), N = tokens -- half
//                 the accumulator columns per token, so chunks of 64-128
//                 tokens (and two accumulator sets) fit in TMEM at larger
//                 batches, where the MMA's cost grows with N anyway.
//
// Per unit = (expert e, token chunk of <= n_chunk grouped pairs, row tile):
//   MODE 0 (gate/up): acc0 = Wg[128 rows] x^T, acc1 = Wu[128 rows] x^T over
//                     K = hidden; epilogue h = silu(min(g, L)) * clamp(u, -L, L)
//                     written straight away as the down GEMM's E4M3 terms
//   MODE 1 (down):    acc0/acc1 = Wd[2 x 128 rows] h^T over K = inter; fp32 out
// Swap-AB: weight rows are the MMA's M = 128, token terms its N.
//
// Pipeline stage = KPS (1 or 2) K-tiles of 128: per K-tile both weight tiles
// (2 x 16 KB of shared memory, 2 x 8 KB from HBM) and the unit's token rows of
// every term (N x 128 bytes), all on one mbarrier; the MMA issuer runs 8 MMAs
// of K 32 per K-tile and commits the stage back to the loader.  Scales travel
// in scale stages of G K-tiles through tensor memory.
//
// Roles (320 threads, one CTA per SM, persistent over units):
//   warps 0-3  epilogue (TMEM lane quadrant = warp): tcgen05.ld of the two
//              accumulators, sum of the terms, SwiGLU and E4M3 split (MODE 0)
//              or fp32 stores (MODE 1);
//   warps 4-7  scale writers (lane quadrant = warp - 4): read the E8M0 bytes
//              of the unit's weight rows and token terms with plain loads and
//              tcgen05.st them in the layout the MMA reads (below), every
//              quadrant holding a full copy;
//   warp 8     loader (one thread): TMA boxes of weights and token terms;
//   warp 9     TMEM owner and MMA issuer (the whole warp runs the loop, an
//              elected lane issues each MMA and commit).
// TMEM (512 columns): acc_bufs accumulator sets (set b: acc0 at 2 b acc,
// acc1 at 2 b acc + acc), then the scale ring.  With two sets the epilogue of
// one unit overlaps the MMAs of the next.  A scale stage holds, for K-tile j
// of the stage, the weight scales at column 8j + 4m + c (m = tile, c = row /
// 32) and the token scales at column 8G + tok_cols j + c: stacked, c = N
// index / 32 (4 columns); summed, c = 4 p + token / 32 (4 columns per term).
// Lane i of every quadrant holds rows (or N indices) 32c + i; byte b of a
// column is k-block 4 kt + b, which the MMA selects with the scale-factor id.
#pragma once

#include <cuda.h>
#include <cuda_fp8.h>

#include "tc_expert.cuh"

namespace moe {

constexpr int kMxThreads = 320;
constexpr int kMxKT = 128;           // K of one pipeline stage (one TMA box of codes)
constexpr int kMxTileBytes = 16384;  // shared-memory bytes of one 128 x 128 weight box
constexpr int kMxTileTx = 8192;      // transaction bytes of that box (4 bits per code)
constexpr int kMxMaxStages = 8;
constexpr int kMxMaxSfStages = 4;
constexpr int kMxMaxParts = 3;
constexpr int kMxNMax = 128;   // MMA N: tokens (summed terms) or terms x padded tokens (stacked)
constexpr int kMxMaxBufs = 2;  // accumulator sets

struct MxArgs {
  const uint8_t* w0;     // MODE 0: gate; MODE 1: down
  const uint8_t* w1;     // MODE 0: up
  int64_t expert_bytes;  // stride between experts
  int rows;              // rows of one projection
  int cols;              // columns (the reduction length K)
  const int32_t* offsets;  // [E+1] grouped pairs
  int E;
  int pairs;             // token rows of one term
  int parts;             // E4M3 terms of the token operand
  const uint8_t* b_scale;  // token E8M0 [parts][pairs][cols / 32]
  int n_chunk;           // tokens per unit: multiple of 16
  int term_acc;          // 0: token terms stacked along N; 1: summed into the same columns
  int max_bufs;          // accumulator sets wanted (1 or 2; the plan may give fewer)
  void* out;             // MODE 0: E4M3 terms of h [out_parts][pairs][rows]; MODE 1: fp32 [pairs][rows]
  uint8_t* out_scale;    // MODE 0: E8M0 of h [out_parts][pairs][rows / 32]
  int out_parts;
  float limit;
  // filled in by mx_plan()
  int g;             // K-tiles per scale stage
  int acc_cols;      // TMEM columns per accumulator
  int acc_bufs;      // accumulator sets
  int tok_cols;      // TMEM columns of token scales per K-tile
  int sf_kt;         // TMEM columns per K-tile in a scale stage (8 weight + tok_cols)
  int sf_stages;     // scale stages in TMEM
  int stages;        // shared-memory stages
  int kps;           // K-tiles per shared-memory stage (1 or 2)
  int stage_bytes;   // weights + token rows of one stage (kps K-tiles)
  int tma_scales;    // 1: E8M0 rows arrive by TMA in a shared-memory scale ring
  int sc_slot_bytes; // one scale-ring slot: [2 x 128 weight rows + parts x n_chunk token rows][4 G]
  int off_sc;        // scale ring
  int off_prefix;    // unit prefix + offsets copy
  int smem_bytes;
};

// Ring depths and the shared-memory carve-up of one launch.  False when the
// shape is outside what the kernel implements.
inline bool mx_plan(MxArgs& a, int mode) {
  const int nc = a.n_chunk;
  if (nc < 16 || nc % 16 || a.parts < 1 || a.parts > kMxMaxParts) return false;
  if (a.term_acc != 0 && a.term_acc != 1) return false;
  const int n = a.term_acc ? nc : a.parts * nc;  // the MMA's N
  if (n > kMxNMax) return false;
  if (mode == 0 && (a.out_parts < 1 || a.out_parts > kMxMaxParts)) return false;
  if (a.cols % kMxKT || a.rows % (mode == 0 ? 128 : 256)) return false;
  // 16U4_ALIGN16B tensor maps: strides in multiples of 32 bytes
  if ((a.cols / 2) % 32 || a.expert_bytes % 32 || (a.cols / 32) % 4) return false;
  const int nkt = a.cols / kMxKT;
  a.acc_cols = (n + 31) / 32 * 32;
  a.tok_cols = a.term_acc ? 4 * a.parts : 4;
  a.sf_kt = 8 + a.tok_cols;
  // the most accumulator sets wanted that leave room for two scale stages,
  // with the longest scale stage (G K-tiles) that does
  a.g = 0;
  const int want = a.max_bufs < 1 ? 1 : a.max_bufs < kMxMaxBufs ? a.max_bufs : kMxMaxBufs;
  for (int nb = want; nb >= 1 && a.g == 0; --nb)
    for (int G = 8; G >= 1 && a.g == 0; G /= 2)
      if (nkt % G == 0 && (kTcTmemCols - nb * 2 * a.acc_cols) / (a.sf_kt * G) >= 2) {
        a.g = G;
        a.acc_bufs = nb;
      }
  if (a.g == 0) return false;
  a.sf_stages = (kTcTmemCols - a.acc_bufs * 2 * a.acc_cols) / (a.sf_kt * a.g);
  if (a.sf_stages > kMxMaxSfStages) a.sf_stages = kMxMaxSfStages;
  const int pre = (2 * (a.E + 1) * 4 + 127) / 128 * 128;
  const int budget = kTcSmemMax - 1024;
  // scale rows by TMA: rows of 4 G bytes, a multiple of 16, with row strides
  // (cols / 32 bytes) a multiple of 16; otherwise the scale writers load them
  a.tma_scales = (a.cols / 32) % 16 == 0 && a.g >= 4 ? 1 : 0;
  a.sc_slot_bytes = a.tma_scales ? ((256 + a.parts * nc) * 4 * a.g + 127) / 128 * 128 : 0;
  // stages of two K-tiles where two of them fit beside two scale slots (half
  // the stage handshakes and TMA instructions per weight byte), else one
  const int kt_bytes = 2 * kMxTileBytes + a.parts * nc * 128;  // one K-tile's weights + token rows
  a.kps = nkt % 2 == 0 && a.g % 2 == 0 && 2 * 2 * kt_bytes + 2 * a.sc_slot_bytes + pre <= budget ? 2 : 1;
  a.stage_bytes = a.kps * kt_bytes;
  auto weight_stages = [&]() { return (budget - pre - a.sf_stages * a.sc_slot_bytes) / a.stage_bytes; };
  a.stages = weight_stages();
  while (a.tma_scales && a.stages < 4 && a.sf_stages > 2) {  // keep weight stages over scale slots
    --a.sf_stages;
    a.stages = weight_stages();
  }
  if (a.stages > kMxMaxStages) a.stages = kMxMaxStages;
  if (a.stages < 2) return false;
  a.off_sc = a.stages * a.stage_bytes;
  a.off_prefix = a.off_sc + a.sf_stages * a.sc_slot_bytes;
  a.smem_bytes = a.off_prefix + pre + 1024;
  // every CTA allocates all 512 TMEM columns, so no second CTA may share its
  // SM: more than half of the SM's shared memory guarantees that
  return a.smem_bytes <= kTcSmemMax && a.smem_bytes > kTcSmemMax / 2;
}

// Box {x, y, z} of a 3-D tensor map into shared memory (no cache hint).
__device__ __forceinline__ void tma_load_3d_nohint(void* dst, const CUtensorMap* map, int x, int y, int z,
                                                   uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// Box {x, y, z, w} of a 4-D tensor map into shared memory (no cache hint).
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int x, int y, int z, int w,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
      "%5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
      : "memory");
}
// The same with an L2 cache hint.
__device__ __forceinline__ void tma_load_4d_hint(void* dst, const CUtensorMap* map, int x, int y, int z, int w,
                                                 uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, "
      "{%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_nohint_if(uint32_t leader, void* dst, const CUtensorMap* map, int x, int y,
                                                      int z, uint64_t* bar) {
  asm volatile(
      "{\n .reg .pred e;\n setp.ne.b32 e, %0, 0;\n"
      " @e cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%1], [%2, {%3, %4, %5}], "
      "[%6];\n}\n" ::"r"(leader),
      "r"(smem_u32(dst)), "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_4d_if(uint32_t leader, void* dst, const CUtensorMap* map, int x, int y, int z,
                                               int w, uint64_t* bar) {
  asm volatile(
      "{\n .reg .pred e;\n setp.ne.b32 e, %0, 0;\n"
      " @e cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%1], [%2, {%3, %4, %5, "
      "%6}], [%7];\n}\n" ::"r"(leader),
      "r"(smem_u32(dst)), "l"(map), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_4d_hint_if(uint32_t leader, void* dst, const CUtensorMap* map, int x, int y,
                                                    int z, int w, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "{\n .reg .pred e;\n setp.ne.b32 e, %0, 0;\n"
      " @e cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%1], [%2, "
      "{%3, %4, %5, %6}], [%7], %8;\n}\n" ::"r"(leader),
      "r"(smem_u32(dst)), "l"(map), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Instruction descriptor, kind::mxf8f6f4 block-scaled: A E2M1, B E4M3, both
// K-major, E8M0 scales, fp32 D; scale-factor ids in bits 4-5 (B) and 29-30 (A).
__host__ __device__ constexpr uint32_t idesc_mx_e2m1_e4m3(int M, int N) {
  return (5u << 7) | (0u << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= (A[smem] * SFA) (B[smem] * SFB)^T, scales from TMEM.  Called
// by all 32 lanes of a converged warp with the same operands; one lane, chosen
// by elect.sync, issues the MMA.  Issuing from a whole warp lets the operands
// stay warp-uniform: a lone thread in a lane-0 branch issues one of these
// every ~80 cycles whatever N is, a warp with an elected lane every ~45
// (N <= 64; measured with the loop shape below on a B200).
__device__ __forceinline__ void umma_mx_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate, uint32_t sfa_tmem, uint32_t sfb_tmem) {
  asm volatile(
      "{\n .reg .pred p, e;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// G consecutive 32-bit words (4 * G bytes, 16-byte aligned for G >= 4).
template <int G>
__device__ __forceinline__ void load_words(const uint8_t* p, uint32_t* w) {
  if constexpr (G == 8) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(p)), b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else if constexpr (G == 4) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
  } else if constexpr (G == 2) {
    const uint2 a = __ldg(reinterpret_cast<const uint2*>(p));
    w[0] = a.x; w[1] = a.y;
  } else {
    w[0] = __ldg(reinterpret_cast<const uint32_t*>(p));
  }
}

// The same from shared memory (a generic pointer into it).
template <int G>
__device__ __forceinline__ void load_words_smem(const uint8_t* p, uint32_t* w) {
  if constexpr (G >= 4) {
#pragma unroll
    for (int i = 0; i < G / 4; ++i) {
      const uint4 a = reinterpret_cast<const uint4*>(p)[i];
      w[4 * i] = a.x; w[4 * i + 1] = a.y; w[4 * i + 2] = a.z; w[4 * i + 3] = a.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < G; ++i) w[i] = reinterpret_cast<const uint32_t*>(p)[i];
  }
}

// E8M0 block scale of a group whose largest magnitude has fp32 bits `amax`:
// 2^(floor(log2 amax) - 7), so every |v| / scale is below 256 and rounds to at
// most 256, inside the E4M3 range (448); 2^-127 for groups under 2^-120 (and
// all-zero groups).
__device__ __forceinline__ int e8m0_of_amax(uint32_t amax) { return max((int)(amax >> 23) - 7, 0); }
// 2^(127 - s) and 2^(s - 127) for an E8M0 byte s in [0, 247]
__device__ __forceinline__ float e8m0_inv(int s) { return __uint_as_float((uint32_t)(254 - s) << 23); }
__device__ __forceinline__ float e8m0_val(int s) {
  return s > 0 ? __uint_as_float((uint32_t)s << 23) : __uint_as_float(0x00400000u);
}
__device__ __forceinline__ uint32_t e4m3_rn(float v) {
  return (uint32_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float e4m3_val(uint32_t code) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3)));
}

// KPS (K-tiles per stage) and SUMMED (term layout) are template parameters so
// that the MMA issue block is straight-line code: with either one a runtime
// loop bound around the MMAs, a microbenchmark of this issue loop runs at 111
// cycles per MMA; with both fixed at compile time (loops unrolled), at 52.
template <int MODE, int G, int KPS, bool SUMMED>
__global__ void __launch_bounds__(kMxThreads, 1)
    mx_expert_kernel(const __grid_constant__ CUtensorMap bmap, const __grid_constant__ CUtensorMap wmap0,
                     const __grid_constant__ CUtensorMap wmap1, const __grid_constant__ CUtensorMap smap0,
                     const __grid_constant__ CUtensorMap smap1, const __grid_constant__ CUtensorMap tsmap,
                     const MxArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kMxMaxStages], empty[kMxMaxStages];
  __shared__ __align__(8) uint64_t sf_full[kMxMaxSfStages], sf_empty[kMxMaxSfStages];
  __shared__ __align__(8) uint64_t sc_full[kMxMaxSfStages], sc_empty[kMxMaxSfStages];
  __shared__ __align__(8) uint64_t acc_full[kMxMaxBufs], acc_empty[kMxMaxBufs], mma_done;
  __shared__ uint32_t s_taddr;
  __shared__ int32_t s_abort;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  int32_t* s_prefix = reinterpret_cast<int32_t*>(smem + args.off_prefix);  // [E + 1] units before group e
  int32_t* s_off = s_prefix + args.E + 1;                                   // [E + 1] copy of offsets

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = args.E;
  const int MT = MODE == 0 ? args.rows / 128 : args.rows / 256;  // row tiles per expert
  const int nkt = args.cols / kMxKT;                             // K-tiles per unit
  const int NC = args.n_chunk;
  const int P = args.parts;
  const int sr = args.cols / 32;  // E8M0 bytes per weight row and per token row
  const int NB = args.acc_bufs;
  constexpr bool summed = SUMMED;
  const int TC = args.tok_cols;
  const uint32_t sf_base = NB * 2 * args.acc_cols;
  const int sf_cols = args.sf_kt * G;

  // ---- unit table: units(e) = MT * ceil(n_e / NC), exclusive prefix ----------
  griddep_wait();  // the offsets and token terms come from earlier kernels of the stream
  for (int i = tid; i <= E; i += blockDim.x) s_off[i] = args.offsets[i];
  __syncthreads();
  if (kDebug) {  // offsets must run from 0 to the pair count without decreasing
    bool bad = false;
    for (int i = tid; i < E; i += blockDim.x) bad |= s_off[i] > s_off[i + 1];
    if (tid == 0) bad |= s_off[0] != 0 || s_off[E] != args.pairs;
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
      if (e < E) c = MT * ((s_off[e + 1] - s_off[e] + NC - 1) / NC);
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
    for (int s = 0; s < kMxMaxStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < kMxMaxSfStages; ++s) {
      mbar_init(&sf_full[s], 4);  // one arrival per scale-writer warp
      mbar_init(&sf_empty[s], 1);
      mbar_init(&sc_full[s], 1);
      mbar_init(&sc_empty[s], 4);  // one arrival per scale-writer warp
    }
    for (int b = 0; b < kMxMaxBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);  // one arrival per epilogue warp
    }
    mbar_init(&mma_done, 1);
    s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(&s_taddr, kTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = s_taddr;
  const int n_units = s_prefix[E];
  // the next kernel may begin launching once every CTA has started its last
  // unit (its CTAs take an SM only as this kernel's CTAs leave)
  if (tid == 0 && (int)blockIdx.x + (int)gridDim.x >= n_units) griddep_launch();

  // unit -> (expert, row tile, first grouped pair, tokens)
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
    pos0 = s_off[e] + chunk * NC;
    n = min(NC, s_off[e + 1] - pos0);
  };
  auto aborted = [&]() { return *reinterpret_cast<volatile int32_t*>(&s_abort) != 0; };
  auto give_up = [&]() {
    set_error(kErrWaitTc);
    *reinterpret_cast<volatile int32_t*>(&s_abort) = 1;
  };
  auto warp_wait = [&](uint64_t* bar, uint32_t ph) {
    return __all_sync(0xffffffffu, mbar_wait(bar, ph) ? 1 : 0) != 0;
  };

  if (warp == 8) {
    // ------------------------------ loader -------------------------------------
    // The whole warp runs the loop (wait outcomes agreed with __all_sync); one
    // elected lane issues every copy and barrier arrival.
    {
      const uint32_t leader = elect_leader();
      TcRing rs(args.stages);
      const uint64_t pol = policy_evict_first();
      int issued = 0, sc_issued = 0;
      TcRing rc(args.sf_stages);  // scale-ring slots, one per scale stage
      // The E8M0 rows of a scale stage (both weight tiles, then every term's
      // token rows, [row][4 G bytes]) run one scale stage ahead of the weights,
      // across unit boundaries, so the scale writers find them landed.  The
      // scale cursor (su, sg) is the next scale stage to load.
      const int ng = nkt / G;
      int su = blockIdx.x, sg = 0, s_e = 0, s_y0 = 0, s_pos0 = 0;
      auto scale_unit = [&]() {
        int mt_, n_;
        decode_unit(su, s_e, mt_, s_pos0, n_);
        s_y0 = MODE == 0 ? mt_ * 128 : mt_ * 256;
      };
      if (su < n_units) scale_unit();
      // issue every scale stage up to (u_lim, g_lim) inclusive; false on a
      // wait that gave up
      auto scales_upto = [&](int u_lim, int g_lim) {
        while (su < n_units && (su < u_lim || (su == u_lim && sg <= g_lim))) {
          if (!warp_wait(&sc_empty[rc.s], rc.ph ^ 1)) return false;
          uint8_t* sd = smem + args.off_sc + rc.s * args.sc_slot_bytes;
          const int xs = 4 * G * sg;
          mbar_arrive_expect_tx_if(leader, &sc_full[rc.s], (uint32_t)((256 + P * NC) * 4 * G));
          tma_load_3d_if(leader, sd, &smap0, xs, s_y0, s_e, &sc_full[rc.s], pol);  // MODE 1: both tiles' 256 rows
          if (MODE == 0) tma_load_3d_if(leader, sd + 128 * 4 * G, &smap1, xs, s_y0, s_e, &sc_full[rc.s], pol);
          tma_load_3d_nohint_if(leader, sd + 256 * 4 * G, &tsmap, xs, s_pos0, 0, &sc_full[rc.s]);  // [term][n_chunk rows]
          rc.next();
          ++sc_issued;
          if (++sg == ng) {
            sg = 0;
            su += gridDim.x;
            if (su < n_units) scale_unit();
          }
        }
        return true;
      };
      auto warp_aborted = [&]() { return __shfl_sync(0xffffffffu, aborted() ? 1 : 0, 0) != 0; };
      for (int u = blockIdx.x; u < n_units && !warp_aborted(); u += gridDim.x) {
        if (u + (int)gridDim.x >= n_units) griddep_launch();  // this CTA's last unit
        int e, mt, pos0, n;
        decode_unit(u, e, mt, pos0, n);
        (void)n;
        const int y0 = MODE == 0 ? mt * 128 : mt * 256;
        // one stage = KPS K-tiles: both weight tiles' KPS K-tiles (MODE 0: a
        // box per projection; MODE 1: one box of 256 rows), then one box of
        // every term's n_chunk token rows for the KPS K-tiles (rows past the
        // unit's tokens are loaded but never stored)
        const uint32_t tx = (uint32_t)KPS * (2 * kMxTileTx + (uint32_t)(P * NC * 128));
        bool ok = true;
        for (int kt = 0; kt < nkt; kt += KPS) {
          if (args.tma_scales && kt % G == 0) {
            const int g1 = kt / G + 1;  // this scale stage and the next one
            if (!(g1 < ng ? scales_upto(u, g1) : scales_upto(u + (int)gridDim.x, 0))) {
              if (lane == 0) give_up();
              ok = false;
              break;
            }
          }
          if (!warp_wait(&empty[rs.s], rs.ph ^ 1)) {
            if (lane == 0) give_up();
            ok = false;
            break;
          }
          mbar_arrive_expect_tx_if(leader, &full[rs.s], tx);
          uint8_t* dst = smem + rs.s * args.stage_bytes;
          // [KPS][rows][128 B] per projection (MODE 1: [KPS][256][128 B])
          tma_load_4d_hint_if(leader, dst, &wmap0, 0, y0, kt, e, &full[rs.s], pol);
          if (MODE == 0) tma_load_4d_hint_if(leader, dst + KPS * kMxTileBytes, &wmap1, 0, y0, kt, e, &full[rs.s], pol);
          tma_load_4d_if(leader, dst + 2 * KPS * kMxTileBytes, &bmap, 0, pos0, 0, kt, &full[rs.s]);  // [KPS][P][NC][128 B]
          rs.next();
          ++issued;
        }
        if (!ok) break;
      }
      // the last fills must have landed before the CTA exits
      for (int i = 0; i < min(issued, rs.n); ++i) {
        const int s = (rs.s - 1 - i + rs.n) % rs.n;
        if (!warp_wait(&full[s], s < rs.s ? rs.ph : rs.ph ^ 1) && lane == 0) set_error(kErrWaitTc);
      }
      for (int i = 0; i < min(sc_issued, rc.n); ++i) {
        const int s = (rc.s - 1 - i + rc.n) % rc.n;
        if (!warp_wait(&sc_full[s], s < rc.s ? rc.ph : rc.ph ^ 1) && lane == 0) set_error(kErrWaitTc);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------ MMA issuer ----------------------------------
    // The whole warp runs the loop (every wait's outcome is agreed with
    // __all_sync, so the warp stays converged); an elected lane issues each
    // MMA and commit.  Descriptors are built once and advanced by adding byte
    // offsets / 16 to their 14-bit address field (every operand lies below
    // 256 KB, so the field never carries into the constant upper bits).
    TcRing rs(args.stages), rf(args.sf_stages);
    uint32_t un = 0;
    bool ok = true;
    const uint64_t d_smem = sdesc_sw128(smem_u32(smem));
    auto warp_aborted = [&]() { return __shfl_sync(0xffffffffu, aborted() ? 1 : 0, 0) != 0; };
    for (int u = blockIdx.x; u < n_units && ok && !warp_aborted(); u += gridDim.x, ++un) {
      int e, mt, pos0, n;
      decode_unit(u, e, mt, pos0, n);
      const int n16 = (n + 15) & ~15;
      // summed terms: one MMA of N = tokens per term; stacked: one of N = P x
      // n_chunk over every term's block of token rows
      const uint32_t idesc = idesc_mx_e2m1_e4m3(128, summed ? n16 : P * NC);
      const int b = (int)(un % (uint32_t)NB);
      const uint32_t acc0 = tbase + (uint32_t)(b * 2 * args.acc_cols), acc1 = acc0 + args.acc_cols;
      if (!warp_wait(&acc_empty[b], ((un / NB) & 1) ^ 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int kt0 = 0; kt0 < nkt && ok; kt0 += KPS) {
        if (!warp_wait(&full[rs.s], rs.ph)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // this stage's operands: MODE 0 gate K-tiles at 0, up K-tiles at KPS x
        // 16 KB; MODE 1 K-tile kk's 256 rows at kk x 32 KB (tile 1 16 KB in);
        // token rows at 2 KPS x 16 KB, [kk][term][n_chunk][128 B]; a k-block
        // is 32 bytes
        const uint64_t ds = d_smem + (uint64_t)((rs.s * args.stage_bytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < KPS; ++kk) {
          const int kt = kt0 + kk, j = kt % G;
          if (j == 0) {
            if (!warp_wait(&sf_full[rf.s], rf.ph)) {
              ok = false;
              break;
            }
            tc_fence_after();  // the scale writers' tcgen05.st before this stage's MMAs
          }
          const uint64_t da0 = ds + (uint64_t)((MODE == 0 ? kk * kMxTileBytes : kk * 2 * kMxTileBytes) >> 4);
          const uint64_t da1 = MODE == 0 ? da0 + (uint64_t)((KPS * kMxTileBytes) >> 4) : da0 + (kMxTileBytes >> 4);
          const uint64_t db = ds + (uint64_t)((2 * KPS * kMxTileBytes + kk * P * NC * 128) >> 4);
          const uint32_t sfc = tbase + sf_base + rf.s * sf_cols;
          const uint32_t sfa0 = sfc + 8 * j, sfa1 = sfa0 + 4, sfb0 = sfc + 8 * G + TC * j;
          const uint32_t first = kt > 0 ? 1u : 0u;
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            const uint32_t id = idesc | ((uint32_t)kb << 29) | ((uint32_t)kb << 4);
            const uint32_t sel = (uint32_t)kb << 30;
            const uint64_t ko = (uint64_t)(2 * kb);
            if constexpr (SUMMED) {
#pragma unroll
              for (int p = 0; p < kMxMaxParts; ++p) {
                if (p < P) {
                  const uint64_t bd = db + ko + (uint64_t)((p * NC * 128) >> 4);
                  const uint32_t sfb = (sfb0 + 4 * p) | sel;
                  const uint32_t acc = (kb > 0 || p > 0) ? 1u : first;
                  umma_mx_warp(acc0, da0 + ko, bd, id, acc, sfa0 | sel, sfb);
                  umma_mx_warp(acc1, da1 + ko, bd, id, acc, sfa1 | sel, sfb);
                }
              }
            } else {
              const uint32_t acc = kb > 0 ? 1u : first;
              umma_mx_warp(acc0, da0 + ko, db + ko, id, acc, sfa0 | sel, sfb0 | sel);
              umma_mx_warp(acc1, da1 + ko, db + ko, id, acc, sfa1 | sel, sfb0 | sel);
            }
          }
          if (j == G - 1) {
            umma_commit_warp(&sf_empty[rf.s]);
            rf.next();
          }
          if (kt == nkt - 1) umma_commit_warp(&acc_full[b]);
        }
        if (!ok) break;
        umma_commit_warp(&empty[rs.s]);
        rs.next();
      }
    }
    if (!ok && lane == 0) give_up();
    // every MMA of this warp done before TMEM is released
    umma_commit_warp(&mma_done);
    if (!warp_wait(&mma_done, 0) && lane == 0) set_error(kErrWaitTc);
  } else if (warp >= 4) {
    // ------------------------------ scale writers --------------------------------
    const int q = warp & 3;
    const uint32_t lrow = (uint32_t)(q * 32) << 16;
    const int64_t plane = (int64_t)args.rows * (args.cols / 2);
    TcRing rf(args.sf_stages);
    for (int u = blockIdx.x; u < n_units && !__any_sync(0xffffffffu, aborted() ? 1 : 0); u += gridDim.x) {
      int e, mt, pos0, n;
      decode_unit(u, e, mt, pos0, n);
      bool ok = true;
      for (int g = 0; g < nkt / G; ++g) {
        // the stage's E8M0 rows: from the scale ring (TMA) or straight from memory
        const uint8_t* ss = nullptr;
        if (args.tma_scales) {
          if (!warp_wait(&sc_full[rf.s], rf.ph)) {
            ok = false;
            break;
          }
          ss = smem + args.off_sc + rf.s * args.sc_slot_bytes;
        }
        // weight scales: a[8 j + 4 m + c] = bytes 4 (G g + j) .. +3 of row 32 c + lane of tile m
        uint32_t a[8 * G], b[4 * G];
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t w[G];
            if (ss != nullptr) {
              load_words_smem<G>(ss + (128 * m + 32 * c + lane) * 4 * G, w);
            } else {
              const int R = MODE == 0 ? mt * 128 + 32 * c + lane : mt * 256 + 128 * m + 32 * c + lane;
              load_words<G>((MODE == 0 && m == 1 ? args.w1 : args.w0) + (int64_t)e * args.expert_bytes + plane +
                                (int64_t)R * sr + 4 * G * g,
                            w);
            }
#pragma unroll
            for (int j = 0; j < G; ++j) a[8 * j + 4 * m + c] = w[j];
          }
        // token scales, 4 columns at a time: stacked, column c holds N index
        // 32 c + lane (term nn / n_chunk, token nn mod n_chunk); summed, block p
        // of 4 columns holds term p, column c of it token 32 c + lane
        auto load_tokens = [&](int q4) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            int p, t;
            if (summed) {
              p = q4;
              t = 32 * c + lane;
            } else {
              const int nn = 32 * c + lane;
              p = nn / NC;
              t = nn - p * NC;
            }
            uint32_t w[G];
#pragma unroll
            for (int j = 0; j < G; ++j) w[j] = 0;
            if (p < P && t < n) {
              if (ss != nullptr) load_words_smem<G>(ss + (256 + p * NC + t) * 4 * G, w);
              else load_words<G>(args.b_scale + ((int64_t)p * args.pairs + pos0 + t) * sr + 4 * G * g, w);
            }
#pragma unroll
            for (int j = 0; j < G; ++j) b[4 * j + c] = w[j];
          }
        };
        load_tokens(0);  // in flight with the weight scales while the stage frees up
        if (!warp_wait(&sf_empty[rf.s], rf.ph ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t col = tbase + lrow + sf_base + rf.s * sf_cols;
#pragma unroll
        for (int i = 0; i < G; ++i) tmem_st8(col + 8 * i, a + 8 * i);
        for (int q4 = 0; q4 < TC / 4; ++q4) {
          if (q4 > 0) {
            tmem_st_wait();  // the previous group's registers are stored before b is refilled
            load_tokens(q4);
          }
#pragma unroll
          for (int j = 0; j < G; ++j)
            asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                             col + 8 * G + TC * j + 4 * q4),
                         "r"(b[4 * j]), "r"(b[4 * j + 1]), "r"(b[4 * j + 2]), "r"(b[4 * j + 3])
                         : "memory");
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sf_full[rf.s]);
          if (ss != nullptr) mbar_arrive(&sc_empty[rf.s]);  // every read of the slot is done
        }
        rf.next();
      }
      if (!ok) {
        give_up();
        break;
      }
    }
  } else {
    // ------------------------------ epilogue ------------------------------------
    const int q = warp;  // TMEM lanes 32q .. 32q + 31
    const uint32_t lrow = (uint32_t)(q * 32) << 16;
    uint32_t un = 0;
    for (int u = blockIdx.x; u < n_units && !__any_sync(0xffffffffu, aborted() ? 1 : 0); u += gridDim.x, ++un) {
      int e, mt, pos0, n;
      decode_unit(u, e, mt, pos0, n);
      const int b = (int)(un % (uint32_t)NB);
      const uint32_t accb = tbase + lrow + (uint32_t)(b * 2 * args.acc_cols);
      if (!warp_wait(&acc_full[b], (un / NB) & 1)) {
        give_up();
        break;
      }
      tc_fence_after();
      const int pe = summed ? 1 : P;  // stacked terms are summed here
      for (int c0 = 0; c0 < n; c0 += 16) {
        float g[16], v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) g[j] = v[j] = 0.f;
        for (int p = 0; p < pe; ++p) {
          uint32_t t0[16], t1[16];
          tmem_ld16(accb + p * NC + c0, t0);
          tmem_ld16(accb + args.acc_cols + p * NC + c0, t1);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            g[j] += __uint_as_float(t0[j]);
            v[j] += __uint_as_float(t1[j]);
          }
        }
        if (MODE == 0) {
          // h of row col for 16 tokens, split into E4M3 terms; the 32 lanes of
          // the warp are one group of 32 h values of a token (the down GEMM's
          // k).  The 16 tokens are independent, so each step runs for all of
          // them before the next (their reductions and conversions overlap);
          // tokens past the chunk are computed and not stored.
          const int col = mt * 128 + q * 32 + lane;
          uint8_t* hq = static_cast<uint8_t*>(args.out);
          float r[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) r[j] = silu_clamped_swiglu(g[j], v[j], args.limit);
          const int nj = n - c0;  // tokens of this 16-chunk that exist (warp-uniform)
          for (int p = 0; p < args.out_parts; ++p) {
            uint32_t amax[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) amax[j] = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(r[j])));
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int s = e8m0_of_amax(amax[j]);
              const uint32_t code = e4m3_rn(r[j] * e8m0_inv(s));
              if (j < nj) {
                const int64_t row = (int64_t)p * args.pairs + pos0 + c0 + j;
                hq[row * args.rows + col] = (uint8_t)code;
                if (lane == 0) args.out_scale[row * (args.rows / 32) + col / 32] = (uint8_t)s;
              }
              r[j] -= e4m3_val(code) * e8m0_val(s);
            }
          }
        } else {
          float* out = static_cast<float*>(args.out);
          const int col = mt * 256 + q * 32 + lane;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < n) {
              out[(int64_t)(pos0 + c0 + j) * args.rows + col] = g[j];
              out[(int64_t)(pos0 + c0 + j) * args.rows + col + 128] = v[j];
            }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tbase, kTcTmemCols);
  }
}

// Activations of every pair in expert order as `parts` E4M3 terms with E8M0
// group-32 scales: q[p][pos][k], sc[p][pos][k / 32] for x[perm[pos] / top_k].
// One thread per 8 values; the 4 threads of a 32-value group are adjacent lanes.
__global__ void gather_split_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm, int top_k,
                                    int hidden, int64_t pairs, int parts, uint8_t* __restrict__ q,
                                    uint8_t* __restrict__ sc) {
  griddep_wait();
  const int h8 = hidden / 8;
  const int64_t n = pairs * h8;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int lane = threadIdx.x & 31;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < n; base += stride) {
    const int64_t i = base + lane;
    const bool ok = i < n;  // whole 4-lane groups: n is a multiple of 4
    float v[8];
    int64_t pos = 0;
    int c8 = 0;
    if (ok) {
      pos = i / h8;
      c8 = (int)(i - pos * h8);
      int64_t pid = perm[pos];
      if (kDebug && (pid < 0 || pid >= pairs)) {
        set_error(kErrBadIndex);
        pid = 0;
      }
      const int64_t t = pid / top_k;
      const uint4 w = x[t * h8 + c8];
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[2 * k] = __uint_as_float(ws[k] << 16);
        v[2 * k + 1] = __uint_as_float(ws[k] & 0xFFFF0000u);
      }
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = 0.f;
    }
    for (int p = 0; p < parts; ++p) {
      uint32_t amax = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) amax = max(amax, __float_as_uint(fabsf(v[k])));
      amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      const int s = e8m0_of_amax(amax);
      const float inv = e8m0_inv(s), val = e8m0_val(s);
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t code = e4m3_rn(v[k] * inv);
        if (k < 4) lo |= code << (8 * k);
        else hi |= code << (8 * (k - 4));
        v[k] -= e4m3_val(code) * val;
      }
      if (ok) {
        const int64_t row = (int64_t)p * pairs + pos;
        reinterpret_cast<uint2*>(q + row * hidden)[c8] = make_uint2(lo, hi);
        if ((c8 & 3) == 0) sc[row * (hidden / 32) + c8 / 4] = (uint8_t)s;
      }
    }
  }
}

}  // namespace moe
