// Launch arguments of moe_expert_gemm's two paths, on the host only (no CUDA
// call): the path choice from T, the token chunk, the E4M3 term counts, the
// workspace carve-up and the pipeline plans.  moe_expert_gemm launches what
// these functions fill in; a CPU test checks them for every token count.
#pragma once

#include <cstddef>
#include <cstdint>

#include "mx_expert.cuh"
#include "tc_expert.cuh"

namespace moe {

inline size_t ws_round_up(size_t v) { return (v + 255) / 256 * 256; }

// Tokens per expert-kernel unit: the accumulator columns a unit reserves.  A
// small chunk (few pairs per expert) leaves TMEM and shared memory for deeper
// rings; a chunk below an expert's pair count makes its weights stream again.
inline int expert_chunk(int T, int K, int E) {
  const int64_t avg = ((int64_t)T * K + E - 1) / E;
  return avg <= 8 ? 32 : avg <= 24 ? 64 : kTcNMax;
}

// Mean pairs per expert up to which moe_expert_gemm takes the block-scaled
// kernel; above it, the kernel that dequantises to f16.  Measured on one B200
// (expert call, same box): at 8, 12, 16, 20 and 24 pairs per expert the
// block-scaled kernel in 32-pair chunks takes 762 / 777 / 808 / 842 / 890 us
// against 1319 / 1323 / 1329 / 1334 / 1341 us dequantising; at 32, 48, 64 and
// 96 the dequantising kernel wins (1393 / 1422 / 1469 / 1605 us against 1788 /
// 1987 / 2161 / 2544 us for the block-scaled kernel's summed layout).
constexpr int kBlockScaledMaxAvg = 24;

// Path choice from the host-known T: with few pairs per expert (32-pair
// chunks: decode and small batches) the weights stream through the
// block-scaled kernel; with many, the kernel that dequantises to f16 keeps
// 128-token units, double the epilogue warps and one read of each expert's
// weights.
inline bool use_block_scaled(int T, int K, int E) {
  return ((int64_t)T * K + E - 1) / E <= kBlockScaledMaxAvg;
}

// E4M3 terms of the activations (exact for bf16) and of h between the GEMMs
// on the block-scaled path (three terms of h: about 12 significant bits).
constexpr int kXTerms = 2;
constexpr int kHTerms = 3;

// Token layout of the block-scaled kernel by mean pairs per expert: on its
// path (up to kBlockScaledMaxAvg), the terms stacked along N in 16-pair (up
// to 4 pairs per expert) or 32-pair chunks (N = terms x chunk) with two
// accumulator sets; an expert with more pairs than a chunk takes more chunks.  Above, the layout the
// kernel was measured in against the dequantising one at prefill (not on any
// path): the terms summed into one accumulator in 128-pair chunks (N 128;
// one set fits), so an expert's weights are read once per 128 of its pairs.
struct MxLayout {
  int chunk, term_acc, max_bufs;
};
// Two accumulator sets at decode let a unit's MMAs start while the previous
// unit's epilogue runs (measured on one B200: the batch-64 expert call 1088 ->
// 1003 us).
constexpr int kMxDecodeBufs = 2;  // accumulator sets of the stacked (decode) layout
inline MxLayout mx_layout(int T, int K, int E) {
  const int64_t avg = ((int64_t)T * K + E - 1) / E;
  // up to 4 pairs per expert (decode batches up to 170 tokens at V4): 16-pair
  // chunks, N 32 and 48 -- smaller MMAs and token boxes; measured on one B200
  // (decode step, same box, two runs each): 65.8k -> 71.4k tokens/s, the
  // batch-64 expert call 0.67 -> 0.73 of the copy peak
  if (avg <= 4) return {16, 0, kMxDecodeBufs};
  if (avg <= kBlockScaledMaxAvg) return {32, 0, kMxDecodeBufs};
  return {128, 1, 2};
}

// The block-scaled path's workspace: E4M3 terms and E8M0 scales of the pairs'
// activations in expert order, then of h: [2][pairs][hidden],
// [2][pairs][hidden / 32], [3][pairs][inter], [3][pairs][inter / 32] bytes.
// The dequantising path uses a prefix of it (x in f16 [pairs][hidden], then
// h in f16 [pairs][inter]: hidden / 16 + inter + 3 inter / 32 bytes fewer per
// pair), so the size grows with T whichever path T selects and a workspace
// sized for some T serves every smaller T.
inline size_t expert_gemm_ws_bytes(const moe_dims& dims, int T) {
  const size_t pairs = (size_t)T * dims.top_k, H = dims.hidden, I = dims.inter;
  return ws_round_up(kXTerms * pairs * H) + ws_round_up(kXTerms * pairs * (H / 32)) +
         ws_round_up(kHTerms * pairs * I) + ws_round_up(kHTerms * pairs * (I / 32));
}

// Block-scaled path: both launches' arguments (planned) and the workspace
// buffers they use.
struct MxLaunch {
  MxArgs g, d;                   // gate/up + SwiGLU, down
  uint8_t *xq, *xs, *hq, *hs;    // E4M3 terms and E8M0 scales of x and of h
  int64_t pairs;
};

// False when the shape is outside the kernel (nothing may be launched then).
inline bool mx_launch_args(const moe_dims& dims, int T, const moe_mxfp4_proj& gate, const moe_mxfp4_proj& up,
                           const moe_mxfp4_proj& down, const int32_t* offsets, float* y_perm, void* ws,
                           MxLaunch& L) {
  const int H = dims.hidden, I = dims.inter;
  L.pairs = (int64_t)T * dims.top_k;
  L.xq = static_cast<uint8_t*>(ws);
  L.xs = L.xq + ws_round_up((size_t)kXTerms * L.pairs * H);
  L.hq = L.xs + ws_round_up((size_t)kXTerms * L.pairs * (H / 32));
  L.hs = L.hq + ws_round_up((size_t)kHTerms * L.pairs * I);
  MxArgs& g = L.g;
  g = MxArgs{};
  g.w0 = gate.base;
  g.w1 = up.base;
  g.expert_bytes = gate.expert_bytes;
  g.rows = I;
  g.cols = H;
  g.offsets = offsets;
  g.E = dims.n_experts;
  g.pairs = (int)L.pairs;
  g.parts = kXTerms;
  g.b_scale = L.xs;
  const MxLayout lay = mx_layout(T, dims.top_k, dims.n_experts);
  g.n_chunk = lay.chunk;
  g.term_acc = lay.term_acc;
  g.max_bufs = lay.max_bufs;
  g.out = L.hq;
  g.out_scale = L.hs;
  g.out_parts = kHTerms;
  g.limit = dims.swiglu_limit;
  MxArgs& d = L.d;
  d = g;
  d.w0 = down.base;
  d.w1 = nullptr;
  d.expert_bytes = down.expert_bytes;
  d.rows = H;
  d.cols = I;
  d.parts = kHTerms;
  d.b_scale = L.hs;
  d.out = y_perm;
  d.out_scale = nullptr;
  return mx_plan(g, 0) && mx_plan(d, 1) && gate.expert_bytes == up.expert_bytes;
}

// Dequantising path: both launches' arguments (each launch plans its own
// copy) and the f16 buffers of x and h.
struct TcLaunch {
  TcArgs g, d;
  __half *x16, *h16;
  int64_t pairs;
};

inline bool tc_launch_args(const moe_dims& dims, int T, const moe_mxfp4_proj& gate, const moe_mxfp4_proj& up,
                           const moe_mxfp4_proj& down, const int32_t* offsets, float* y_perm, void* ws,
                           TcLaunch& L) {
  const int H = dims.hidden, I = dims.inter;
  if (H % 64 || I % 64) return false;
  L.pairs = (int64_t)T * dims.top_k;
  L.x16 = static_cast<__half*>(ws);
  L.h16 = reinterpret_cast<__half*>(static_cast<uint8_t*>(ws) + ws_round_up((size_t)L.pairs * H * 2));
  TcArgs& g = L.g;
  g = TcArgs{};
  g.w0 = gate.base;
  g.w1 = up.base;
  g.expert_bytes = gate.expert_bytes;
  g.rows = I;
  g.a_cols = H;
  g.k_total = H;
  g.b_cols = H;
  g.offsets = offsets;
  g.E = dims.n_experts;
  g.n_chunk = expert_chunk(T, dims.top_k, dims.n_experts);
  g.out = L.h16;
  g.limit = dims.swiglu_limit;
  TcArgs& d = L.d;
  d = g;
  d.w0 = down.base;
  d.w1 = nullptr;
  d.expert_bytes = down.expert_bytes;
  d.rows = H;
  d.a_cols = I;
  d.k_total = I;
  d.b_cols = I;
  d.out = y_perm;
  TcArgs pg = g, pd = d;  // the shape check; the launches plan their own copies
  return tc_plan(pg, kAMxfp4) && tc_plan(pd, kAMxfp4);
}

}  // namespace moe
