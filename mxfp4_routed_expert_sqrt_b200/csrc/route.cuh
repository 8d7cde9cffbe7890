// Routing: router logits (fp32), sqrt-softplus scores, biased top-k, normalised
// weights, and token-id hash routing.
//
// "DeepSeek-V4-Flash export design" (ONNX Runtime mobius), Source
// configuration, MoE bullet: normalized sqrt(softplus(logit)) routing, top 6 of
// 256, scale 1.5; the first three layers take their experts from a token-id
// hash table.  "Model techniques map", rows "Mixture of experts" and
// "Auxiliary-loss-free load balancing": the bias enters the top-k only and the
// weights are gathered from the unbiased scores.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kLogitTok = 8;  // tokens per CTA in the SIMT logits kernel

// logits[t][e] = sum_h x[t][h] * Wr[e][h], fp32 products and sums.
// One warp per expert; lanes stride the hidden dim in float4 chunks; a CTA
// covers 4 experts x kLogitTok tokens, so Wr is read once per token block.
__global__ void __launch_bounds__(128) route_logits_kernel(const __nv_bfloat16* __restrict__ x,
                                                           int T, int H,
                                                           const float* __restrict__ wr, int E,
                                                           float* __restrict__ logits) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 4 + warp;
  const int t0 = blockIdx.y * kLogitTok;
  if (e >= E) return;
  const float4* w4 = reinterpret_cast<const float4*>(wr + (int64_t)e * H);
  float acc[kLogitTok];
#pragma unroll
  for (int i = 0; i < kLogitTok; ++i) acc[i] = 0.f;
  const int nt = min(kLogitTok, T - t0);
  for (int j = lane; j < H / 4; j += 32) {
    const float4 w = __ldg(w4 + j);
#pragma unroll
    for (int i = 0; i < kLogitTok; ++i) {
      if (i < nt) {
        const uint2 xv = __ldg(reinterpret_cast<const uint2*>(x + (int64_t)(t0 + i) * H) + j);
        acc[i] = fmaf(__uint_as_float(xv.x << 16), w.x, acc[i]);
        acc[i] = fmaf(__uint_as_float(xv.x & 0xFFFF0000u), w.y, acc[i]);
        acc[i] = fmaf(__uint_as_float(xv.y << 16), w.z, acc[i]);
        acc[i] = fmaf(__uint_as_float(xv.y & 0xFFFF0000u), w.w, acc[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kLogitTok; ++i) {
    float v = acc[i];
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0 && i < nt) logits[(int64_t)(t0 + i) * E + e] = v;
  }
}

__device__ __forceinline__ float sqrt_softplus(float z) {
  return sqrtf(log1pf(expf(-fabsf(z))) + fmaxf(z, 0.f));
}

// One warp per token: scores, top-k (learned) or table lookup (hash), weights.
// Shared memory: 4 warps x E scores.
__global__ void __launch_bounds__(128) route_select_kernel(
    const float* __restrict__ logits, int T, int E, int K, float scale,
    const float* __restrict__ bias, const int32_t* __restrict__ tok,
    const int32_t* __restrict__ table, int vocab, int32_t* __restrict__ topk_idx,
    float* __restrict__ topk_w) {
  extern __shared__ float s_sm[];  // [4][E]
  __shared__ int32_t sel[4][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 4 + warp;
  if (t >= T) return;
  float* s = s_sm + warp * E;
  for (int j = lane; j < E; j += 32) s[j] = sqrt_softplus(logits[(int64_t)t * E + j]);
  __syncwarp();
  if (table != nullptr) {
    int v = tok[t];
    if (v < 0 || v >= vocab) v = 0;
    if (lane < K) sel[warp][lane] = table[(int64_t)v * K + lane];
  } else {
    // candidates of this lane: j = lane + 32 m; taken bits per m
    uint32_t taken = 0;
    const int nm = (E + 31) / 32;
    for (int k = 0; k < K; ++k) {
      float bv = -INFINITY;
      int bid = 0x7fffffff;
      for (int m = 0; m < nm; ++m) {
        const int j = lane + 32 * m;
        if (j < E && !((taken >> m) & 1u)) {
          const float v = s[j] + (bias ? bias[j] : 0.f);
          if (v > bv || (v == bv && j < bid)) { bv = v; bid = j; }
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oid = __shfl_xor_sync(0xffffffffu, bid, o);
        if (ov > bv || (ov == bv && oid < bid)) { bv = ov; bid = oid; }
      }
      if (bid < E && (bid & 31) == lane) taken |= 1u << (bid >> 5);
      if (lane == 0) sel[warp][k] = bid < E ? bid : 0;
    }
  }
  __syncwarp();
  float sv = 0.f;
  int id = 0;
  if (lane < K) {
    id = sel[warp][lane];
    id = min(max(id, 0), E - 1);
    sv = s[id];
  }
  float sum = sv;
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < K) {
    topk_idx[(int64_t)t * K + lane] = id;
    topk_w[(int64_t)t * K + lane] = scale * sv / sum;
  }
}

}  // namespace moe
