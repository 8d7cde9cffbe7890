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

constexpr int kLogitExperts = 2;     // expert rows per CTA, staged in shared memory
constexpr int kLogitThreads = 256;
constexpr int kLogitTokBlock = 64;   // tokens per CTA (grid.y covers the rest)
constexpr int kLogitTokStep = 4;     // tokens a warp works on at once

// logits[t][e] = sum_h x[t][h] * Wr[e][h], fp32 products and sums.
// A CTA stages kLogitExperts router rows (fp32) in shared memory with every
// thread loading in parallel, then its 8 warps stream the x rows (bf16, from
// L2) of up to kLogitTokBlock tokens, kLogitTokStep tokens per warp at a
// time, lanes striding the hidden dim in groups of 8 columns.  E/2 CTAs keep
// every SM busy at any token count, and the router (4 MiB at V4-Flash shape)
// is read from HBM once per token block.  Shared memory: kLogitExperts * H
// floats.
__global__ void __launch_bounds__(kLogitThreads) route_logits_kernel(const __nv_bfloat16* __restrict__ x,
                                                                     int T, int H,
                                                                     const float* __restrict__ wr, int E,
                                                                     float* __restrict__ logits) {
  extern __shared__ float4 s_w4[];  // [kLogitExperts][H / 4]
  griddep_wait();
  griddep_launch();
  const int e0 = blockIdx.x * kLogitExperts;
  const int ne = min(kLogitExperts, E - e0);
  const int h4 = H / 4, h8 = H / 8;
  const float4* src = reinterpret_cast<const float4*>(wr + (int64_t)e0 * H);
  for (int i = threadIdx.x; i < ne * h4; i += kLogitThreads) s_w4[i] = __ldg(src + i);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t_end = min(T, (blockIdx.y + 1) * kLogitTokBlock);
  for (int t0 = blockIdx.y * kLogitTokBlock + warp * kLogitTokStep; t0 < t_end;
       t0 += (kLogitThreads / 32) * kLogitTokStep) {
    float acc[kLogitTokStep][kLogitExperts];
#pragma unroll
    for (int i = 0; i < kLogitTokStep; ++i)
#pragma unroll
      for (int e = 0; e < kLogitExperts; ++e) acc[i][e] = 0.f;
#pragma unroll 4
    for (int j = lane; j < h8; j += 32) {
      uint4 xv[kLogitTokStep];
#pragma unroll
      for (int i = 0; i < kLogitTokStep; ++i)
        xv[i] = t0 + i < t_end ? __ldg(reinterpret_cast<const uint4*>(x + (int64_t)(t0 + i) * H) + j)
                               : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int e = 0; e < kLogitExperts; ++e) {
        if (e < ne) {
          const float4 wa = s_w4[e * h4 + 2 * j], wb = s_w4[e * h4 + 2 * j + 1];
#pragma unroll
          for (int i = 0; i < kLogitTokStep; ++i) {
            float a = acc[i][e];
            a = fmaf(__uint_as_float(xv[i].x << 16), wa.x, a);
            a = fmaf(__uint_as_float(xv[i].x & 0xFFFF0000u), wa.y, a);
            a = fmaf(__uint_as_float(xv[i].y << 16), wa.z, a);
            a = fmaf(__uint_as_float(xv[i].y & 0xFFFF0000u), wa.w, a);
            a = fmaf(__uint_as_float(xv[i].z << 16), wb.x, a);
            a = fmaf(__uint_as_float(xv[i].z & 0xFFFF0000u), wb.y, a);
            a = fmaf(__uint_as_float(xv[i].w << 16), wb.z, a);
            a = fmaf(__uint_as_float(xv[i].w & 0xFFFF0000u), wb.w, a);
            acc[i][e] = a;
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kLogitTokStep; ++i)
#pragma unroll
      for (int e = 0; e < kLogitExperts; ++e) {
        float v = acc[i][e];
#pragma unroll
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && e < ne && t0 + i < t_end) logits[(int64_t)(t0 + i) * E + e0 + e] = v;
      }
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
  griddep_wait();
  griddep_launch();
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
