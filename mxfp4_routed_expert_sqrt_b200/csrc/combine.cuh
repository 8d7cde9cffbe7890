// Weighted combine: out[t] = shared[t] + sum_k w[t][k] * y_perm[inv[t*K + k]].
//
// "Model techniques map" (DeepSeek-V4-Flash), row "Shared expert": the routed
// output experts(flat, indices, weights) plus shared_experts(residual).  The
// K slots are summed in the fixed order k = 0..K-1, so the result does not
// depend on how pairs were scheduled.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kCombineThreads = 128;

// grid (ceil(H / (4 * 128)), T); each thread produces 4 consecutive columns.
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(
    const float* __restrict__ y_perm, const int32_t* __restrict__ inv,
    const float* __restrict__ w, const float* __restrict__ shared, float* __restrict__ out,
    __nv_bfloat16* __restrict__ out_bf16, int K, int H) {
  griddep_wait();
  griddep_launch();
  const int t = blockIdx.y;
  const int c4 = blockIdx.x * kCombineThreads + threadIdx.x;
  if (c4 * 4 >= H) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k = 0; k < K; ++k) {
    const int64_t pos = inv[(int64_t)t * K + k];
    const float wk = w[(int64_t)t * K + k];
    if (kDebug && (pos < 0 || pos >= (int64_t)gridDim.y * K)) {  // gridDim.y = T
      set_error(kErrBadIndex);
      continue;
    }
    const float4 y = __ldg(reinterpret_cast<const float4*>(y_perm + pos * H) + c4);
    acc.x = fmaf(wk, y.x, acc.x);
    acc.y = fmaf(wk, y.y, acc.y);
    acc.z = fmaf(wk, y.z, acc.z);
    acc.w = fmaf(wk, y.w, acc.w);
  }
  if (shared != nullptr) {
    const float4 s = __ldg(reinterpret_cast<const float4*>(shared + (int64_t)t * H) + c4);
    acc.x = s.x + acc.x;
    acc.y = s.y + acc.y;
    acc.z = s.z + acc.z;
    acc.w = s.w + acc.w;
  }
  reinterpret_cast<float4*>(out + (int64_t)t * H)[c4] = acc;
  if (out_bf16 != nullptr) {
    __nv_bfloat162 a = __floats2bfloat162_rn(acc.x, acc.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 v;
    v.x = *reinterpret_cast<uint32_t*>(&a);
    v.y = *reinterpret_cast<uint32_t*>(&b);
    reinterpret_cast<uint2*>(out_bf16 + (int64_t)t * H)[c4] = v;
  }
}

}  // namespace moe
