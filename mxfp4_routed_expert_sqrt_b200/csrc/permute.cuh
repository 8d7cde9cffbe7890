// Grouping of (token, slot) pairs by expert: a stable counting sort in one CTA.
//
// The routed experts are applied as experts(flat, indices, weights) ("Model
// techniques map", row "Shared expert"); grouping the pairs per expert makes
// each expert's token list contiguous so its weights are streamed once.
//
// Stability without a serial pass: the pairs are cut into 32 contiguous
// chunks, one per warp.  Each warp counts its chunk per expert; a scan over
// (expert, warp) in expert-major order gives every warp the first output slot
// of each expert; each warp then walks its chunk in order, 32 pairs at a time,
// ranking equal experts inside a round with __match_any_sync.  The result is
// the unique (expert, pair id) order.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kPermuteThreads = 1024;

__global__ void __launch_bounds__(kPermuteThreads) permute_kernel(
    const int32_t* __restrict__ idx, int n, int E, int32_t* __restrict__ offsets,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  extern __shared__ int32_t hist[];  // [32 warps][E]
  __shared__ int32_t scan_buf[kPermuteThreads];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  griddep_wait();
  griddep_launch();
  for (int i = tid; i < 32 * E; i += kPermuteThreads) hist[i] = 0;
  __syncthreads();

  const int chunk = (n + 31) / 32;
  const int start = min(n, warp * chunk), end = min(n, start + chunk);
  for (int p = start + lane; p < end; p += 32) {
    int e = idx[p];
    if (e < 0 || e >= E) { set_error(kErrBadExpert); e = 0; }
    atomicAdd(&hist[warp * E + e], 1);
  }
  __syncthreads();

  // per expert: prefix over warps (in place) and the expert's total
  int total = 0;
  const int e = tid;  // E <= kPermuteThreads
  if (e < E) {
    for (int w = 0; w < 32; ++w) {
      const int c = hist[w * E + e];
      hist[w * E + e] = total;
      total += c;
    }
  }
  // exclusive scan of the totals over experts (block-wide, Hillis-Steele)
  scan_buf[tid] = (e < E) ? total : 0;
  __syncthreads();
  for (int o = 1; o < kPermuteThreads; o <<= 1) {
    const int v = (tid >= o) ? scan_buf[tid - o] : 0;
    __syncthreads();
    scan_buf[tid] += v;
    __syncthreads();
  }
  const int excl = scan_buf[tid] - ((e < E) ? total : 0);
  if (e < E) {
    offsets[e] = excl;
    for (int w = 0; w < 32; ++w) hist[w * E + e] += excl;
  }
  if (tid == 0) offsets[E] = n;
  __syncthreads();

  // in-order placement, 32 pairs per round
  const unsigned lt = (1u << lane) - 1u;
  for (int p0 = start; p0 < end; p0 += 32) {
    const int p = p0 + lane;
    const bool valid = p < end;
    const unsigned act = __ballot_sync(0xffffffffu, valid);
    int ex = 0, rank = 0;
    unsigned m = 0;
    if (valid) {
      ex = idx[p];
      if (ex < 0 || ex >= E) ex = 0;
      m = __match_any_sync(act, ex);
      rank = __popc(m & lt);
      const int pos = hist[warp * E + ex] + rank;
      perm[pos] = p;
      inv[p] = pos;
    }
    __syncwarp();
    if (valid && rank == 0) hist[warp * E + ex] += __popc(m);
    __syncwarp();
  }
}

}  // namespace moe
