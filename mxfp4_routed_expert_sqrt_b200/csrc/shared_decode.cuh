// The bf16 shared expert in the decode regime (few tokens): HBM bound on its
// 48 MiB of weights ("Model techniques map", row "Shared expert": every token's
// routed output plus the shared expert of the same input; same clamped SwiGLU).
//
// One CTA per fragment row block (MODE 0: 8 gate rows + the same 8 up rows;
// MODE 1: 16 down rows); its 8 warps split K.  Lanes load their m16n8k16
// fragments of weights and activations straight from global memory (16 bytes
// per lane per 32-column group, coalesced per row), bf16 x bf16 products are
// exact and accumulate in fp32 inside the MMA.  The k-to-lane assignment:
// lane (g, t) owns columns 32G + 8t + [0, 8) of every 32-column group.
//
// MODE 0 writes h as a bf16 pair, hi = bf16(h) at [t][row] and lo = bf16(h -
// hi) at [t][I + row]; MODE 1 runs over K = 2I with the down weights repeated
// (column k -> k mod I), so h enters with 16 significant bits.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kShThreads = 256;
constexpr int kShWarps = kShThreads / 32;
constexpr int kShMaxNt = 8;  // token tiles of 8 (T <= 64)
constexpr int kShBatch = 8;  // column groups whose weights are loaded together

struct ShArgs {
  const __nv_bfloat16* w0;  // MODE 0: gate [I][H]; MODE 1: down [H][I]
  const __nv_bfloat16* w1;  // MODE 0: up [I][H]
  int rows;                 // I (MODE 0) or H (MODE 1)
  int a_cols;               // H (MODE 0) or I (MODE 1)
  int k_total;              // H (MODE 0) or 2I (MODE 1)
  const __nv_bfloat16* xin; // MODE 0: x [T][H]; MODE 1: h pair [T][2I]
  int T;
  void* out;                // MODE 0: h pair bf16 [T][2I]; MODE 1: fp32 [T][H]
  float limit;
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int MODE>
__global__ void __launch_bounds__(kShThreads) shared_decode_kernel(const ShArgs args) {
  __shared__ float s_red[kShWarps][32][4];
  griddep_wait();
  griddep_launch();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int I_or_H = args.rows;
  // fragment rows g and g + 8 of this block
  const __nv_bfloat16 *rg, *rg8;
  int r0;
  if (MODE == 0) {
    r0 = blockIdx.x * 8;
    rg = args.w0 + (int64_t)(r0 + g) * args.a_cols;
    rg8 = args.w1 + (int64_t)(r0 + g) * args.a_cols;
  } else {
    r0 = blockIdx.x * 16;
    rg = args.w0 + (int64_t)(r0 + g) * args.a_cols;
    rg8 = args.w0 + (int64_t)(r0 + g + 8) * args.a_cols;
  }
  const int kw = args.k_total / kShWarps;  // columns per warp, multiple of 32
  const int G0 = warp * (kw / 32), NG = kw / 32;
  const int a_groups = args.a_cols / 32;
  const int ntiles = (args.T + 7) / 8;

  const __nv_bfloat16* xr[kShMaxNt];
#pragma unroll
  for (int nt = 0; nt < kShMaxNt; ++nt) xr[nt] = args.xin + (int64_t)min(nt * 8 + g, args.T - 1) * args.k_total;
  float acc[kShMaxNt][4];
#pragma unroll
  for (int nt = 0; nt < kShMaxNt; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;

  // The weight fragments of kShBatch column groups are loaded before any of
  // their MMAs, so each warp keeps 2 * kShBatch 16-byte HBM loads in flight.
  for (int gi0 = 0; gi0 < NG; gi0 += kShBatch) {
    uint4 a[kShBatch], b[kShBatch];
#pragma unroll
    for (int u = 0; u < kShBatch; ++u) {
      const int GA = (G0 + min(gi0 + u, NG - 1)) % a_groups;
      a[u] = __ldg(reinterpret_cast<const uint4*>(rg + GA * 32 + 8 * t));
      b[u] = __ldg(reinterpret_cast<const uint4*>(rg8 + GA * 32 + 8 * t));
    }
#pragma unroll
    for (int u = 0; u < kShBatch; ++u) {
      if (gi0 + u < NG) {
        const int G = G0 + gi0 + u;
#pragma unroll
        for (int nt = 0; nt < kShMaxNt; ++nt) {
          if (nt < ntiles) {
            const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xr[nt] + G * 32 + 8 * t));
            mma_bf16_16816(acc[nt], a[u].x, b[u].x, a[u].y, b[u].y, xv.x, xv.y);
            mma_bf16_16816(acc[nt], a[u].z, b[u].z, a[u].w, b[u].w, xv.z, xv.w);
          }
        }
      }
    }
  }

  for (int nt = 0; nt < ntiles; ++nt) {
    float a4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a4[i] = acc[0][i];
#pragma unroll
    for (int m = 1; m < kShMaxNt; ++m)
      if (m == nt) {
#pragma unroll
        for (int i = 0; i < 4; ++i) a4[i] = acc[m][i];
      }
#pragma unroll
    for (int i = 0; i < 4; ++i) s_red[warp][lane][i] = a4[i];
    __syncthreads();
    if (MODE == 0) {
      if (tid < 64) {  // (fragment lane l, column half c): gate in [c], up in [2 + c]
        const int l = tid & 31, c = tid >> 5;
        float gs = 0.f, us = 0.f;
        for (int w = 0; w < kShWarps; ++w) { gs += s_red[w][l][c]; us += s_red[w][l][2 + c]; }
        const int tok = nt * 8 + 2 * (l & 3) + c;
        if (tok < args.T) {
          const int row = r0 + (l >> 2);
          const float hv = silu_clamped_swiglu(gs, us, args.limit);
          const __nv_bfloat16 hi = __float2bfloat16_rn(hv);
          __nv_bfloat16* o = static_cast<__nv_bfloat16*>(args.out) + (int64_t)tok * 2 * I_or_H;
          o[row] = hi;
          o[I_or_H + row] = __float2bfloat16_rn(hv - __bfloat162float(hi));
        }
      }
    } else {
      if (tid < 128) {  // (fragment lane l, value v): row g + 8 (v >> 1), token 2t + (v & 1)
        const int l = tid & 31, v = tid >> 5;
        float sum = 0.f;
        for (int w = 0; w < kShWarps; ++w) sum += s_red[w][l][v];
        const int tok = nt * 8 + 2 * (l & 3) + (v & 1);
        if (tok < args.T) {
          const int row = r0 + (l >> 2) + 8 * (v >> 1);
          static_cast<float*>(args.out)[(int64_t)tok * I_or_H + row] = sum;
        }
      }
    }
    __syncthreads();
  }
}

}  // namespace moe
