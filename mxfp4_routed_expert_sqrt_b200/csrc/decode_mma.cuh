// Decode-regime routed experts: weight streaming with register decode and
// warp-level MMA fragments.
//
// Decode is bound by expert-weight bandwidth ("EasyDeL / DeepSeek-V4-Flash",
// Loading).  At the HBM rate a B200 SM has about 2-3 lane instructions per
// weight, so the per-weight work must stay near one instruction whatever the
// tokens-per-expert count.  Each warp therefore feeds 16 x 16 fragments of
// decoded weights (E2M1 -> f16 by cvt, exact) and 16 x 8 activation fragments
// (f16) to mma.sync m16n8k16 with fp32 accumulation: every product is exact
// and sums are fp32.  The E8M0 scale of each 32-column group is applied in
// fp32 to the group's partial sum (so any exponent 0..254 is exact); the
// k-to-lane assignment below keeps every MMA k-step inside one group.
//
// Units and streaming.  MODE 0 (gate/up): a unit is (active expert, 8 rows);
// fragment rows 0-7 are gate rows r0..r0+7 and rows 8-15 the up rows r0..r0+7,
// so each lane ends with gate and up sums of the same (row, token) and applies
// the clamped SwiGLU ("Model techniques map", row "SwiGLU feed-forward") in
// registers; h is written in f16.  MODE 1 (down): a unit is (active expert,
// 32 rows = 2 fragment row blocks) over K = inter, fp32 output.  Each unit's
// rows are brought into a shared-memory ring by 1-D bulk copies (TMA engine),
// one per row into a padded row stride so the fragment reads are bank-conflict
// free.  The 8 warps of a CTA split K; partial sums meet in shared memory.
//
// Fragment mapping (m16n8k16, row.col): lane = 4 g + t.  For group G (32
// columns, 16 code bytes per row), lane t owns code bytes [4t, 4t+4) of rows g
// and g+8, i.e. columns 32G + 8t + [0, 8).  MMA step s in {0, 1} of the group
// takes byte 2s as a0/a1 (columns +4s+{0,1}) and byte 2s+1 as a2/a3 (columns
// +4s+{2,3}); the activation fragment of lane (g, t) is then the 8 f16 at
// columns 32G + 8t + [0, 8) of token g: one 16-byte load.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecStages = 3;
constexpr int kDecMaxNt = 8;  // token tiles of 8 kept in registers per pass

struct DecArgs {
  const uint8_t* w0;      // MODE 0: gate blobs; MODE 1: down blobs
  const uint8_t* w1;      // MODE 0: up blobs
  int64_t expert_bytes;
  int rows, cols;         // of one projection
  const __half* xin;      // MODE 0: x in f16 [T][cols]; MODE 1: h in f16 [pos][cols]
  const int32_t* offsets; // [E+1]
  const int32_t* perm;    // MODE 0: token of pos = perm[pos] / K
  int K, E;
  void* out;              // MODE 0: h f16 [pos][rows]; MODE 1: y fp32 [pos][rows]
  float limit;
};

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %11, %12, %13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f), "f"(0.f), "f"(0.f), "f"(0.f));
}

// Two E8M0 bytes (low 16 bits of e2) -> fp32 scales 2^(e-127), exact for every e.
__device__ __forceinline__ void e8m0x2_to_f32(uint32_t e2, float& s_lo, float& s_hi) {
  uint32_t b;
  const uint16_t v = (uint16_t)e2;
  asm("cvt.rn.bf16x2.ue8m0x2 %0, %1;" : "=r"(b) : "h"(v));
  s_lo = __uint_as_float(b << 16);
  s_hi = __uint_as_float(b & 0xFFFF0000u);
}

// Rows per unit (per projection) and the layout of one stage.
template <int MODE>
struct DecLayout {
  static constexpr int kRowBlocks = MODE == 0 ? 1 : 2;  // 16-row fragment blocks per unit
  static constexpr int kRows = 16 * kRowBlocks;         // fragment rows per unit
  static constexpr int kKSplit = kDecWarps / kRowBlocks;
};

template <int MODE>
__global__ void __launch_bounds__(kDecThreads, 2) decode_mma_kernel(const DecArgs args) {
  using L = DecLayout<MODE>;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[kDecStages];
  __shared__ int16_t s_active[1024];
  __shared__ int32_t s_cnt[kDecThreads];
  __shared__ float s_red[kDecWarps][32][4];
  __shared__ int32_t s_nact;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int cols = args.cols, rows = args.rows;
  const int nib_row = cols / 2, sc_row = cols / 32;
  const int nib_stride = nib_row + 16;  // padded: consecutive rows shift by 4 banks
  // stage: [kRows][nib_stride] codes, then [kRows][sc_row] scales
  const int stage_bytes = ((L::kRows * nib_stride + L::kRows * sc_row) + 127) / 128 * 128;
  const int unit_rows = MODE == 0 ? 8 : L::kRows;  // rows of each projection per unit

  // ---- active experts ---------------------------------------------------------
  const int E = args.E;
  {
    const int per = (E + kDecThreads - 1) / kDecThreads;
    int c = 0;
    for (int e = tid * per; e < min(E, tid * per + per); ++e) c += args.offsets[e + 1] > args.offsets[e];
    s_cnt[tid] = c;
    __syncthreads();
    if (tid == 0) {
      int run = 0;
      for (int i = 0; i < kDecThreads; ++i) { const int v = s_cnt[i]; s_cnt[i] = run; run += v; }
      s_nact = run;
    }
    __syncthreads();
    int w = s_cnt[tid];
    for (int e = tid * per; e < min(E, tid * per + per); ++e)
      if (args.offsets[e + 1] > args.offsets[e]) s_active[w++] = (int16_t)e;
    __syncthreads();
  }
  const int n_active = s_nact;
  const int units_per_expert = rows / unit_rows;
  const int n_units = n_active * units_per_expert;
  const int u_begin = (int)((int64_t)n_units * blockIdx.x / gridDim.x);
  const int u_end = (int)((int64_t)n_units * (blockIdx.x + 1) / gridDim.x);
  if (u_begin >= u_end) return;

  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) mbar_init(&full_bar[s], 1);
    fence_mbar_init();
  }
  __syncthreads();

  const uint64_t pol = policy_evict_first();
  // one thread issues a unit's copies: per fragment row its codes (padded
  // destination) and per projection its block of scale rows
  auto issue = [&](int u, int s) {
    const int e = s_active[u / units_per_expert];
    const int r0 = (u % units_per_expert) * unit_rows;
    uint8_t* dst = smem + (int64_t)s * stage_bytes;
    mbar_arrive_expect_tx(&full_bar[s], (uint32_t)(L::kRows * (nib_row + sc_row)));
    for (int fr = 0; fr < L::kRows; ++fr) {
      const uint8_t* blob;
      int R;
      if (MODE == 0) { blob = (fr < 8 ? args.w0 : args.w1) + (int64_t)e * args.expert_bytes; R = r0 + (fr & 7); }
      else { blob = args.w0 + (int64_t)e * args.expert_bytes; R = r0 + fr; }
      bulk_g2s_stream(dst + fr * nib_stride, blob + (int64_t)R * nib_row, (uint32_t)nib_row, &full_bar[s], pol);
    }
    uint8_t* sdst = dst + L::kRows * nib_stride;
    if (MODE == 0) {
      for (int p = 0; p < 2; ++p) {
        const uint8_t* blob = (p == 0 ? args.w0 : args.w1) + (int64_t)e * args.expert_bytes;
        bulk_g2s_stream(sdst + p * 8 * sc_row, blob + (int64_t)rows * nib_row + (int64_t)r0 * sc_row,
                        (uint32_t)(8 * sc_row), &full_bar[s], pol);
      }
    } else {
      const uint8_t* blob = args.w0 + (int64_t)e * args.expert_bytes;
      bulk_g2s_stream(sdst, blob + (int64_t)rows * nib_row + (int64_t)r0 * sc_row, (uint32_t)(L::kRows * sc_row),
                      &full_bar[s], pol);
    }
  };
  if (tid == 0)
    for (int k = 0; k < kDecStages && u_begin + k < u_end; ++k) issue(u_begin + k, k);

  // this warp: fragment row block and K range.  The K split is capped so a
  // warp always owns an even number of groups (narrow shapes idle some warps).
  const int rblk = warp / L::kKSplit, ks = warp % L::kKSplit;
  const int ksplit = min(L::kKSplit, cols / 64);
  const int kw = cols / ksplit;                // columns per warp (multiple of 64)
  const int g0 = ks * (kw / 32);               // first group
  const int ng = ks < ksplit ? kw / 32 : 0;    // groups per warp

  for (int u = u_begin; u < u_end; ++u) {
    const int k = u - u_begin, s = k % kDecStages;
    const int e = s_active[u / units_per_expert];
    const int r0 = (u % units_per_expert) * unit_rows;
    const int pos0 = args.offsets[e], n_tok = args.offsets[e + 1] - pos0;
    if (!__syncthreads_and(mbar_wait(&full_bar[s], (k / kDecStages) & 1))) {
      if (tid == 0) {
        set_error(kErrWaitDecode);
        for (int k2 = k + 1; k2 < min(u_end - u_begin, k + kDecStages); ++k2)
          mbar_wait(&full_bar[k2 % kDecStages], (k2 / kDecStages) & 1);
      }
      return;
    }
    const uint8_t* st = smem + (int64_t)s * stage_bytes;
    const uint8_t* rowg = st + (rblk * 16 + g) * nib_stride;
    const uint8_t* rowg8 = rowg + 8 * nib_stride;
    const uint8_t* scb = st + L::kRows * nib_stride;
    const uint8_t* scg = scb + (rblk * 16 + g) * sc_row;
    const uint8_t* scg8 = scg + 8 * sc_row;

    for (int j0 = 0; j0 < n_tok; j0 += 8 * kDecMaxNt) {
      const int ntiles = min(kDecMaxNt, (n_tok - j0 + 7) / 8);
      // activation rows of this lane's token (column g of each token tile)
      const __half* xr[kDecMaxNt];
#pragma unroll
      for (int nt = 0; nt < kDecMaxNt; ++nt) {
        const int j = min(j0 + nt * 8 + g, n_tok - 1);  // tail lanes repeat a valid token
        const int pos = pos0 + j;
        const int row = MODE == 0 ? args.perm[pos] / args.K : pos;
        xr[nt] = args.xin + (int64_t)row * cols;
      }
      float acc[kDecMaxNt][4];
#pragma unroll
      for (int nt = 0; nt < kDecMaxNt; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;

      for (int gi = 0; gi < ng; gi += 2) {
        const int G = g0 + gi;
        // codes: 4 bytes of rows g and g+8 for groups G and G+1; scales of both
        const uint32_t wg0 = *reinterpret_cast<const uint32_t*>(rowg + G * 16 + 4 * t);
        const uint32_t wg1 = *reinterpret_cast<const uint32_t*>(rowg + (G + 1) * 16 + 4 * t);
        const uint32_t w80 = *reinterpret_cast<const uint32_t*>(rowg8 + G * 16 + 4 * t);
        const uint32_t w81 = *reinterpret_cast<const uint32_t*>(rowg8 + (G + 1) * 16 + 4 * t);
        float sg0, sg1, s80, s81;
        e8m0x2_to_f32(*reinterpret_cast<const uint16_t*>(scg + G), sg0, sg1);
        e8m0x2_to_f32(*reinterpret_cast<const uint16_t*>(scg8 + G), s80, s81);
        uint32_t ga[4], gb[4], ha[4], hb[4];
        e2m1x8_to_f16x2(wg0, ga);
        e2m1x8_to_f16x2(w80, gb);
        e2m1x8_to_f16x2(wg1, ha);
        e2m1x8_to_f16x2(w81, hb);
        const uint32_t A00[4] = {ga[0], gb[0], ga[1], gb[1]}, A01[4] = {ga[2], gb[2], ga[3], gb[3]};
        const uint32_t A10[4] = {ha[0], hb[0], ha[1], hb[1]}, A11[4] = {ha[2], hb[2], ha[3], hb[3]};
#pragma unroll
        for (int nt = 0; nt < kDecMaxNt; ++nt) {
          if (nt < ntiles) {
            const uint4 x0 = __ldg(reinterpret_cast<const uint4*>(xr[nt] + G * 32 + 8 * t));
            const uint4 x1 = __ldg(reinterpret_cast<const uint4*>(xr[nt] + (G + 1) * 32 + 8 * t));
            float c0[4], c1[4], d0[4], d1[4];
            mma_f16_16816(c0, A00, x0.x, x0.y);
            mma_f16_16816(c1, A01, x0.z, x0.w);
            mma_f16_16816(d0, A10, x1.x, x1.y);
            mma_f16_16816(d1, A11, x1.z, x1.w);
            acc[nt][0] = fmaf(sg0, c0[0] + c1[0], fmaf(sg1, d0[0] + d1[0], acc[nt][0]));
            acc[nt][1] = fmaf(sg0, c0[1] + c1[1], fmaf(sg1, d0[1] + d1[1], acc[nt][1]));
            acc[nt][2] = fmaf(s80, c0[2] + c1[2], fmaf(s81, d0[2] + d1[2], acc[nt][2]));
            acc[nt][3] = fmaf(s80, c0[3] + c1[3], fmaf(s81, d0[3] + d1[3], acc[nt][3]));
          }
        }
      }

      // ---- K-split reduction and epilogue, one token tile at a time ---------------
      for (int nt = 0; nt < ntiles; ++nt) {
        float a4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a4[i] = acc[0][i];
#pragma unroll
        for (int m = 1; m < kDecMaxNt; ++m)
          if (m == nt) {
#pragma unroll
            for (int i = 0; i < 4; ++i) a4[i] = acc[m][i];
          }
        s_red[warp][lane][0] = a4[0];
        s_red[warp][lane][1] = a4[1];
        s_red[warp][lane][2] = a4[2];
        s_red[warp][lane][3] = a4[3];
        __syncthreads();
        if (MODE == 0) {
          // 64 outputs: (fragment lane l, column half c): gate in [c], up in [2 + c]
          if (tid < 64) {
            const int l = tid & 31, c = tid >> 5;
            float gs = 0.f, us = 0.f;
            for (int w = 0; w < ksplit; ++w) { gs += s_red[w][l][c]; us += s_red[w][l][2 + c]; }
            const int j = j0 + nt * 8 + 2 * (l & 3) + c;
            if (j < n_tok) {
              const int row = r0 + (l >> 2);
              static_cast<__half*>(args.out)[(int64_t)(pos0 + j) * rows + row] =
                  __float2half_rn(silu_clamped_swiglu(gs, us, args.limit));
            }
          }
        } else {
          // kRowBlocks x 128 outputs: (row block, fragment lane l, value v)
          for (int o = tid; o < L::kRowBlocks * 128; o += kDecThreads) {
            const int rb2 = o >> 7, l = o & 31, v = (o >> 5) & 3;
            float sum = 0.f;
            for (int w = 0; w < ksplit; ++w) sum += s_red[rb2 * L::kKSplit + w][l][v];
            const int j = j0 + nt * 8 + 2 * (l & 3) + (v & 1);
            if (j < n_tok) {
              const int row = r0 + rb2 * 16 + (l >> 2) + 8 * (v >> 1);
              static_cast<float*>(args.out)[(int64_t)(pos0 + j) * rows + row] = sum;
            }
          }
        }
        __syncthreads();
      }
    }
    // every thread is past its reads of stage s (the last __syncthreads above)
    if (tid == 0 && u + kDecStages < u_end) issue(u + kDecStages, s);
  }
}

// x (bf16) -> f16, n elements (multiple of 8), 16-byte aligned.
__global__ void bf16_to_f16_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, int64_t n8) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = in[i];
    out[i] = make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z), bf16x2_to_f16x2(v.w));
  }
}

}  // namespace moe
