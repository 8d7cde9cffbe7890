// Decode-regime expert GEMV on CUDA cores: streams the weights of the active
// experts once through shared memory with 1-D bulk copies (TMA engine) and
// decodes them in registers.
//
// Decode is bound by expert-weight bandwidth ("EasyDeL / DeepSeek-V4-Flash",
// Loading: decode is bound by expert weight bandwidth); the weights are MXFP4
// ("ElytronAI / DeepSeek-v4-Flash", Sizes: E2M1 nibble plane + E8M0 group-32
// plane), expert xid at base + xid * expert_bytes (same page, Layout).
//
// Work decomposition.  A unit is (active expert, block of RB weight rows).
// Each CTA (128 threads) owns a contiguous range of units; a 1-D bulk copy per
// plane brings the unit's rows (codes and scales of gate+up, or of down) into
// a stage of a kStages-deep ring in shared memory, so up to kStages units of
// weights are in flight per SM.  Thread i owns input columns [32 g, 32 g + 32)
// with g = i % gpr (gpr = cols / 32), i.e. exactly one E8M0 group and one
// 16-byte chunk of codes per weight row, and rows q, q + rp, ... of the unit
// (q = i / gpr, rp = 128 / gpr).  The unit's token activations for its columns
// sit in registers, so each weight is decoded once per token pass and reused
// for kNtp tokens.  Per group and token, 16 packed-f16 FMAs in 4 chains of 4
// products are moved to fp32 with mixed-precision adds, then scaled by the
// group's 2^(e-127) and summed in fp32; E2M1 values and the f16 activations
// are exact, so only 3 f16 roundings per 4 products enter.  Partial sums are
// reduced across the gpr threads of a row with shuffles and shared memory.
#pragma once

#include "common.cuh"

namespace moe {

enum { kWMxfp4 = 0, kWBf16 = 1 };

constexpr int kGemvThreads = 512;
constexpr int kGemvStages = 4;
constexpr int kGemvStageTarget = 36 * 1024;  // bytes of weights per stage (approx.)
constexpr int kGemvRedFloats = 2048;         // cross-segment reduction buffer
constexpr int kGemvSmemBudget = 200 * 1024;  // dynamic shared memory for the stage ring

struct GemvProj {
  const uint8_t* base;   // expert 0
  int64_t expert_bytes;  // stride between experts
  int rows, cols;
};

struct GemvArgs {
  GemvProj a, b;           // a: gate (or down, or the only projection); b: up (SwiGLU)
  float limit;             // SwiGLU clamp
  const void* xin;         // activations: bf16 [*][cols] or fp32 [*][cols]
  int xin_f32;             // 1: fp32 rows (h), 0: bf16 rows (x)
  const int32_t* offsets;  // [E+1] grouped pair ranges; null: one expert covering n_single rows
  const int32_t* perm;     // pair ids; input row = perm[pos] / K. null: input row = pos
  int K;
  int E;
  int n_single;
  int rb;                  // rows per unit (multiple of rp, divides rows)
  int n_stages;            // depth of the shared-memory ring, 1..kGemvStages
  float* out;              // fp32 [pos][out_ld], column = weight row
  int out_ld;
};

template <int WF>
struct WTraits;
template <>
struct WTraits<kWMxfp4> {
  static constexpr int kRowBytesNum = 17, kRowBytesDen = 32;  // cols/2 + cols/32
};
template <>
struct WTraits<kWBf16> {
  static constexpr int kRowBytesNum = 2, kRowBytesDen = 1;
};

__host__ __device__ inline int64_t gemv_row_bytes(int wf, int cols) {
  return wf == kWMxfp4 ? (int64_t)cols / 2 + cols / 32 : (int64_t)cols * 2;
}

// Dot product of one MXFP4 group (16 bytes of codes) with 32 f16 activations,
// returned in fp32 (before the group scale).
__device__ __forceinline__ float dot_group_mxfp4(const uint32_t (&w)[16], const uint32_t (&xv)[16]) {
  uint32_t c0 = hmul2(w[0], xv[0]), c1 = hmul2(w[1], xv[1]);
  uint32_t c2 = hmul2(w[2], xv[2]), c3 = hmul2(w[3], xv[3]);
#pragma unroll
  for (int m = 4; m < 16; m += 4) {
    c0 = hfma2(w[m + 0], xv[m + 0], c0);
    c1 = hfma2(w[m + 1], xv[m + 1], c1);
    c2 = hfma2(w[m + 2], xv[m + 2], c2);
    c3 = hfma2(w[m + 3], xv[m + 3], c3);
  }
  float acc = add_f16x2_to_f32(c0, 0.f);
  acc = add_f16x2_to_f32(c1, acc);
  acc = add_f16x2_to_f32(c2, acc);
  return add_f16x2_to_f32(c3, acc);
}

template <int WF, int P, int RBI, int NTP>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(const GemvArgs args) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[kGemvStages];
  __shared__ int32_t s_active[1024];
  __shared__ int32_t s_cnt[kGemvThreads];
  __shared__ float s_red[kGemvRedFloats];

  const int tid = threadIdx.x;
  const int cols = args.a.cols, rows = args.a.rows;
  const int gpr = cols / 32;          // groups per weight row
  const int rp = kGemvThreads / gpr;  // rows processed in parallel
  const int g = tid % gpr, q = tid / gpr;
  const int seg = gpr < 32 ? gpr : 32;  // lanes holding one row's partials within a warp
  const int rb = args.rb;
  const int64_t row_bytes = gemv_row_bytes(WF, cols);
  const int64_t stage_bytes = ((int64_t)P * rb * row_bytes + 127) / 128 * 128;

  // ---- active experts (those with at least one pair) -----------------------
  int n_active;
  if (args.offsets != nullptr) {
    const int E = args.E;
    const int per = (E + kGemvThreads - 1) / kGemvThreads;
    int c = 0;
    for (int e = tid * per; e < min(E, tid * per + per); ++e) c += args.offsets[e + 1] > args.offsets[e];
    s_cnt[tid] = c;
    __syncthreads();
    if (tid == 0) {
      int run = 0;
      for (int i = 0; i < kGemvThreads; ++i) { const int v = s_cnt[i]; s_cnt[i] = run; run += v; }
      s_red[0] = __int_as_float(run);
    }
    __syncthreads();
    int w = s_cnt[tid];
    for (int e = tid * per; e < min(E, tid * per + per); ++e)
      if (args.offsets[e + 1] > args.offsets[e]) s_active[w++] = e;
    n_active = __float_as_int(s_red[0]);
    __syncthreads();
  } else {
    n_active = args.n_single > 0 ? 1 : 0;
    if (tid == 0) s_active[0] = 0;
    __syncthreads();
  }
  const int units_per_expert = rows / rb;
  const int n_units = n_active * units_per_expert;
  const int u_begin = (int)((int64_t)n_units * blockIdx.x / gridDim.x);
  const int u_end = (int)((int64_t)n_units * (blockIdx.x + 1) / gridDim.x);
  if (u_begin >= u_end) return;

  if (tid == 0) {
    for (int s = 0; s < kGemvStages; ++s) mbar_init(&full_bar[s], 1);  // all slots; n_stages used
    fence_mbar_init();
  }
  __syncthreads();

  const uint64_t pol = policy_evict_first();
  auto issue = [&](int u, int s) {
    const int e = s_active[u / units_per_expert];
    const int r0 = (u % units_per_expert) * rb;
    uint8_t* dst = smem + (int64_t)s * stage_bytes;
    const uint32_t bytes = (uint32_t)(P * rb * row_bytes);
    mbar_arrive_expect_tx(&full_bar[s], bytes);
#pragma unroll
    for (int p = 0; p < P; ++p) {
      const GemvProj& pr = p == 0 ? args.a : args.b;
      const uint8_t* blob = pr.base + (int64_t)e * pr.expert_bytes;
      uint8_t* d = dst + (int64_t)p * rb * row_bytes;
      if (WF == kWMxfp4) {
        bulk_g2s_stream(d, blob + (int64_t)r0 * (cols / 2), (uint32_t)rb * (cols / 2), &full_bar[s], pol);
        bulk_g2s_stream(d + (int64_t)rb * (cols / 2), blob + (int64_t)rows * (cols / 2) + (int64_t)r0 * (cols / 32),
                        (uint32_t)rb * (cols / 32), &full_bar[s], pol);
      } else {
        bulk_g2s_stream(d, blob + (int64_t)r0 * cols * 2, (uint32_t)rb * cols * 2, &full_bar[s], pol);
      }
    }
  };
  const int NS = args.n_stages;
  if (tid == 0)
    for (int k = 0; k < NS && u_begin + k < u_end; ++k) issue(u_begin + k, k);

  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(args.xin);
  const float* xf = static_cast<const float*>(args.xin);

  for (int u = u_begin; u < u_end; ++u) {
    const int k = u - u_begin, s = k % NS;
    const int e = s_active[u / units_per_expert];
    const int r0 = (u % units_per_expert) * rb;
    int pos0, n_tok;
    if (args.offsets != nullptr) { pos0 = args.offsets[e]; n_tok = args.offsets[e + 1] - pos0; }
    else { pos0 = 0; n_tok = args.n_single; }
    // all threads agree on the outcome of the (bounded) wait
    if (!__syncthreads_and(mbar_wait(&full_bar[s], (k / NS) & 1))) {
      if (tid == 0) {
        set_error(kErrWaitGemv);
        // let every copy already issued land before the CTA's shared memory goes away
        for (int k2 = k + 1; k2 < min(u_end - u_begin, k + NS); ++k2)
          mbar_wait(&full_bar[k2 % NS], (k2 / NS) & 1);
      }
      return;
    }
    const uint8_t* st = smem + (int64_t)s * stage_bytes;

    for (int j0 = 0; j0 < n_tok; j0 += NTP) {
      // ---- activations of this pass, columns [32 g, 32 g + 32) ------------
      // MXFP4: f16x2 pairs; bf16 weights: fp32 values.
      uint32_t xv[NTP][16];
      float xs[WF == kWBf16 ? NTP : 1][WF == kWBf16 ? 32 : 1];
#pragma unroll
      for (int j = 0; j < NTP; ++j) {
        const bool ok = j0 + j < n_tok;
        if (!ok) continue;
        int row = 0;
        if (ok) {
          const int pos = pos0 + j0 + j;
          row = args.perm ? args.perm[pos] / args.K : pos;
        }
        if (args.xin_f32) {
          const float4* src = reinterpret_cast<const float4*>(xf + (int64_t)row * cols + g * 32);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float4 v = ok ? __ldg(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
            if (WF == kWMxfp4) {
              xv[j][2 * c] = f32x2_to_f16x2(v.x, v.y);
              xv[j][2 * c + 1] = f32x2_to_f16x2(v.z, v.w);
            } else {
              xs[WF == kWBf16 ? j : 0][4 * c] = v.x; xs[WF == kWBf16 ? j : 0][4 * c + 1] = v.y;
              xs[WF == kWBf16 ? j : 0][4 * c + 2] = v.z; xs[WF == kWBf16 ? j : 0][4 * c + 3] = v.w;
            }
          }
        } else {
          const uint4* src = reinterpret_cast<const uint4*>(xb + (int64_t)row * cols + g * 32);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 v = ok ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
            const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if (WF == kWMxfp4) {
                xv[j][4 * c + i] = bf16x2_to_f16x2(vv[i]);
              } else {
                xs[WF == kWBf16 ? j : 0][8 * c + 2 * i] = __uint_as_float(vv[i] << 16);
                xs[WF == kWBf16 ? j : 0][8 * c + 2 * i + 1] = __uint_as_float(vv[i] & 0xFFFF0000u);
              }
            }
          }
        }
      }

      // ---- partial dot products ---------------------------------------------
      float part[P][RBI][NTP];
#pragma unroll
      for (int p = 0; p < P; ++p) {
        const uint8_t* pst = st + (int64_t)p * rb * row_bytes;
#pragma unroll
        for (int ri = 0; ri < RBI; ++ri) {
          const int r = q + ri * rp;
          if (WF == kWMxfp4) {
            const uint4 nb = *reinterpret_cast<const uint4*>(pst + (int64_t)r * (cols / 2) + g * 16);
            const float sc = e8m0_to_f32(pst[(int64_t)rb * (cols / 2) + (int64_t)r * (cols / 32) + g]);
            uint32_t w[16];
            {
              uint32_t t4[4];
              e2m1x8_to_f16x2(nb.x, t4); w[0] = t4[0]; w[1] = t4[1]; w[2] = t4[2]; w[3] = t4[3];
              e2m1x8_to_f16x2(nb.y, t4); w[4] = t4[0]; w[5] = t4[1]; w[6] = t4[2]; w[7] = t4[3];
              e2m1x8_to_f16x2(nb.z, t4); w[8] = t4[0]; w[9] = t4[1]; w[10] = t4[2]; w[11] = t4[3];
              e2m1x8_to_f16x2(nb.w, t4); w[12] = t4[0]; w[13] = t4[1]; w[14] = t4[2]; w[15] = t4[3];
            }
#pragma unroll
            for (int j = 0; j < NTP; ++j)
              part[p][ri][j] = (j0 + j < n_tok) ? dot_group_mxfp4(w, xv[j]) * sc : 0.f;
          } else {
            const uint4* wr = reinterpret_cast<const uint4*>(pst + (int64_t)r * cols * 2 + g * 64);
            float acc[NTP];
#pragma unroll
            for (int j = 0; j < NTP; ++j) acc[j] = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint4 v = wr[c];
              const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float wlo = __uint_as_float(vv[i] << 16), whi = __uint_as_float(vv[i] & 0xFFFF0000u);
#pragma unroll
                for (int j = 0; j < NTP; ++j) {
                  if (j0 + j < n_tok) {
                    acc[j] = fmaf(wlo, xs[WF == kWBf16 ? j : 0][8 * c + 2 * i], acc[j]);
                    acc[j] = fmaf(whi, xs[WF == kWBf16 ? j : 0][8 * c + 2 * i + 1], acc[j]);
                  }
                }
              }
            }
#pragma unroll
            for (int j = 0; j < NTP; ++j) part[p][ri][j] = acc[j];
          }
        }
      }

      // ---- reduce over the gpr threads of each row ----------------------------
#pragma unroll
      for (int p = 0; p < P; ++p)
#pragma unroll
        for (int ri = 0; ri < RBI; ++ri)
#pragma unroll
          for (int j = 0; j < NTP; ++j) {
            if (j0 + j < n_tok) {
              float v = part[p][ri][j];
              for (int o = seg >> 1; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
              part[p][ri][j] = v;
            }
          }
      // one writer per segment: s_red[segment][p][ri][j]
      const int seg_id = tid / seg;
      if (tid % seg == 0) {
#pragma unroll
        for (int p = 0; p < P; ++p)
#pragma unroll
          for (int ri = 0; ri < RBI; ++ri)
#pragma unroll
            for (int j = 0; j < NTP; ++j) s_red[((seg_id * P + p) * RBI + ri) * NTP + j] = part[p][ri][j];
      }
      __syncthreads();
      // outputs: (row slot qq, ri, j); row slot qq is held by segments
      // [qq * gpr / seg, (qq + 1) * gpr / seg)
      const int nseg_row = gpr / seg;
      for (int o = tid; o < rp * RBI * NTP; o += kGemvThreads) {
        const int j = o % NTP, ri = (o / NTP) % RBI, qq = o / (NTP * RBI);
        if (j0 + j >= n_tok) continue;
        float v[P];
#pragma unroll
        for (int p = 0; p < P; ++p) {
          float acc = 0.f;
          for (int sgi = 0; sgi < nseg_row; ++sgi)
            acc += s_red[(((qq * nseg_row + sgi) * P + p) * RBI + ri) * NTP + j];
          v[p] = acc;
        }
        const float res = (P == 2) ? silu_clamped_swiglu(v[0], v[P - 1], args.limit) : v[0];
        const int row = r0 + qq + ri * rp;
        args.out[(int64_t)(pos0 + j0 + j) * args.out_ld + row] = res;
      }
      __syncthreads();
    }

    // stage s is free again: refill it with unit u + NS
    if (tid == 0 && u + NS < u_end) issue(u + NS, s);
  }
}

}  // namespace moe
