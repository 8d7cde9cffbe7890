// Host-only check of moe_expert_gemm's launch arguments for every token count
// (no GPU, no CUDA call): the path choice, that each argument points at the
// buffer it should, that the workspace carve-up fits the advertised size, and
// that every pipeline plan fits TMEM (512 columns), shared memory and one CTA
// per SM.  Prints one line per failure and "ok <cases>" at the end; exit 0
// when nothing failed.
#include <cstdio>
#include <cstdint>

#include "expert_launch.h"

using namespace moe;

static int fails = 0;
#define CHECK(c, ...)                                       \
  do {                                                      \
    if (!(c)) {                                             \
      if (++fails <= 40) {                                  \
        printf("FAIL %s: ", #c);                            \
        printf(__VA_ARGS__);                                \
        printf("\n");                                       \
      }                                                     \
    }                                                       \
  } while (0)

static moe_mxfp4_proj proj(uintptr_t base, int rows, int cols) {
  moe_mxfp4_proj p;
  p.base = reinterpret_cast<const uint8_t*>(base);
  p.expert_bytes = (int64_t)rows * cols / 2 + (int64_t)rows * cols / 32;
  p.rows = rows;
  p.cols = cols;
  return p;
}

static void check_mx_plan(const MxArgs& a, int mode, const char* name, int T) {
  const int n = a.term_acc ? a.n_chunk : a.parts * a.n_chunk;  // the MMA's N
  CHECK(a.term_acc == 0 || a.term_acc == 1, "%s T=%d layout", name, T);
  CHECK(n <= kMxNMax && n % 16 == 0, "%s T=%d N=%d", name, T, n);
  CHECK(a.acc_cols >= n && a.acc_cols % 32 == 0, "%s T=%d", name, T);
  CHECK(a.acc_bufs >= 1 && a.acc_bufs <= kMxMaxBufs && a.acc_bufs <= (a.max_bufs > 1 ? a.max_bufs : 1),
        "%s T=%d accumulator sets", name, T);
  // token scales: stacked, N <= 128 indices in 4 columns; summed, 4 columns
  // (128 tokens) per term; each term block starts on a multiple of 4
  CHECK(a.tok_cols == (a.term_acc ? 4 * a.parts : 4) && a.sf_kt == 8 + a.tok_cols, "%s T=%d scale cols", name, T);
  CHECK(a.term_acc ? a.n_chunk <= 128 : a.parts * a.n_chunk <= 128, "%s T=%d scale coverage", name, T);
  CHECK(a.acc_bufs * 2 * a.acc_cols + a.sf_stages * a.sf_kt * a.g <= kTcTmemCols, "%s T=%d TMEM", name, T);
  CHECK(a.sf_stages >= 2 && a.sf_stages <= kMxMaxSfStages && a.stages >= 2, "%s T=%d rings", name, T);
  CHECK((a.cols / kMxKT) % a.g == 0, "%s T=%d G", name, T);
  CHECK(a.stage_bytes % 1024 == 0, "%s T=%d stage", name, T);
  // a stage holds kps K-tiles of both weight tiles and every term's n_chunk
  // token rows; two-K-tile stages need an even K-tile count and scale stage
  CHECK(a.kps == 1 || a.kps == 2, "%s T=%d kps", name, T);
  CHECK(a.stage_bytes == a.kps * (2 * kMxTileBytes + a.parts * a.n_chunk * 128), "%s T=%d stage size", name, T);
  CHECK((a.cols / kMxKT) % a.kps == 0 && a.g % a.kps == 0, "%s T=%d kps divides", name, T);
  CHECK(a.n_chunk <= 256 && a.kps * a.parts <= 256, "%s T=%d box dims", name, T);
  // shared memory: weight stages, then the scale ring (TMA-fed E8M0 rows),
  // then the unit prefix and offsets copy
  CHECK(a.off_sc == a.stages * a.stage_bytes, "%s T=%d scale ring offset", name, T);
  CHECK(a.off_prefix == a.off_sc + a.sf_stages * a.sc_slot_bytes, "%s T=%d prefix", name, T);
  if (a.tma_scales) {
    // a slot holds both weight tiles' 128 rows and every term's n_chunk token
    // rows of 4 G bytes; TMA rows are 16-byte multiples with 16-byte strides
    CHECK(a.sc_slot_bytes >= (256 + a.parts * a.n_chunk) * 4 * a.g && a.sc_slot_bytes % 128 == 0,
          "%s T=%d scale slot", name, T);
    CHECK(a.g >= 4 && (4 * a.g) % 16 == 0 && (a.cols / 32) % 16 == 0, "%s T=%d scale boxes", name, T);
    CHECK(a.off_sc % 1024 == 0, "%s T=%d scale ring alignment", name, T);
  } else {
    CHECK(a.sc_slot_bytes == 0, "%s T=%d scale slot without TMA", name, T);
  }
  CHECK(a.off_prefix + 2 * (a.E + 1) * 4 + 1024 <= a.smem_bytes, "%s T=%d prefix room", name, T);
  CHECK(a.smem_bytes <= kTcSmemMax && 2 * a.smem_bytes > kTcSmemMax, "%s T=%d smem %d", name, T, a.smem_bytes);
  CHECK(a.rows % (mode == 0 ? 128 : 256) == 0, "%s T=%d rows", name, T);
}

static void check_tc_plan(TcArgs a, const char* name, int T) {
  CHECK(tc_plan(a, kAMxfp4), "%s T=%d plan", name, T);
  CHECK(a.acc_cols >= a.n_chunk, "%s T=%d", name, T);
  CHECK(2 * a.acc_cols + a.stages * kTcStageCols <= kTcTmemCols, "%s T=%d TMEM", name, T);
  CHECK(a.stages >= 2 && a.w_slots >= 2, "%s T=%d rings", name, T);
  // the token ring runs at least as deep as the TMEM stages, and one deeper
  // with at least three weight stages in flight where the shared memory allows
  CHECK(a.b_stages >= a.stages && a.b_stages <= kTcMaxStages, "%s T=%d token ring", name, T);
  CHECK(a.b_stages == a.stages || a.w_slots * a.st_per_slot >= 3, "%s T=%d weight stages", name, T);
  CHECK(a.st_per_slot * 64 == a.w_inner && (a.a_cols / 2) % a.w_inner == 0, "%s T=%d weight box", name, T);
  // shared memory: weight slots, then the token ring, the E8M0 rows, the prefix
  CHECK(a.off_b == a.w_slots * a.w_slot_bytes && a.off_sc == a.off_b + a.b_stages * kTcKG * a.n_chunk * 128,
        "%s T=%d offsets", name, T);
  CHECK(a.smem_bytes <= kTcSmemMax && 2 * a.smem_bytes > kTcSmemMax, "%s T=%d smem %d", name, T, a.smem_bytes);
}

static int check_shape(const moe_dims& d, int t_max, const char* shape) {
  const int H = d.hidden, I = d.inter;
  const moe_mxfp4_proj gate = proj(0x10000000, I, H), up = proj(0x20000000, I, H), down = proj(0x30000000, H, I);
  const int32_t* offsets = reinterpret_cast<const int32_t*>(uintptr_t(0x40000000));
  float* y = reinterpret_cast<float*>(uintptr_t(0x50000000));
  uint8_t* ws = reinterpret_cast<uint8_t*>(uintptr_t(0x1000000000ull));
  size_t prev_ws = 0;
  int cases = 0;
  for (int T = 1; T <= t_max; T += (T < 1200 ? 1 : 97)) {
    ++cases;
    const size_t ws_bytes = expert_gemm_ws_bytes(d, T);
    CHECK(ws_bytes >= prev_ws, "%s T=%d workspace shrinks", shape, T);
    prev_ws = ws_bytes;
    const int64_t P = (int64_t)T * d.top_k;
    if (use_block_scaled(T, d.top_k, d.n_experts)) {
      MxLaunch L;
      CHECK(mx_launch_args(d, T, gate, up, down, offsets, y, ws, L), "%s T=%d block-scaled args", shape, T);
      const MxArgs &g = L.g, &dn = L.d;
      CHECK(L.pairs == P && g.pairs == P && dn.pairs == P, "%s T=%d pairs", shape, T);
      CHECK(g.w0 == gate.base && g.w1 == up.base && dn.w0 == down.base && dn.w1 == nullptr, "%s T=%d weights", shape, T);
      CHECK(g.expert_bytes == gate.expert_bytes && dn.expert_bytes == down.expert_bytes, "%s T=%d strides", shape, T);
      CHECK(g.offsets == offsets && dn.offsets == offsets, "%s T=%d offsets", shape, T);
      CHECK(g.rows == I && g.cols == H && dn.rows == H && dn.cols == I, "%s T=%d dims", shape, T);
      CHECK(g.b_scale == L.xs && g.out == L.hq && g.out_scale == L.hs, "%s T=%d gate/up buffers", shape, T);
      CHECK(dn.b_scale == L.hs && dn.out == y && dn.out_scale == nullptr, "%s T=%d down buffers", shape, T);
      CHECK(dn.parts == g.out_parts, "%s T=%d h terms", shape, T);
      CHECK(g.limit == d.swiglu_limit && g.E == d.n_experts && dn.E == d.n_experts, "%s T=%d scalars", shape, T);
      // the four workspace regions, in order, inside the advertised size
      CHECK(L.xq == ws, "%s T=%d xq", shape, T);
      CHECK(L.xq + (size_t)g.parts * P * H <= L.xs, "%s T=%d xq/xs overlap", shape, T);
      CHECK(L.xs + (size_t)g.parts * P * (H / 32) <= L.hq, "%s T=%d xs/hq overlap", shape, T);
      CHECK(L.hq + (size_t)g.out_parts * P * I <= L.hs, "%s T=%d hq/hs overlap", shape, T);
      CHECK(L.hs + (size_t)dn.parts * P * (I / 32) <= ws + ws_bytes, "%s T=%d hs past the workspace", shape, T);
      check_mx_plan(g, 0, "gate/up", T);
      check_mx_plan(dn, 1, "down", T);
    } else {
      TcLaunch L;
      CHECK(tc_launch_args(d, T, gate, up, down, offsets, y, ws, L), "%s T=%d dequantising args", shape, T);
      const TcArgs &g = L.g, &dn = L.d;
      CHECK(L.pairs == P, "%s T=%d pairs", shape, T);
      CHECK(g.w0 == gate.base && g.w1 == up.base && dn.w0 == down.base && dn.w1 == nullptr, "%s T=%d weights", shape, T);
      CHECK(g.offsets == offsets && dn.offsets == offsets, "%s T=%d offsets", shape, T);
      CHECK(g.out == L.h16 && dn.out == y, "%s T=%d outputs", shape, T);
      CHECK(reinterpret_cast<uint8_t*>(L.x16) == ws, "%s T=%d x16", shape, T);
      CHECK(reinterpret_cast<uint8_t*>(L.x16) + (size_t)P * H * 2 <= reinterpret_cast<uint8_t*>(L.h16),
            "%s T=%d x16/h16 overlap", shape, T);
      CHECK(reinterpret_cast<uint8_t*>(L.h16) + (size_t)P * I * 2 <= ws + ws_bytes, "%s T=%d h16 past the workspace",
            shape, T);
      check_tc_plan(g, "gate/up", T);
      check_tc_plan(dn, "down", T);
    }
  }
  return cases;
}

int main() {
  const moe_dims v4 = {4096, 2048, 256, 6, 1.5f, 10.0f};
  const moe_dims tiny = {256, 128, 16, 2, 1.5f, 10.0f};
  int cases = check_shape(v4, 8192, "v4") + check_shape(tiny, 8192, "tiny");
  if (fails) {
    printf("%d failures\n", fails);
    return 1;
  }
  printf("ok %d\n", cases);
  return 0;
}
