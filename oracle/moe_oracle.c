/*
 * CPU oracle of the routed MoE layer (MXFP4 experts, sqrt-softplus routing).
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA path and never calls it.
 *
 * Plain, slow and written to be checked by eye: every value is converted from
 * the exact input bits to double and all arithmetic is fp64.  No blocking, no
 * fusion, no reordering beyond what the definitions state.
 *
 * Passages followed (page title, section):
 *  [MOBIUS]  "DeepSeek-V4-Flash export design" (ONNX Runtime mobius), Source
 *            configuration, MoE bullet: 256 routed experts, top 6, intermediate
 *            2048, one shared expert, scale 1.5, normalized sqrt(softplus(logit))
 *            routing; first three layers pick experts from a token-id hash
 *            table.  Section "V3 reuse and V4 differences": clamped SwiGLU.
 *  [MAP-MOE] "Model techniques map" (DeepSeek-V4-Flash), row "Mixture of
 *            experts": top-k of (scores + e_score_correction_bias).
 *  [MAP-BAL] same page, row "Auxiliary-loss-free load balancing": the bias is
 *            used only to select; weights are gathered from unbiased scores.
 *  [MAP-SH]  same page, row "Shared expert": routed output + shared expert of
 *            the same input.
 *  [MAP-SW]  same page, row "SwiGLU feed-forward": gate clamped above at the
 *            limit, up clamped to [-limit, limit], silu(gate) * up, then down.
 *  [PULSAR]  "ElytronAI / DeepSeek-v4-Flash", sections Layout and Sizes:
 *            experts of one projection stored back to back, expert xid at
 *            base + xid * expert_bytes; E2M1 nibble plane plus E8M0 group-32
 *            scale plane.
 *  [JANG]    "DeepSeek-V4-Flash-0731-JANG", Dynamic affine recipe table: the
 *            router is kept in f32 (its weight is an fp32 input here); the
 *            affine low-bit expert format (oracle_affine_*: the oracle step
 *            of a variant whose CUDA path is not built).
 *
 * Readings where the pages are silent (each one a choice of this oracle):
 *  - nibble order: the low nibble of a byte is the even column;
 *  - blob order: nibble plane [rows][cols/2], then scale plane [rows][cols/32];
 *  - the scale group is 32 consecutive input columns of one output row;
 *  - normalisation is over the K selected unbiased scores, times the scale;
 *  - hash layers use the same sqrt-softplus scores gathered at the hashed ids;
 *  - top-k ties go to the lower expert id; ids are emitted in descending
 *    biased score (hash layers: table order);
 *  - the shared expert uses the same clamped SwiGLU.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* Element formats [PULSAR Sizes]: E2M1 codes and E8M0 group scales.   */
/* ------------------------------------------------------------------ */

/* E2M1 (OCP MX): bit 3 sign, bits 2-1 exponent (bias 1), bit 0 mantissa. */
static const double E2M1_VALUE[16] = {
    +0.0, +0.5, +1.0, +1.5, +2.0, +3.0, +4.0, +6.0,
    -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0};

double oracle_e2m1(int code) { return E2M1_VALUE[code & 15]; }

/* E8M0: an unsigned biased exponent, value 2^(e-127); e = 255 is NaN. */
double oracle_e8m0(int e) { return e == 255 ? NAN : ldexp(1.0, e - 127); }

/* Bytes of one expert of one projection: nibble plane + scale plane. */
int64_t oracle_expert_bytes(int64_t rows, int64_t cols) {
  return rows * cols / 2 + rows * cols / 32;
}

/* Dequantise one row of an expert blob into out[cols] (exact in fp64). */
static void dequant_row(const uint8_t* blob, int rows, int cols, int r, double* out) {
  const uint8_t* nib = blob;
  const uint8_t* scl = blob + (int64_t)rows * cols / 2;
  for (int c = 0; c < cols; ++c) {
    uint8_t byte = nib[(int64_t)r * (cols / 2) + c / 2];
    int code = (c % 2 == 0) ? (byte & 15) : (byte >> 4);
    int e = scl[(int64_t)r * (cols / 32) + c / 32];
    out[c] = oracle_e2m1(code) * oracle_e8m0(e);
  }
}

/* W[r][c] for the whole blob into out[rows*cols]. */
void oracle_dequant(const uint8_t* blob, int rows, int cols, double* out) {
  for (int r = 0; r < rows; ++r) dequant_row(blob, rows, cols, r, out + (int64_t)r * cols);
}

static double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* ------------------------------------------------------------------ */
/* Affine low-bit experts [JANG Dynamic affine recipe]: b-bit codes q in */
/* [0, 2^b - 1] with one scale and one bias per group of G consecutive   */
/* input columns of a row, w = scale * q + bias (2-bit G32 down, 2-bit   */
/* G64 gate/up, 3-bit G64 gate in the lifted layers, 8-bit G64 shared).  */
/* Readings (the page gives bits and group sizes per tensor role only):  */
/*  - the codes of a row are one little-endian bit stream: column c      */
/*    holds bits [c*b, c*b + b) of the row's cols*b/8 bytes, the lowest  */
/*    bit first;                                                         */
/*  - scales and biases are bf16;                                        */
/*  - blob: codes [rows][cols*b/8], then scales [rows][cols/G], then     */
/*    biases [rows][cols/G], experts back to back as for MXFP4.          */
/* ------------------------------------------------------------------ */

/* Bytes of one affine expert blob; -1 for a shape the format cannot hold. */
int64_t oracle_affine_expert_bytes(int64_t rows, int64_t cols, int bits, int group) {
  if (rows <= 0 || bits < 1 || bits > 8 || group <= 0 || cols <= 0 || cols % group || (cols * bits) % 8 ||
      (rows * cols * bits / 8) % 2)
    return -1;
  return rows * cols * bits / 8 + 2 * 2 * rows * (cols / group);
}

/* Code of column c from a row's bit stream, one bit at a time. */
static int affine_code(const uint8_t* row_codes, int c, int bits) {
  int q = 0;
  for (int i = 0; i < bits; ++i) {
    const int64_t bit = (int64_t)c * bits + i;
    q |= ((row_codes[bit / 8] >> (bit % 8)) & 1) << i;
  }
  return q;
}

static void affine_dequant_row(const uint8_t* blob, int rows, int cols, int bits, int group, int r,
                               double* out) {
  const int64_t row_bytes = (int64_t)cols * bits / 8;
  const uint8_t* codes = blob + (int64_t)r * row_bytes;
  const uint8_t* scales = blob + (int64_t)rows * row_bytes;
  const uint8_t* biases = scales + 2 * (int64_t)rows * (cols / group);
  for (int c = 0; c < cols; ++c) {
    const int64_t gi = (int64_t)r * (cols / group) + c / group;
    uint16_t sb, bb;
    memcpy(&sb, scales + 2 * gi, 2);
    memcpy(&bb, biases + 2 * gi, 2);
    out[c] = bf16_to_double(sb) * (double)affine_code(codes, c, bits) + bf16_to_double(bb);
  }
}

/* W[r][c] of an affine blob into out[rows*cols]; -1 for a bad shape. */
int oracle_affine_dequant(const uint8_t* blob, int rows, int cols, int bits, int group, double* out) {
  if (oracle_affine_expert_bytes(rows, cols, bits, group) < 0) return -1;
  for (int r = 0; r < rows; ++r) affine_dequant_row(blob, rows, cols, bits, group, r, out + (int64_t)r * cols);
  return 0;
}

/* ------------------------------------------------------------------ */
/* Routing [MOBIUS MoE bullet], [MAP-MOE], [MAP-BAL]                   */
/* ------------------------------------------------------------------ */

/* sqrt(softplus(z)); softplus(z) = log(1 + e^z) = log1p(e^-|z|) + max(z, 0). */
double oracle_sqrt_softplus(double z) {
  double sp = log1p(exp(-fabs(z))) + (z > 0 ? z : 0.0);
  return sqrt(sp);
}

/* scores[e] = sqrt(softplus(x . Wr[e])) for one token. */
static void token_scores(const uint16_t* xrow, int H, const float* wr, int E, double* s) {
  for (int e = 0; e < E; ++e) {
    double z = 0.0;
    for (int h = 0; h < H; ++h) z += bf16_to_double(xrow[h]) * (double)wr[(int64_t)e * H + h];
    s[e] = oracle_sqrt_softplus(z);
  }
}

/* w_k = alpha * s[idx_k] / sum_j s[idx_j]. */
static void normalise(const double* s, const int32_t* idx, int K, double alpha, double* w) {
  double sum = 0.0;
  for (int k = 0; k < K; ++k) sum += s[idx[k]];
  for (int k = 0; k < K; ++k) w[k] = alpha * s[idx[k]] / sum;
}

/*
 * Learned routing for T tokens.  idx[T][K] holds the K experts of largest
 * s + bias (ties to the lower id), in descending biased score; w[T][K] the
 * normalised unbiased scores times alpha.  gap[t] (nullable) is the biased
 * score of the K-th pick minus the largest unpicked biased score.
 * scores (nullable) receives s[T][E].
 */
void oracle_route(const uint16_t* x, int T, int H, const float* wr, const float* bias, int E,
                  int K, double alpha, int32_t* idx, double* w, double* scores, double* gap) {
  double* s = (double*)malloc(sizeof(double) * E);
  char* taken = (char*)malloc(E);
  for (int t = 0; t < T; ++t) {
    token_scores(x + (int64_t)t * H, H, wr, E, s);
    if (scores) memcpy(scores + (int64_t)t * E, s, sizeof(double) * E);
    memset(taken, 0, E);
    for (int k = 0; k < K; ++k) {
      int best = -1;
      double bv = 0.0;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        double v = s[e] + (bias ? (double)bias[e] : 0.0);
        if (best < 0 || v > bv) { best = e; bv = v; } /* strict: ties keep the lower id */
      }
      taken[best] = 1;
      idx[(int64_t)t * K + k] = best;
    }
    normalise(s, idx + (int64_t)t * K, K, alpha, w + (int64_t)t * K);
    if (gap) {
      double kth = s[idx[(int64_t)t * K + K - 1]] +
                   (bias ? (double)bias[idx[(int64_t)t * K + K - 1]] : 0.0);
      double next = -INFINITY;
      for (int e = 0; e < E; ++e)
        if (!taken[e]) {
          double v = s[e] + (bias ? (double)bias[e] : 0.0);
          if (v > next) next = v;
        }
      gap[t] = kth - next;
    }
  }
  free(s);
  free(taken);
}

/*
 * Hash routing (first three layers) [MOBIUS MoE bullet]: idx = table[tok[t]]
 * in table order; weights as for learned routing, from the router's unbiased
 * scores at those ids.
 */
void oracle_route_hash(const uint16_t* x, int T, int H, const float* wr, int E, int K,
                       double alpha, const int32_t* tok, const int32_t* table, int vocab,
                       int32_t* idx, double* w) {
  double* s = (double*)malloc(sizeof(double) * E);
  for (int t = 0; t < T; ++t) {
    int v = tok[t];
    if (v < 0 || v >= vocab) v = 0; /* callers validate; keep the oracle total */
    token_scores(x + (int64_t)t * H, H, wr, E, s);
    for (int k = 0; k < K; ++k) idx[(int64_t)t * K + k] = table[(int64_t)v * K + k];
    normalise(s, idx + (int64_t)t * K, K, alpha, w + (int64_t)t * K);
  }
  free(s);
}

/* ------------------------------------------------------------------ */
/* Grouping: stable counting sort of the T*K (token, slot) pairs by     */
/* expert.  Pair p = t*K + k.  offsets[E+1] exclusive prefix of counts; */
/* perm[pos] = p in (expert, p) order; inv[p] = pos.                    */
/* ------------------------------------------------------------------ */
void oracle_permute(const int32_t* idx, int T, int K, int E, int32_t* offsets, int32_t* perm,
                    int32_t* inv) {
  int64_t n = (int64_t)T * K;
  for (int e = 0; e <= E; ++e) offsets[e] = 0;
  for (int64_t p = 0; p < n; ++p) offsets[idx[p] + 1] += 1;
  for (int e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
  int32_t* next = (int32_t*)malloc(sizeof(int32_t) * (E > 0 ? E : 1));
  for (int e = 0; e < E; ++e) next[e] = offsets[e];
  for (int64_t p = 0; p < n; ++p) {
    int e = idx[p];
    perm[next[e]] = (int32_t)p;
    inv[p] = next[e];
    next[e] += 1;
  }
  free(next);
}

/* ------------------------------------------------------------------ */
/* Expert FFN [MAP-SW], [MOBIUS V3 reuse and V4 differences]:           */
/*   g = Wg x, u = Wu x, h = silu(min(g, L)) * clamp(u, -L, L), y = Wd h */
/* ------------------------------------------------------------------ */
static double silu(double v) { return v / (1.0 + exp(-v)); }

double oracle_swiglu(double g, double u, double limit) {
  double gc = g < limit ? g : limit;
  double uc = u < -limit ? -limit : (u > limit ? limit : u);
  return silu(gc) * uc;
}

/*
 * One MXFP4 expert on n activation rows xs[n][H] (fp64), ys[n][H] out.
 * Gate/up blobs are [I][H]; the down blob is [H][I].  Each weight row is
 * dequantised once and applied to every row of xs.
 */
void oracle_expert_ffn(const uint8_t* g_blob, const uint8_t* u_blob, const uint8_t* d_blob,
                       int H, int I, double limit, const double* xs, int n, double* ys) {
  double* wrow = (double*)malloc(sizeof(double) * (H > I ? H : I));
  double* g = (double*)malloc(sizeof(double) * (int64_t)n * I);
  double* u = (double*)malloc(sizeof(double) * (int64_t)n * I);
  for (int r = 0; r < I; ++r) {
    dequant_row(g_blob, I, H, r, wrow);
    for (int j = 0; j < n; ++j) {
      double acc = 0.0;
      for (int c = 0; c < H; ++c) acc += wrow[c] * xs[(int64_t)j * H + c];
      g[(int64_t)j * I + r] = acc;
    }
    dequant_row(u_blob, I, H, r, wrow);
    for (int j = 0; j < n; ++j) {
      double acc = 0.0;
      for (int c = 0; c < H; ++c) acc += wrow[c] * xs[(int64_t)j * H + c];
      u[(int64_t)j * I + r] = acc;
    }
  }
  for (int64_t i = 0; i < (int64_t)n * I; ++i) g[i] = oracle_swiglu(g[i], u[i], limit);
  for (int r = 0; r < H; ++r) {
    dequant_row(d_blob, H, I, r, wrow);
    for (int j = 0; j < n; ++j) {
      double acc = 0.0;
      for (int c = 0; c < I; ++c) acc += wrow[c] * g[(int64_t)j * I + c];
      ys[(int64_t)j * H + r] = acc;
    }
  }
  free(wrow);
  free(g);
  free(u);
}

/*
 * One affine expert on n activation rows xs[n][H] (fp64), ys[n][H] out: the
 * same clamped SwiGLU FFN as oracle_expert_ffn with each projection in the
 * affine format of its own bits and group size.  -1 for a bad shape.
 */
int oracle_affine_expert_ffn(const uint8_t* g_blob, int g_bits, int g_group, const uint8_t* u_blob, int u_bits,
                             int u_group, const uint8_t* d_blob, int d_bits, int d_group, int H, int I,
                             double limit, const double* xs, int n, double* ys) {
  if (oracle_affine_expert_bytes(I, H, g_bits, g_group) < 0 || oracle_affine_expert_bytes(I, H, u_bits, u_group) < 0 ||
      oracle_affine_expert_bytes(H, I, d_bits, d_group) < 0)
    return -1;
  double* wrow = (double*)malloc(sizeof(double) * (H > I ? H : I));
  double* g = (double*)malloc(sizeof(double) * (int64_t)n * I);
  double* u = (double*)malloc(sizeof(double) * (int64_t)n * I);
  for (int r = 0; r < I; ++r) {
    affine_dequant_row(g_blob, I, H, g_bits, g_group, r, wrow);
    for (int j = 0; j < n; ++j) {
      double acc = 0.0;
      for (int c = 0; c < H; ++c) acc += wrow[c] * xs[(int64_t)j * H + c];
      g[(int64_t)j * I + r] = acc;
    }
    affine_dequant_row(u_blob, I, H, u_bits, u_group, r, wrow);
    for (int j = 0; j < n; ++j) {
      double acc = 0.0;
      for (int c = 0; c < H; ++c) acc += wrow[c] * xs[(int64_t)j * H + c];
      u[(int64_t)j * I + r] = acc;
    }
  }
  for (int64_t i = 0; i < (int64_t)n * I; ++i) g[i] = oracle_swiglu(g[i], u[i], limit);
  for (int r = 0; r < H; ++r) {
    affine_dequant_row(d_blob, H, I, d_bits, d_group, r, wrow);
    for (int j = 0; j < n; ++j) {
      double acc = 0.0;
      for (int c = 0; c < I; ++c) acc += wrow[c] * g[(int64_t)j * I + c];
      ys[(int64_t)j * H + r] = acc;
    }
  }
  free(wrow);
  free(g);
  free(u);
  return 0;
}

/* The bf16 shared expert [MAP-SH] on n rows: same clamped SwiGLU FFN. */
void oracle_shared_ffn(const uint16_t* wg, const uint16_t* wu, const uint16_t* wd, int H, int I,
                       double limit, const double* xs, int n, double* ys) {
  double* h = (double*)malloc(sizeof(double) * (int64_t)n * I);
  for (int j = 0; j < n; ++j) {
    const double* x = xs + (int64_t)j * H;
    for (int r = 0; r < I; ++r) {
      double g = 0.0, u = 0.0;
      for (int c = 0; c < H; ++c) {
        g += bf16_to_double(wg[(int64_t)r * H + c]) * x[c];
        u += bf16_to_double(wu[(int64_t)r * H + c]) * x[c];
      }
      h[(int64_t)j * I + r] = oracle_swiglu(g, u, limit);
    }
    for (int r = 0; r < H; ++r) {
      double y = 0.0;
      for (int c = 0; c < I; ++c) y += bf16_to_double(wd[(int64_t)r * I + c]) * h[(int64_t)j * I + c];
      ys[(int64_t)j * H + r] = y;
    }
  }
  free(h);
}

/* Combine [MAP-SH]: out[t] = shared[t] + sum_{k=0..K-1} w[t][k] * y_perm[inv[t*K+k]]. */
void oracle_combine(int T, int K, int H, const double* y_perm, const int32_t* inv, const double* w,
                    const double* shared, double* out) {
  for (int t = 0; t < T; ++t)
    for (int c = 0; c < H; ++c) {
      double acc = 0.0;
      for (int k = 0; k < K; ++k)
        acc += w[(int64_t)t * K + k] * y_perm[(int64_t)inv[(int64_t)t * K + k] * H + c];
      out[(int64_t)t * H + c] = (shared ? shared[(int64_t)t * H + c] : 0.0) + acc;
    }
}

/* ------------------------------------------------------------------ */
/* Whole layer on a subset of tokens (the layer is per token, so the    */
/* outputs of a subset are exactly those rows of the full output).     */
/* ------------------------------------------------------------------ */
typedef struct {
  int H, I, E, K;
  double limit;
  const double* xs;        /* [n_sel][H] */
  const int32_t* idx;      /* [n_sel][K] */
  const uint8_t* const* gate;
  const uint8_t* const* up;
  const uint8_t* const* down;
  int n_sel;
  double* y;               /* [n_sel][K][H] */
  const uint16_t *wg, *wu, *wd;
  double* ys;              /* [n_sel][H] */
  int next_job;            /* atomic job counter: jobs 0..E-1 experts, E.. shared tokens */
  int err;
} layer_job;

static void* layer_worker(void* arg) {
  layer_job* J = (layer_job*)arg;
  int64_t H = J->H;
  for (;;) {
    int job = __atomic_fetch_add(&J->next_job, 1, __ATOMIC_RELAXED);
    if (job >= J->E + J->n_sel) break;
    if (job < J->E) {
      int e = job, n = 0;
      for (int j = 0; j < J->n_sel; ++j)
        for (int k = 0; k < J->K; ++k) n += (J->idx[(int64_t)j * J->K + k] == e);
      if (n == 0) continue;
      if (!J->gate[e] || !J->up[e] || !J->down[e]) { __atomic_store_n(&J->err, 1, __ATOMIC_RELAXED); continue; }
      double* xs = (double*)malloc(sizeof(double) * n * H);
      double* ys = (double*)malloc(sizeof(double) * n * H);
      int m = 0;
      for (int j = 0; j < J->n_sel; ++j)
        for (int k = 0; k < J->K; ++k)
          if (J->idx[(int64_t)j * J->K + k] == e) memcpy(xs + (int64_t)(m++) * H, J->xs + j * H, sizeof(double) * H);
      oracle_expert_ffn(J->gate[e], J->up[e], J->down[e], J->H, J->I, J->limit, xs, n, ys);
      m = 0;
      for (int j = 0; j < J->n_sel; ++j)
        for (int k = 0; k < J->K; ++k)
          if (J->idx[(int64_t)j * J->K + k] == e)
            memcpy(J->y + ((int64_t)j * J->K + k) * H, ys + (int64_t)(m++) * H, sizeof(double) * H);
      free(xs);
      free(ys);
    } else if (J->wg) {
      int j = job - J->E;
      oracle_shared_ffn(J->wg, J->wu, J->wd, J->H, J->I, J->limit, J->xs + (int64_t)j * H, 1,
                        J->ys + (int64_t)j * H);
    }
  }
  return NULL;
}

/*
 * out[j][H] (fp64) for the tokens sel[0..n_sel) of x[T][H] (bf16 bits).
 * Routing is learned (bias nullable) unless table/tok are given (hash).
 * gate/up/down are per-expert blob pointers (E entries; only the experts the
 * selected tokens use are read).  wg/wu/wd (nullable) is the shared expert.
 * idx_out[n_sel][K], w_out[n_sel][K] (nullable) receive the routing.
 * Returns 0, or 1 if a needed expert pointer was NULL.
 */
int oracle_moe_layer(int H, int I, int E, int K, double alpha, double limit,
                     const uint16_t* x, int T, const int32_t* sel, int n_sel,
                     const float* wr, const float* bias,
                     const int32_t* tok, const int32_t* table, int vocab,
                     const uint8_t* const* gate, const uint8_t* const* up,
                     const uint8_t* const* down,
                     const uint16_t* wg, const uint16_t* wu, const uint16_t* wd,
                     int nthreads, double* out, int32_t* idx_out, double* w_out) {
  (void)T;
  uint16_t* xsel = (uint16_t*)malloc(sizeof(uint16_t) * (int64_t)n_sel * H);
  double* xs = (double*)malloc(sizeof(double) * (int64_t)n_sel * H);
  for (int j = 0; j < n_sel; ++j)
    for (int h = 0; h < H; ++h) {
      xsel[(int64_t)j * H + h] = x[(int64_t)sel[j] * H + h];
      xs[(int64_t)j * H + h] = bf16_to_double(x[(int64_t)sel[j] * H + h]);
    }
  int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (int64_t)n_sel * K);
  double* w = (double*)malloc(sizeof(double) * (int64_t)n_sel * K);
  if (table && tok) {
    int32_t* toks = (int32_t*)malloc(sizeof(int32_t) * (n_sel > 0 ? n_sel : 1));
    for (int j = 0; j < n_sel; ++j) toks[j] = tok[sel[j]];
    oracle_route_hash(xsel, n_sel, H, wr, E, K, alpha, toks, table, vocab, idx, w);
    free(toks);
  } else {
    oracle_route(xsel, n_sel, H, wr, bias, E, K, alpha, idx, w, NULL, NULL);
  }
  layer_job J;
  memset(&J, 0, sizeof(J));
  J.H = H; J.I = I; J.E = E; J.K = K; J.limit = limit;
  J.xs = xs; J.idx = idx; J.gate = gate; J.up = up; J.down = down; J.n_sel = n_sel;
  J.y = (double*)calloc((size_t)n_sel * K * H, sizeof(double));
  J.wg = wg; J.wu = wu; J.wd = wd;
  J.ys = (double*)calloc((size_t)n_sel * H, sizeof(double));
  if (nthreads < 1) nthreads = 1;
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
  for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, layer_worker, &J);
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  free(th);
  /* combine in fixed slot order */
  for (int j = 0; j < n_sel; ++j)
    for (int h = 0; h < H; ++h) {
      double acc = 0.0;
      for (int k = 0; k < K; ++k) acc += w[(int64_t)j * K + k] * J.y[((int64_t)j * K + k) * H + h];
      out[(int64_t)j * H + h] = (wg ? J.ys[(int64_t)j * H + h] : 0.0) + acc;
    }
  if (idx_out) memcpy(idx_out, idx, sizeof(int32_t) * (int64_t)n_sel * K);
  if (w_out) memcpy(w_out, w, sizeof(double) * (int64_t)n_sel * K);
  int err = J.err;
  free(J.y); free(J.ys); free(idx); free(w); free(xs); free(xsel);
  return err;
}
