/*
 * moe.h -- C ABI of libmoe.so: the routed MoE layer of DeepSeek-V4-Flash with
 * MXFP4 experts, on one NVIDIA B200 (sm_100a).
 *
 * The layer, per token x (hidden H):
 *   s_e   = sqrt(softplus(x . Wr_e))                          (moe_route)
 *   idx   = top-k of s_e + b_e   (b selects only)              (moe_route)
 *   w_k   = scale * s_idx_k / sum_j s_idx_j                    (moe_route)
 *   pairs grouped by expert, stable                            (moe_permute)
 *   y_k   = Wd (silu(min(Wg x, L)) * clamp(Wu x, -L, L))       (moe_expert_gemm)
 *   ys    = the same FFN with the bf16 shared expert           (shared_expert)
 *   out   = ys + sum_k w_k y_k                                 (moe_combine)
 *
 * Sources (page title, section):
 *  - "DeepSeek-V4-Flash export design" (ONNX Runtime mobius), Source
 *    configuration, MoE bullet: 256 routed experts, top 6, intermediate 2048,
 *    one shared expert, scale 1.5, normalized sqrt(softplus(logit)) routing,
 *    first three layers routed by a token-id hash table; section "V3 reuse and
 *    V4 differences": clamped SwiGLU.
 *  - "Model techniques map" (DeepSeek-V4-Flash): rows "Mixture of experts",
 *    "Auxiliary-loss-free load balancing", "Shared expert", "SwiGLU
 *    feed-forward" (the router's topk / gather, routed + shared, the clamps).
 *  - "ElytronAI / DeepSeek-v4-Flash", Layout and Sizes: MXFP4 storage as an
 *    E2M1 nibble plane plus an E8M0 group-32 scale plane; experts of a
 *    projection back to back, expert xid at base + xid * expert_bytes; 32-byte
 *    aligned tensor offsets.
 *  - "DeepSeek-V4-Flash-0731-JANG", Dynamic affine recipe: router kept in f32.
 *
 * Conventions for every entry point:
 *  - Pointers named *_host are host pointers; every other pointer is a DEVICE
 *    pointer, allocated and owned by the caller.  The library allocates no
 *    device memory, never synchronises, and keeps no per-call state, so calls
 *    on different streams are independent.  Work is enqueued on `stream`
 *    (a cudaStream_t; NULL is the legacy default stream).
 *  - Argument errors are detected on the host before any launch and returned
 *    synchronously (nothing is enqueued).  A failed launch returns
 *    MOE_ERR_CUDA.  Device-side faults show up as CUDA errors of later calls.
 *  - Bounded waits: a kernel that gives up waiting on a copy sets a device
 *    error word and returns; moe_device_error() reads and clears it.
 *  - No C++ exception crosses this ABI.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 1

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, bad size, bad index range */
  MOE_ERR_ALIGNMENT = 2,   /* a pointer or byte size misses its alignment */
  MOE_ERR_UNSUPPORTED = 3, /* shape outside what the kernels implement */
  MOE_ERR_WORKSPACE = 4,   /* ws_bytes below the *_workspace_size() value */
  MOE_ERR_CUDA = 5,        /* a CUDA launch or API call failed */
  MOE_ERR_DEVICE = 6       /* a kernel reported a device-side error */
} moe_status;

/* Layer shape.  hidden H, inter I, n_experts E, top_k K; route_scale is the
 * factor applied after normalising the K selected scores (1.5 for V4-Flash);
 * swiglu_limit is the clamp L (the gate is clamped above at L, the up
 * projection to [-L, L]).  Supported: H and I multiples of 32 with H/32 and
 * I/32 powers of two up to 128; 1 <= K <= min(E, 32); E <= 1024. */
typedef struct {
  int32_t hidden, inter, n_experts, top_k;
  float route_scale, swiglu_limit;
} moe_dims;

/* One MXFP4 projection of all experts (device memory).  The blob of expert
 * xid starts at base + xid * expert_bytes and holds
 *   [rows][cols/2] bytes of E2M1 codes (low nibble = even column), then
 *   [rows][cols/32] bytes of E8M0 exponents (scale 2^(e-127) for 32
 *   consecutive columns of a row; e = 255 (NaN) is not allowed),
 * so expert_bytes == rows*cols/2 + rows*cols/32 (no padding between experts).
 * base must be 32-byte aligned.  Gate and up are [inter][hidden]; down is
 * [hidden][inter]. */
typedef struct {
  const uint8_t* base;
  int64_t expert_bytes;
  int32_t rows, cols;
} moe_mxfp4_proj;

int moe_abi_version(void);
const char* moe_status_string(moe_status status);

/* Reads and clears the device error word of the current device (host call,
 * synchronises the current device).  0 = no error; otherwise the first code
 * recorded since the last read:
 *   0x201  an expert id outside [0, E) reached moe_permute;
 *   0x301  a tensor-core kernel gave up waiting on a copy (each wait is
 *          bounded to 2 s);
 *   0x302  moe_expert_gemm's dequantising path met a weight row whose E8M0
 *          bytes span more than 36 octaves and flushed its lowest groups;
 *   0x303  moe_expert_gemm's dequantising path met an activation beyond the
 *          f16 range (|x| > 65504); that call's output is undefined;
 *   0x304  moe_expert_gemm's dequantising path produced an h (between the
 *          GEMMs, f16) whose 32 rows of a unit all fell below f16's normal
 *          range (2^-14): those outputs kept only f16-subnormal precision;
 *   0x501  debug build: a pair index (perm / inv) outside [0, T * top_k);
 *   0x502  debug build: group offsets not non-decreasing from 0;
 *   0x401  moe_selftest_wait. */
int32_t moe_device_error(void);

/* Health check of the bounded-wait path (no counterpart on the pages): a
 * kernel waits on a barrier that nothing releases, gives up after wait_us
 * microseconds (1 .. 2,000,000), records device error 0x401 and returns,
 * exactly as the pipeline kernels do when a copy never lands.  Afterwards
 * moe_device_error() returns 0x401 and the device stays usable.  Enqueued on
 * `stream`; returns MOE_ERR_INVALID_ARG for a wait outside the range. */
moe_status moe_selftest_wait(int32_t wait_us, void* stream);

/* --- routing ---------------------------------------------------------- */

/* Workspace bytes moe_route needs for T tokens (logits scratch). */
size_t moe_route_workspace_size(const moe_dims* dims, int32_t T);

/*
 * Routing of T tokens.
 *  x          bf16 [T][hidden], row-major, 16-byte aligned.
 *  router_w   fp32 [n_experts][hidden] (the router is kept in f32).
 *  bias       fp32 [n_experts] or NULL: added to the scores for selection
 *             only (aux-loss-free balancing); never enters the weights.
 *  token_ids, hash_table, vocab: hash routing when both pointers are given:
 *             topk_idx[t] = hash_table[token_ids[t]] ([vocab][top_k] int32,
 *             table order); token ids outside [0, vocab) are clamped to 0.
 *  topk_idx   int32 [T][top_k] out: learned routing emits the experts in
 *             descending s + b, ties to the lower id.
 *  topk_w     fp32 [T][top_k] out: route_scale * s_idx / sum of the K s_idx.
 *  ws         device workspace of moe_route_workspace_size() bytes.
 * T == 0 is a no-op.
 */
moe_status moe_route(const moe_dims* dims, const void* x, int32_t T, const float* router_w,
                     const float* bias, const int32_t* token_ids, const int32_t* hash_table,
                     int32_t vocab, int32_t* topk_idx, float* topk_w, void* ws,
                     size_t ws_bytes, void* stream);

/*
 * moe_route_noalloc: the same routing as moe_route, for callers that cannot
 * allocate device memory at all -- for example a serving runtime that hands
 * every byte of the device to its own pool at start-up, or embedding code
 * that must not call cudaMalloc/cudaFree on its hot path.  The pages describe
 * no such interface; this entry point has no counterpart there.
 *
 * Instead of a caller workspace it uses one scratch array that the library
 * keeps in device memory (a file-scope __device__ array of
 * MOE_ROUTE_NOALLOC_MAX_LOGITS floats, 256 KiB, present on every device that
 * loads libmoe.so until the process exits).  Limits and behaviour:
 *  - T * n_experts must not exceed MOE_ROUTE_NOALLOC_MAX_LOGITS; larger calls
 *    return MOE_ERR_UNSUPPORTED and enqueue nothing.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.  A failed lookup returns MOE_ERR_CUDA.
 *  - All calls share the one array: two calls whose kernels overlap on the
 *    GPU (different streams without ordering) race on it and may return
 *    each other's scores.  Order such calls on one stream.
 *  - The array keeps the previous call's logits; every call overwrites the
 *    T * n_experts entries it reads before reading them, so nothing has to
 *    start at zero.
 *  - The looked-up address is kept per device and driver context; a new
 *    context on a device (after cudaDeviceReset, say) is looked up again
 *    on its first call.
 * Arguments and outputs are those of moe_route (no ws / ws_bytes).
 * No device memory is allocated or freed by this call.
 */
#define MOE_ROUTE_NOALLOC_MAX_LOGITS 65536
moe_status moe_route_noalloc(const moe_dims* dims, const void* x, int32_t T, const float* router_w,
                             const float* bias, const int32_t* token_ids, const int32_t* hash_table,
                             int32_t vocab, int32_t* topk_idx, float* topk_w, void* stream);

/* --- grouping ----------------------------------------------------------- */

size_t moe_permute_workspace_size(int32_t T, int32_t K, int32_t E);

/*
 * Stable counting sort of the T*K (token, slot) pairs by expert.  Pair
 * p = t*K + k has expert topk_idx[p] (must lie in [0, E)).
 *  offsets  int32 [E+1] out: exclusive prefix sum of the per-expert counts.
 *  perm     int32 [T*K] out: perm[pos] = p, in (expert, p) order, so the
 *           pairs of expert e are perm[offsets[e] .. offsets[e+1]).
 *  inv      int32 [T*K] out: inv[p] = pos.
 * Bit-exact and deterministic.  T*K <= 1<<22.
 */
moe_status moe_permute(const int32_t* topk_idx, int32_t T, int32_t K, int32_t E, int32_t* offsets,
                       int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes, void* stream);

/* --- routed experts ------------------------------------------------------ */

size_t moe_expert_gemm_workspace_size(const moe_dims* dims, int32_t T);

/*
 * The path moe_expert_gemm takes for T tokens (host only, no GPU work):
 * 1 = block-scaled tensor-core MMAs, 0 = dequantising to f16 (see below);
 * -MOE_ERR_INVALID_ARG for a null dims, invalid dims or T < 0.
 */
int32_t moe_expert_gemm_path(const moe_dims* dims, int32_t T);

/*
 * All routed experts for the grouped pairs:
 *   y_perm[pos] = Wd_e (silu(min(Wg_e x_t, L)) * clamp(Wu_e x_t, -L, L))
 * for pos in [offsets[e], offsets[e+1]), p = perm[pos], t = p / top_k.
 *  x        bf16 [T][hidden], 16-byte aligned.
 *  gate, up MXFP4 [inter][hidden]; down MXFP4 [hidden][inter] (see
 *           moe_mxfp4_proj).
 *  offsets, perm  as written by moe_permute.
 *  y_perm   fp32 [T*top_k][hidden] out.
 *  ws       device workspace of moe_expert_gemm_workspace_size(dims, T)
 *           bytes: the block-scaled path's layout below, of which the
 *           dequantising path uses a prefix, so the size grows with T and a
 *           workspace sized for some T serves every smaller T.
 * Two paths, chosen from T alone (mean pairs per expert, ceil(T*top_k / E)):
 *  - at most 24 (decode, small batches): block-scaled tensor-core MMAs
 *    (tcgen05 kind::mxf8f6f4): the E2M1 codes and E8M0 scales go to the
 *    tensor core as stored and are applied there.  Each activation enters as
 *    two E4M3 terms with E8M0 group-32 scales (a bf16 x is carried exactly
 *    unless a residual falls below the E4M3 range of its 32-value group), h
 *    between the GEMMs as three terms (about 12 significant bits); sums fp32.
 *    Workspace: E4M3 terms and E8M0 scales of x in expert order
 *    [2][T*top_k][hidden] and [2][T*top_k][hidden/32], then of h
 *    [3][T*top_k][inter] and [3][T*top_k][inter/32] bytes.
 *  - above 24 (prefill): each weight is dequantised to f16 times a power of
 *    two per weight row (undone in fp32): exactly for every E8M0 group within
 *    36 octaves of the largest group of its row, whatever the bytes; groups
 *    further below are flushed to zero (their products lie below 2^-36 of
 *    the row's largest group's) and the call records device error 0x302.
 *    x goes in as f16: exact for |x| in [2^-17, 65504], f16 subnormal
 *    precision below (absolute error at most 2^-25); a value beyond 65504
 *    is not representable and the call records device error 0x303 (its
 *    output is undefined).  h between the GEMMs is f16 (11 significant bits
 *    down to 2^-14, subnormal below; a unit whose h all lies below 2^-14
 *    records device error 0x304); f16 x f16 MMAs with fp32 sums.
 *    Workspace: x in expert order as f16 [T*top_k][hidden], then h in f16
 *    [T*top_k][inter].
 * Shapes: inter a multiple of 128, hidden a multiple of 256 (the row tiles of
 * the two GEMMs), besides the moe_dims limits; other shapes return
 * MOE_ERR_UNSUPPORTED before anything is enqueued.
 * Either path is one grouped tcgen05 GEMM pair plus the activation gather; the
 * number of units follows the device-side counts, the launches do not depend
 * on them.  A kernel that gives up a bounded wait records device error 0x301.
 */
moe_status moe_expert_gemm(const moe_dims* dims, const void* x, int32_t T, moe_mxfp4_proj gate,
                           moe_mxfp4_proj up, moe_mxfp4_proj down, const int32_t* offsets,
                           const int32_t* perm, float* y_perm, void* ws, size_t ws_bytes,
                           void* stream);

/* --- shared expert -------------------------------------------------------- */

size_t shared_expert_workspace_size(const moe_dims* dims, int32_t T);

/*
 * The bf16 shared expert on every token:
 *   out[t] = wd (silu(min(wg x_t, L)) * clamp(wu x_t, -L, L)), fp32 [T][hidden].
 *  wg, wu bf16 [inter][hidden]; wd bf16 [hidden][inter]; all 16-byte aligned.
 *  ws     device workspace of shared_expert_workspace_size() bytes.
 */
moe_status shared_expert(const moe_dims* dims, const void* x, int32_t T, const void* wg,
                         const void* wu, const void* wd, float* out, void* ws, size_t ws_bytes,
                         void* stream);

/* --- combine ---------------------------------------------------------------- */

/*
 * out_f32[t] = shared_out[t] + sum_{k=0..K-1} topk_w[t][k] * y_perm[inv[t*K+k]]
 * summed in that fixed slot order (deterministic).  shared_out may be NULL
 * (treated as 0).  out_bf16 (nullable) receives the same values rounded to
 * bf16 (round to nearest even).
 */
moe_status moe_combine(const moe_dims* dims, int32_t T, const float* y_perm, const int32_t* inv,
                       const float* topk_w, const float* shared_out, float* out_f32,
                       void* out_bf16, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
