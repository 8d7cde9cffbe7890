// libmoe.so: the C ABI declared in include/moe.h.  One translation unit: the
// kernels live in the headers included below.
#include <atomic>
#include <cstdio>
#include <mutex>

#include "combine.cuh"
#include "common.cuh"
#include "permute.cuh"
#include "route.cuh"
#include "expert_launch.h"
#include "mx_expert.cuh"
#include "tc_expert.cuh"
#include "shared_decode.cuh"

using namespace moe;

namespace {

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline bool pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Raises a kernel's dynamic shared-memory limit on the current device, once
// per device (the attribute belongs to each device's context); `done` holds
// one bit per device id.
template <class Kernel>
bool smem_limit_once(std::atomic<uint64_t>& done, Kernel* kernel, int bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  const uint64_t bit = 1ull << dev;
  if (done.load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  done.fetch_or(bit, std::memory_order_release);
  return true;
}

moe_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    fprintf(stderr, "libmoe: launch failed: %s\n", cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// Programmatic stream serialization: with it, each kernel may begin (its
// prologue: barriers, TMEM, descriptor fetches) while its predecessor in the
// stream finishes, and waits in griddep_wait() before its first global
// access, so stream order holds for every byte.  Measured on one B200 (decode
// layer passes, interleaved A/B in CUDA graphs): no gain in the expert call
// and ~1.5% slower whole layers, so it is off; the kernels keep their waits
// (no-ops without the attribute).
constexpr bool kUsePdl = false;

template <typename... KArgs, typename... Args>
moe_status launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                    const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kUsePdl ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess) {
    fprintf(stderr, "libmoe: launch failed: %s\n", cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Row-major 16-bit [rows][cols] viewed by TMA with a {64, box_rows} box (one
// k-block of a unit's n_chunk token rows) and 128-byte swizzle (the
// token-operand layout of the tensor-core expert kernel).
bool make_row_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows,
                  CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, type, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D view of a weight array for the expert kernel's loader: {row bytes of
// the E2M1 plane, rows, experts} for MXFP4 (box {min(128, cols/2), 128, 1},
// swizzle matching the box's inner extent), {columns, rows, 1} for a bf16
// matrix (box {64, 128, 1}, 128-byte swizzle).
bool make_weight_map(CUtensorMap* map, const uint8_t* base, int af, const TcArgs& a) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr || base == nullptr) return false;
  cuuint64_t dims[3], strides[2];
  cuuint32_t box[3], estr[3] = {1, 1, 1};
  CUtensorMapDataType type;
  CUtensorMapSwizzle swizzle;
  if (af == kAMxfp4) {
    dims[0] = (cuuint64_t)a.a_cols / 2;
    dims[1] = (cuuint64_t)a.rows;
    dims[2] = (cuuint64_t)(a.offsets != nullptr ? a.E : 1);
    strides[0] = (cuuint64_t)a.a_cols / 2;
    strides[1] = (cuuint64_t)a.expert_bytes;
    box[0] = (cuuint32_t)a.w_inner;
    type = CU_TENSOR_MAP_DATA_TYPE_UINT8;
    swizzle = a.w_inner == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
              : a.w_inner == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                : CU_TENSOR_MAP_SWIZZLE_32B;
  } else {
    dims[0] = (cuuint64_t)a.a_cols;
    dims[1] = (cuuint64_t)a.rows;
    dims[2] = 1;
    strides[0] = (cuuint64_t)a.a_cols * 2;
    strides[1] = (cuuint64_t)a.a_cols * 2 * a.rows;
    box[0] = 64;
    type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    swizzle = CU_TENSOR_MAP_SWIZZLE_128B;
  }
  box[1] = 128;
  box[2] = 1;
  // a 64-byte box reads half of a row's 128-byte line; the next stage's box
  // reads the other half, so L2 fills go by 128 bytes, not 256
  const CUtensorMapL2promotion promo =
      box[0] * (type == CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 ? 2 : 1) >= 128 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B
                                                                         : CU_TENSOR_MAP_L2_PROMOTION_L2_128B;
  return fn(map, type, 3, const_cast<uint8_t*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Plans the pipeline of one tensor-core expert launch, builds its weight
// tensor maps and launches it (one CTA per SM); EPI epilogue warps.
template <int MODE, int AF, int EPI>
moe_status launch_tc_epi(const CUtensorMap& bmap, TcArgs a, cudaStream_t s) {
  static std::atomic<uint64_t> configured{0};
  if (!smem_limit_once(configured, tc_expert_kernel<MODE, AF, EPI>, kTcSmemMax)) return MOE_ERR_CUDA;
  if (!tc_plan(a, AF)) return MOE_ERR_UNSUPPORTED;
  CUtensorMap w0, w1;
  if (!make_weight_map(&w0, a.w0, AF, a)) return MOE_ERR_CUDA;
  if (MODE == 0) {
    if (!make_weight_map(&w1, a.w1, AF, a)) return MOE_ERR_CUDA;
  } else {
    w1 = w0;
  }
  return launch_k(tc_expert_kernel<MODE, AF, EPI>, dim3(sm_count()), dim3(tc_threads(EPI)), a.smem_bytes, s, bmap, w0,
                  w1, a);
}

// 128-token chunks get 8 epilogue warps, smaller ones 4.
template <int MODE, int AF>
moe_status launch_tc(const CUtensorMap& bmap, const TcArgs& a, cudaStream_t s) {
  return a.n_chunk > 64 ? launch_tc_epi<MODE, AF, 8>(bmap, a, s) : launch_tc_epi<MODE, AF, 4>(bmap, a, s);
}

// E2M1 plane of an MXFP4 weight array viewed by the block-scaled expert
// kernel's loader as {codes of a K-tile (128), rows, K-tiles, experts}: boxes of
// 128 codes x box_rows rows (128: one tile; 256: both tiles of a down unit) x
// kps K-tiles, widened to the f8f6f4 shared-memory layout (16U4_ALIGN16B),
// 128-byte swizzle; in shared memory [K-tile][row][128 B].
bool make_mx_weight_map(CUtensorMap* map, const uint8_t* base, const MxArgs& a, int box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr || base == nullptr) return false;
  cuuint64_t dims[4] = {(cuuint64_t)kMxKT, (cuuint64_t)a.rows, (cuuint64_t)(a.cols / kMxKT), (cuuint64_t)a.E};
  cuuint64_t strides[3] = {(cuuint64_t)a.cols / 2, (cuuint64_t)kMxKT / 2, (cuuint64_t)a.expert_bytes};
  cuuint32_t box[4] = {(cuuint32_t)kMxKT, (cuuint32_t)box_rows, (cuuint32_t)a.kps, 1}, estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 4, const_cast<uint8_t*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// E4M3 token terms [parts][pairs][cols] bytes viewed as {bytes of a K-tile
// (128), pairs, parts, K-tiles} with one {128, n_chunk, parts, kps} box per
// stage (every term's rows of a unit for the stage's K-tiles in one copy),
// 128-byte swizzle; in shared memory [K-tile][term][row][128 B].
bool make_term_map(CUtensorMap* map, const uint8_t* base, int64_t pairs, int parts, int64_t cols, int n_chunk,
                   int kps) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return false;
  cuuint64_t dims[4] = {(cuuint64_t)kMxKT, (cuuint64_t)pairs, (cuuint64_t)parts, (cuuint64_t)(cols / kMxKT)};
  cuuint64_t strides[3] = {(cuuint64_t)cols, (cuuint64_t)(cols * pairs), (cuuint64_t)kMxKT};
  cuuint32_t box[4] = {(cuuint32_t)kMxKT, (cuuint32_t)n_chunk, (cuuint32_t)parts, (cuuint32_t)kps};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<uint8_t*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// E8M0 plane of an MXFP4 weight array: {row bytes (cols / 32), rows, experts}
// with boxes of one scale stage's bytes (4 G) of box_rows rows, no swizzle.
bool make_mx_scale_map(CUtensorMap* map, const uint8_t* base, const MxArgs& a, int box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr || base == nullptr) return false;
  const int64_t plane = (int64_t)a.rows * (a.cols / 2);
  cuuint64_t dims[3] = {(cuuint64_t)a.cols / 32, (cuuint64_t)a.rows, (cuuint64_t)a.E};
  cuuint64_t strides[2] = {(cuuint64_t)a.cols / 32, (cuuint64_t)a.expert_bytes};
  cuuint32_t box[3] = {(cuuint32_t)(4 * a.g), (cuuint32_t)box_rows, 1}, estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(base + plane), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// E8M0 scales of the token terms [parts][pairs][cols / 32] viewed as
// {cols / 32, pairs, parts} with one {4 G, n_chunk, parts} box per scale
// stage, no swizzle.
bool make_token_scale_map(CUtensorMap* map, const MxArgs& a) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr || a.b_scale == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)a.cols / 32, (cuuint64_t)a.pairs, (cuuint64_t)a.parts};
  cuuint64_t strides[2] = {(cuuint64_t)a.cols / 32, (cuuint64_t)(a.cols / 32) * a.pairs};
  cuuint32_t box[3] = {(cuuint32_t)(4 * a.g), (cuuint32_t)a.n_chunk, (cuuint32_t)a.parts}, estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(a.b_scale), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// One block-scaled expert launch (planned by mx_plan), one CTA per SM.
template <int MODE, int G, int KPS, bool SUMMED>
moe_status launch_mx_g(const CUtensorMap& bmap, const MxArgs& a, cudaStream_t s) {
  static std::atomic<uint64_t> configured{0};
  if (!smem_limit_once(configured, mx_expert_kernel<MODE, G, KPS, SUMMED>, kTcSmemMax)) return MOE_ERR_CUDA;
  CUtensorMap w0, w1, s0, s1, ts;
  const int box_rows = MODE == 0 ? 128 : 256;  // MODE 1: both 128-row tiles of a unit in one box
  if (!make_mx_weight_map(&w0, a.w0, a, box_rows)) return MOE_ERR_CUDA;
  if (MODE == 0) {
    if (!make_mx_weight_map(&w1, a.w1, a, box_rows)) return MOE_ERR_CUDA;
  } else {
    w1 = w0;
  }
  if (a.tma_scales) {
    if (!make_mx_scale_map(&s0, a.w0, a, box_rows) || !make_token_scale_map(&ts, a)) return MOE_ERR_CUDA;
    if (MODE == 0) {
      if (!make_mx_scale_map(&s1, a.w1, a, box_rows)) return MOE_ERR_CUDA;
    } else {
      s1 = s0;
    }
  } else {  // unused: the scale writers load the E8M0 rows themselves
    s0 = s1 = ts = w0;
  }
  return launch_k(mx_expert_kernel<MODE, G, KPS, SUMMED>, dim3(sm_count()), dim3(kMxThreads), a.smem_bytes, s, bmap, w0, w1, s0,
                  s1, ts, a);
}

template <int MODE>
moe_status launch_mx(const CUtensorMap& bmap, const MxArgs& a, cudaStream_t s) {
  // the plan gives two-K-tile stages only with an even G
  const bool k2 = a.kps == 2, sum = a.term_acc != 0;
  switch (a.g) {
    case 8:
      return k2 ? (sum ? launch_mx_g<MODE, 8, 2, true>(bmap, a, s) : launch_mx_g<MODE, 8, 2, false>(bmap, a, s))
                : (sum ? launch_mx_g<MODE, 8, 1, true>(bmap, a, s) : launch_mx_g<MODE, 8, 1, false>(bmap, a, s));
    case 4:
      return k2 ? (sum ? launch_mx_g<MODE, 4, 2, true>(bmap, a, s) : launch_mx_g<MODE, 4, 2, false>(bmap, a, s))
                : (sum ? launch_mx_g<MODE, 4, 1, true>(bmap, a, s) : launch_mx_g<MODE, 4, 1, false>(bmap, a, s));
    case 2:
      return k2 ? (sum ? launch_mx_g<MODE, 2, 2, true>(bmap, a, s) : launch_mx_g<MODE, 2, 2, false>(bmap, a, s))
                : (sum ? launch_mx_g<MODE, 2, 1, true>(bmap, a, s) : launch_mx_g<MODE, 2, 1, false>(bmap, a, s));
    default:
      return sum ? launch_mx_g<MODE, 1, 1, true>(bmap, a, s) : launch_mx_g<MODE, 1, 1, false>(bmap, a, s);
  }
}

// Router and shared expert run on the tensor cores above this token count
// (and when their shapes fit the kernel's tiles).
constexpr int kTcMinT = 65;

bool tc_router_ok(const moe_dims* d, int T) { return T >= kTcMinT && d->n_experts % 256 == 0 && d->hidden % 64 == 0; }
bool tc_shared_ok(const moe_dims* d, int T) {
  return T >= kTcMinT && d->inter % 128 == 0 && d->hidden % 256 == 0 && d->hidden % 64 == 0 && d->inter % 64 == 0;
}

}  // namespace

namespace {

moe_status check_dims(const moe_dims* d) {
  if (d == nullptr) return MOE_ERR_INVALID_ARG;
  if (d->hidden <= 0 || d->inter <= 0 || d->n_experts <= 0 || d->top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (d->hidden % 32 || d->inter % 32) return MOE_ERR_UNSUPPORTED;
  if (!pow2(d->hidden / 32) || !pow2(d->inter / 32) || d->hidden / 32 > 128 || d->inter / 32 > 128)
    return MOE_ERR_UNSUPPORTED;
  if (d->n_experts > 1024 || d->top_k > 32 || d->top_k > d->n_experts) return MOE_ERR_UNSUPPORTED;
  if (!(d->swiglu_limit > 0.f) || !(d->swiglu_limit <= 32.f)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status check_proj(const moe_mxfp4_proj& p, int rows, int cols) {
  if (p.base == nullptr) return MOE_ERR_INVALID_ARG;
  if (p.rows != rows || p.cols != cols) return MOE_ERR_INVALID_ARG;
  if (p.expert_bytes != (int64_t)rows * cols / 2 + (int64_t)rows * cols / 32) return MOE_ERR_INVALID_ARG;
  if (!aligned(p.base, 32) || p.expert_bytes % 16) return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}

}  // namespace

// ---- routing without a caller workspace -------------------------------------
// Scratch for moe_route_noalloc: the logits of one call, T * n_experts floats.
// Lives in device memory on every device that loads the library.
static __device__ __align__(256) float g_route_noalloc_logits[MOE_ROUTE_NOALLOC_MAX_LOGITS];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
// Per device: the scratch array's device address and the context it was
// looked up in.  A device reset (cudaDeviceReset) tears the context down and
// the module is loaded again, possibly elsewhere; a new context on the same
// device is the sign that the address has to be looked up again.
struct NoallocSlot {
  const void* ctx;
  float* ptr;
};
NoallocSlot g_noalloc[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The current thread's driver context (through the runtime's entry point
// table, so the library needs no libcuda link); null if unavailable.
void* current_context() {
  static CtxGetCurrentFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
  CUcontext c = nullptr;
  return fn(&c) == CUDA_SUCCESS ? static_cast<void*>(c) : nullptr;
}

// Device address of the scratch array on the current device, looked up with
// that device current the first time it is needed in a context (the host-side
// symbol is not a device address).
cudaError_t noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const void* ctx = current_context();  // null before the runtime has made one current
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  NoallocSlot& slot = g_noalloc[dev];
  if (slot.ptr == nullptr || ctx == nullptr || slot.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_noalloc_logits);  // makes the device's context current
    if (e != cudaSuccess) return e;
    slot.ptr = static_cast<float*>(p);
    slot.ctx = current_context();
  }
  *out = slot.ptr;
  return cudaSuccess;
}
}  // namespace

extern "C" {

int moe_abi_version(void) { return MOE_ABI_VERSION; }

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_ALIGNMENT: return "misaligned pointer or size";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE: return "device-side error";
  }
  return "unknown status";
}

int32_t moe_device_error(void) {
  int32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_error, sizeof(v)) != cudaSuccess) return -1;
  if (cudaMemcpyToSymbol(g_error, &zero, sizeof(zero)) != cudaSuccess) return -1;
  return v;
}

moe_status moe_selftest_wait(int32_t wait_us, void* stream) {
  if (wait_us <= 0 || wait_us > 2000000) return MOE_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((uint64_t)wait_us * 1000u);
  return launch_status();
}

size_t moe_route_workspace_size(const moe_dims* dims, int32_t T) {
  if (dims == nullptr || T < 0) return 0;
  size_t b = round_up((size_t)T * dims->n_experts * sizeof(float), 256);
  // tensor-core router: the router weight split into bf16 hi | mid | lo
  if (tc_router_ok(dims, T)) b += round_up((size_t)dims->n_experts * 3 * dims->hidden * 2, 256);
  return b;
}

moe_status moe_route(const moe_dims* dims, const void* x, int32_t T, const float* router_w,
                     const float* bias, const int32_t* token_ids, const int32_t* hash_table,
                     int32_t vocab, int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                     void* stream) {
  moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !router_w || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  const bool hashed = token_ids != nullptr || hash_table != nullptr;
  if (hashed && (!token_ids || !hash_table || vocab <= 0)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(router_w, 16)) return MOE_ERR_ALIGNMENT;
  if (ws_bytes < moe_route_workspace_size(dims, T) || ws == nullptr) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int E = dims->n_experts, H = dims->hidden;
  float* logits = static_cast<float*>(ws);
  if (tc_router_ok(dims, T)) {
    // logits = x . (hi + mid + lo) on the tensor cores: every product exact, fp32 sums
    __nv_bfloat16* split = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(ws) +
                                                            round_up((size_t)T * E * sizeof(float), 256));
    if ((st = launch_k(split3_bf16_kernel, dim3(2 * sm_count()), dim3(256), 0, s, router_w, split, E, H)) != MOE_OK)
      return st;
    CUtensorMap xmap;
    if (!make_row_map(&xmap, x, T, H, 32)) return MOE_ERR_CUDA;
    TcArgs a{};
    a.w0 = reinterpret_cast<const uint8_t*>(split);
    a.rows = E;
    a.a_cols = 3 * H;
    a.k_total = 3 * H;
    a.b_cols = H;
    a.n_single = T;
    a.n_chunk = 32;
    a.out = logits;
    if ((st = launch_tc<1, kABf16>(xmap, a, s)) != MOE_OK) return st;
  } else {
    dim3 g1((E + kLogitExperts - 1) / kLogitExperts, (T + kLogitTokBlock - 1) / kLogitTokBlock);
    if ((st = launch_k(route_logits_kernel, g1, dim3(kLogitThreads), kLogitExperts * H * sizeof(float), s,
                       static_cast<const __nv_bfloat16*>(x), T, H, router_w, E, logits)) != MOE_OK)
      return st;
  }
  return launch_k(route_select_kernel, dim3((T + 3) / 4), dim3(128), 4 * E * sizeof(float), s,
                  static_cast<const float*>(logits), T, E, dims->top_k, dims->route_scale,
                  hashed ? nullptr : bias, token_ids, hash_table, vocab, topk_idx, topk_w);
}

moe_status moe_route_noalloc(const moe_dims* dims, const void* x, int32_t T, const float* router_w,
                             const float* bias, const int32_t* token_ids, const int32_t* hash_table,
                             int32_t vocab, int32_t* topk_idx, float* topk_w, void* stream) {
  moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !router_w || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if ((int64_t)T * dims->n_experts > MOE_ROUTE_NOALLOC_MAX_LOGITS) return MOE_ERR_UNSUPPORTED;
  const bool hashed = token_ids != nullptr || hash_table != nullptr;
  if (hashed && (!token_ids || !hash_table || vocab <= 0)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(router_w, 16)) return MOE_ERR_ALIGNMENT;
  float* logits = nullptr;
  if (noalloc_scratch(&logits) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int E = dims->n_experts, H = dims->hidden;
  dim3 g1((E + kLogitExperts - 1) / kLogitExperts, (T + kLogitTokBlock - 1) / kLogitTokBlock);
  route_logits_kernel<<<g1, kLogitThreads, kLogitExperts * H * sizeof(float), s>>>(
      static_cast<const __nv_bfloat16*>(x), T, H, router_w, E, logits);
  if ((st = launch_status()) != MOE_OK) return st;
  route_select_kernel<<<(T + 3) / 4, 128, 4 * E * sizeof(float), s>>>(
      logits, T, E, dims->top_k, dims->route_scale, hashed ? nullptr : bias, token_ids, hash_table, vocab,
      topk_idx, topk_w);
  return launch_status();
}

size_t moe_permute_workspace_size(int32_t T, int32_t K, int32_t E) {
  (void)T; (void)K; (void)E;
  return 0;
}

moe_status moe_permute(const int32_t* topk_idx, int32_t T, int32_t K, int32_t E, int32_t* offsets,
                       int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes, void* stream) {
  (void)ws; (void)ws_bytes;
  if (T < 0 || K <= 0 || E <= 0 || E > 1024 || K > 32) return MOE_ERR_INVALID_ARG;
  if ((int64_t)T * K > (1 << 22)) return MOE_ERR_UNSUPPORTED;
  if (!offsets || (T > 0 && (!topk_idx || !perm || !inv))) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int smem = 32 * E * (int)sizeof(int32_t);
  static std::atomic<uint64_t> configured{0};
  if (!smem_limit_once(configured, permute_kernel, 32 * 1024 * 4)) return MOE_ERR_CUDA;
  return launch_k(permute_kernel, dim3(1), dim3(kPermuteThreads), smem, s, topk_idx, T * K, E, offsets, perm, inv);
}

size_t moe_expert_gemm_workspace_size(const moe_dims* dims, int32_t T) {
  if (dims == nullptr || T < 0) return 0;
  return expert_gemm_ws_bytes(*dims, T);
}

int32_t moe_expert_gemm_path(const moe_dims* dims, int32_t T) {
  if (check_dims(dims) != MOE_OK || T < 0) return -(int32_t)MOE_ERR_INVALID_ARG;
  return use_block_scaled(T, dims->top_k, dims->n_experts) ? 1 : 0;
}

namespace {

moe_status expert_gemm_block_scaled(const moe_dims* dims, const void* x, int32_t T, const moe_mxfp4_proj& gate,
                                    const moe_mxfp4_proj& up, const moe_mxfp4_proj& down, const int32_t* offsets,
                                    const int32_t* perm, float* y_perm, void* ws, cudaStream_t s) {
  MxLaunch L;
  // shape check before anything is enqueued
  if (!mx_launch_args(*dims, T, gate, up, down, offsets, y_perm, ws, L)) return MOE_ERR_UNSUPPORTED;
  const int H = dims->hidden, I = dims->inter;
  // the activations of every pair, in expert order, as E4M3 terms
  const int64_t n8 = L.pairs * H / 8;
  moe_status st = launch_k(gather_split_kernel, dim3((int)((n8 + 255) / 256 < 4 * 1184 ? (n8 + 255) / 256 : 4 * 1184)),
                           dim3(256), 0, s, static_cast<const uint4*>(x), perm, dims->top_k, H, L.pairs, kXTerms,
                           L.xq, L.xs);
  if (st != MOE_OK) return st;
  CUtensorMap xmap, hmap;
  if (!make_term_map(&xmap, L.xq, L.pairs, kXTerms, H, L.g.n_chunk, L.g.kps) ||
      !make_term_map(&hmap, L.hq, L.pairs, kHTerms, I, L.d.n_chunk, L.d.kps))
    return MOE_ERR_CUDA;
  if ((st = launch_mx<0>(xmap, L.g, s)) != MOE_OK) return st;
  return launch_mx<1>(hmap, L.d, s);
}

moe_status expert_gemm_dequant(const moe_dims* dims, const void* x, int32_t T, const moe_mxfp4_proj& gate,
                               const moe_mxfp4_proj& up, const moe_mxfp4_proj& down, const int32_t* offsets,
                               const int32_t* perm, float* y_perm, void* ws, cudaStream_t s) {
  TcLaunch L;
  // shape check before anything is enqueued
  if (!tc_launch_args(*dims, T, gate, up, down, offsets, y_perm, ws, L)) return MOE_ERR_UNSUPPORTED;
  const int H = dims->hidden, I = dims->inter;
  // the activations of every pair, in expert order and f16 (the token operand
  // of the gate/up GEMM is then read with plain TMA boxes)
  const int64_t n8 = L.pairs * H / 8;
  moe_status st = launch_k(gather_f16_kernel, dim3((int)((n8 + 255) / 256 < 4 * 1184 ? (n8 + 255) / 256 : 4 * 1184)),
                           dim3(256), 0, s, static_cast<const uint4*>(x), perm, dims->top_k, H / 8, L.pairs,
                           reinterpret_cast<uint4*>(L.x16));
  if (st != MOE_OK) return st;
  CUtensorMap xmap, hmap;
  if (!make_row_map(&xmap, L.x16, L.pairs, H, L.g.n_chunk, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
      !make_row_map(&hmap, L.h16, L.pairs, I, L.d.n_chunk, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
    return MOE_ERR_CUDA;
  if ((st = launch_tc<0, kAMxfp4>(xmap, L.g, s)) != MOE_OK) return st;
  return launch_tc<1, kAMxfp4>(hmap, L.d, s);
}

}  // namespace

moe_status moe_expert_gemm(const moe_dims* dims, const void* x, int32_t T, moe_mxfp4_proj gate,
                           moe_mxfp4_proj up, moe_mxfp4_proj down, const int32_t* offsets,
                           const int32_t* perm, float* y_perm, void* ws, size_t ws_bytes,
                           void* stream) {
  moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !offsets || !perm || !y_perm) return MOE_ERR_INVALID_ARG;
  const int H = dims->hidden, I = dims->inter;
  if ((st = check_proj(gate, I, H)) != MOE_OK) return st;
  if ((st = check_proj(up, I, H)) != MOE_OK) return st;
  if ((st = check_proj(down, H, I)) != MOE_OK) return st;
  if (!aligned(x, 16) || !aligned(y_perm, 16)) return MOE_ERR_ALIGNMENT;
  if (ws == nullptr || ws_bytes < moe_expert_gemm_workspace_size(dims, T)) return MOE_ERR_WORKSPACE;
  if (I % 128 || H % 256) return MOE_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return use_block_scaled(T, dims->top_k, dims->n_experts)
             ? expert_gemm_block_scaled(dims, x, T, gate, up, down, offsets, perm, y_perm, ws, s)
             : expert_gemm_dequant(dims, x, T, gate, up, down, offsets, perm, y_perm, ws, s);
}

size_t shared_expert_workspace_size(const moe_dims* dims, int32_t T) {
  if (dims == nullptr || T < 0) return 0;
  return round_up((size_t)T * dims->inter * sizeof(float), 256);
}

moe_status shared_expert(const moe_dims* dims, const void* x, int32_t T, const void* wg,
                         const void* wu, const void* wd, float* out, void* ws, size_t ws_bytes,
                         void* stream) {
  moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !wg || !wu || !wd || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(wg, 16) || !aligned(wu, 16) || !aligned(wd, 16) || !aligned(out, 16))
    return MOE_ERR_ALIGNMENT;
  if (ws == nullptr || ws_bytes < shared_expert_workspace_size(dims, T)) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int H = dims->hidden, I = dims->inter;
  if (tc_shared_ok(dims, T)) {
    // h as an exact-to-16-bits bf16 pair [T][2I] (hi | lo): the down GEMM runs
    // over K = 2I with the bf16 down weights repeated, so no operand is rounded
    // below 16 significant bits
    __nv_bfloat16* h2 = static_cast<__nv_bfloat16*>(ws);
    CUtensorMap xmap, hmap;
    if (!make_row_map(&xmap, x, T, H, kTcNMax) || !make_row_map(&hmap, h2, T, 2 * I, kTcNMax)) return MOE_ERR_CUDA;
    TcArgs g{};
    g.w0 = static_cast<const uint8_t*>(wg);
    g.w1 = static_cast<const uint8_t*>(wu);
    g.rows = I;
    g.a_cols = H;
    g.k_total = H;
    g.b_cols = H;
    g.n_single = T;
    g.n_chunk = kTcNMax;
    g.out = h2;
    g.limit = dims->swiglu_limit;
    if ((st = launch_tc<0, kABf16>(xmap, g, s)) != MOE_OK) return st;
    TcArgs d = g;
    d.w0 = static_cast<const uint8_t*>(wd);
    d.w1 = nullptr;
    d.rows = H;
    d.a_cols = I;
    d.k_total = 2 * I;
    d.b_cols = 2 * I;
    d.out = out;
    return launch_tc<1, kABf16>(hmap, d, s);
  }
  if (H % 256 || I % 32 || 2 * I % 256 || T > 8 * kShMaxNt) return MOE_ERR_UNSUPPORTED;
  __nv_bfloat16* h2 = static_cast<__nv_bfloat16*>(ws);
  ShArgs g{};
  g.w0 = static_cast<const __nv_bfloat16*>(wg);
  g.w1 = static_cast<const __nv_bfloat16*>(wu);
  g.rows = I;
  g.a_cols = H;
  g.k_total = H;
  g.xin = static_cast<const __nv_bfloat16*>(x);
  g.T = T;
  g.out = h2;
  g.limit = dims->swiglu_limit;
  if ((st = launch_k(shared_decode_kernel<0>, dim3(I / 8), dim3(kShThreads), 0, s, g)) != MOE_OK) return st;
  ShArgs d = g;
  d.w0 = static_cast<const __nv_bfloat16*>(wd);
  d.w1 = nullptr;
  d.rows = H;
  d.a_cols = I;
  d.k_total = 2 * I;
  d.xin = h2;
  d.out = out;
  return launch_k(shared_decode_kernel<1>, dim3(H / 16), dim3(kShThreads), 0, s, d);
}

moe_status moe_combine(const moe_dims* dims, int32_t T, const float* y_perm, const int32_t* inv,
                       const float* topk_w, const float* shared_out, float* out_f32, void* out_bf16,
                       void* stream) {
  moe_status st = check_dims(dims);
  if (st != MOE_OK) return st;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!y_perm || !inv || !topk_w || !out_f32) return MOE_ERR_INVALID_ARG;
  if (!aligned(y_perm, 16) || !aligned(out_f32, 16) || (shared_out && !aligned(shared_out, 16)) ||
      (out_bf16 && !aligned(out_bf16, 8)))
    return MOE_ERR_ALIGNMENT;
  const int H = dims->hidden;
  dim3 grid((H / 4 + kCombineThreads - 1) / kCombineThreads, T);
  return launch_k(combine_kernel, grid, dim3(kCombineThreads), 0, static_cast<cudaStream_t>(stream), y_perm, inv,
                  topk_w, shared_out, out_f32, static_cast<__nv_bfloat16*>(out_bf16), dims->top_k, H);
}

}  // extern "C"
