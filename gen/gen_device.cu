// Device-side fill of synthetic MXFP4 expert blobs (test-input generator).
//
// The same counter-based SplitMix64 stream as gen/__init__.py: output number i
// of stream `key` is mix64(key + (i + 1) * GOLDEN).  Byte j of a projection's
// concatenated nibble planes is byte (j % 8) (little-endian) of output j / 8 of
// the codes stream; scale byte j of the concatenated scale planes is
// lo + (((output j of the scales stream) >> 32) * (hi - lo + 1)) >> 32.
// Blob of expert x: [rows*cols/2 nibble bytes][rows*cols/32 scale bytes] at
// base + x * expert_bytes.  Integer-only, so bit-identical to the host side.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void fill_codes(uint8_t* base, int64_t n_experts, int64_t nib_words,
                           int64_t expert_bytes, uint64_t key) {
  const int64_t total = n_experts * nib_words;
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < total;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int64_t x = w / nib_words, i = w % nib_words;
    const uint64_t r = mix64(key + (uint64_t)(w + 1) * kGolden);
    // expert_bytes and the nibble plane are multiples of 8 and the base is
    // 32-byte aligned, so this 8-byte store is aligned.
    *reinterpret_cast<uint64_t*>(base + x * expert_bytes + i * 8) = r;
  }
}

__device__ __forceinline__ uint32_t below(uint64_t r, uint32_t n) { return (uint32_t)(((r >> 32) * n) >> 32); }

// row_span < 0: byte = lo + below(draw, span).  row_span >= 0: byte = base of
// the weight row (lo + below(row draw, span - row_span), row draw = output
// x * rows + r of the row stream) + below(draw, row_span + 1).
__global__ void fill_scales(uint8_t* base, int64_t n_experts, int64_t rows, int64_t per_row, int64_t nib_bytes,
                            int64_t sc_bytes, int64_t expert_bytes, uint64_t key, uint64_t key_rows,
                            uint32_t lo, uint32_t span, int row_span) {
  const int64_t total = n_experts * sc_bytes;
  for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < total;
       j += (int64_t)gridDim.x * blockDim.x) {
    const int64_t x = j / sc_bytes, i = j % sc_bytes;
    const uint64_t r = mix64(key + (uint64_t)(j + 1) * kGolden);
    uint32_t v;
    if (row_span < 0) {
      v = lo + below(r, span);
    } else {
      const uint64_t grow = (uint64_t)(x * rows + i / per_row);
      const uint64_t rb = mix64(key_rows + (grow + 1) * kGolden);
      v = lo + below(rb, span - (uint32_t)row_span) + below(r, (uint32_t)row_span + 1);
    }
    base[x * expert_bytes + nib_bytes + i] = (uint8_t)v;
  }
}

}  // namespace

extern "C" int moegen_fill_mxfp4(uint8_t* base, int64_t n_experts, int64_t rows, int64_t cols,
                                 uint64_t key_codes, uint64_t key_scales, uint64_t key_rows, int e_lo,
                                 int e_hi, int row_span, cudaStream_t stream) {
  if (!base || n_experts <= 0 || rows <= 0 || cols <= 0 || cols % 32 != 0 ||
      ((uintptr_t)base & 31) || e_lo < 0 || e_hi > 254 || e_lo > e_hi || row_span > e_hi - e_lo)
    return (int)cudaErrorInvalidValue;
  const int64_t nib = rows * cols / 2, sc = rows * cols / 32, eb = nib + sc;
  if (nib % 8 != 0) return (int)cudaErrorInvalidValue;
  fill_codes<<<148 * 8, 256, 0, stream>>>(base, n_experts, nib / 8, eb, key_codes);
  fill_scales<<<148 * 4, 256, 0, stream>>>(base, n_experts, rows, cols / 32, nib, sc, eb, key_scales, key_rows,
                                           (uint32_t)e_lo, (uint32_t)(e_hi - e_lo + 1), row_span);
  return (int)cudaGetLastError();
}
