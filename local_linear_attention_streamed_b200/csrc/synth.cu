// Device side of the seeded synthetic-input generator (see include/plx_synth.h).
// Holds no Parallax arithmetic.  Every step is integer arithmetic or a single
// IEEE-rounded double operation so that the host generator reproduces each
// element bit for bit.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/plx_synth.h"

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ int64_t irwin_hall(uint64_t key, uint64_t idx) {
  uint64_t h = mix64(key + (idx + 1ull) * kGamma);
  int64_t s = (int64_t)(h & 0xFFFFull) + (int64_t)((h >> 16) & 0xFFFFull) +
              (int64_t)((h >> 32) & 0xFFFFull) + (int64_t)(h >> 48);
  return s - 2 * 65535;
}

// float -> bf16 bits, round to nearest even (finite inputs), written out on
// the bit pattern so that it matches the host generator exactly.
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

__device__ __forceinline__ void store(void* dst, int dtype, uint64_t i, double v) {
  float f = __double2float_rn(v);
  if (dtype == 0) {
    reinterpret_cast<float*>(dst)[i] = f;
  } else {
    reinterpret_cast<uint16_t*>(dst)[i] = f32_to_bf16_bits(f);
  }
}

__global__ void fill_normal(void* dst, int dtype, uint64_t key, uint64_t count, double scale) {
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride) {
    double v = __dmul_rn((double)irwin_hall(key, i), scale);
    store(dst, dtype, i, v);
  }
}

// One warp per row: lanes take elements lane, lane+32, ...; the exact integer
// sum of squares is reduced across the warp (integer addition is exact in any
// order), then every lane stores n / sqrt(ss / row) for its elements.
__global__ void fill_rms_rows(void* dst, int dtype, uint64_t key, uint64_t rows, int64_t row) {
  const int lane = threadIdx.x & 31;
  uint64_t warps = ((uint64_t)gridDim.x * blockDim.x) >> 5;
  for (uint64_t r = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += warps) {
    uint64_t base = r * (uint64_t)row;
    long long ss = 0;
    for (int64_t j = lane; j < row; j += 32) {
      long long n = irwin_hall(key, base + j);
      ss += n * n;
    }
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    double den = __dsqrt_rn(__ddiv_rn((double)ss, (double)row));
    for (int64_t j = lane; j < row; j += 32) {
      int64_t n = irwin_hall(key, base + j);
      store(dst, dtype, base + j, __ddiv_rn((double)n, den));
    }
  }
}

}  // namespace

extern "C" int plx_synth_fill(void* dst, int dtype, uint64_t key, uint64_t count, int dist,
                              double scale, int64_t row, void* stream) {
  if (dst == nullptr || (dtype != 0 && dtype != 1) || (dist != 0 && dist != 1)) return -1;
  if (count == 0) return 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (dist == 0) {
    uint64_t blocks = (count + 255) / 256;
    uint64_t cap = (uint64_t)sms * 16;
    fill_normal<<<(unsigned)(blocks < cap ? blocks : cap), 256, 0, st>>>(dst, dtype, key, count, scale);
  } else {
    if (row <= 0 || count % (uint64_t)row) return -1;
    uint64_t rows = count / (uint64_t)row;
    uint64_t blocks = (rows + 7) / 8;  // 8 warps (rows) per block
    uint64_t cap = (uint64_t)sms * 16;
    fill_rms_rows<<<(unsigned)(blocks < cap ? blocks : cap), 256, 0, st>>>(dst, dtype, key, rows, row);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}
