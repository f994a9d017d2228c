// Pieces shared by the tensor-core decode kernels (bf16 caches in
// decode_gqa_tc.cu, e4m3 caches in decode_fp8kv.cu): the instruction
// descriptor, the 128B-swizzled tile addressing, TMEM column loads and
// stores of accumulator width, and the work-unit arithmetic of the split plan.
#pragma once

#include "plx_internal.cuh"
#include "sm100.cuh"

namespace plx {
namespace dtc {

using namespace sm100;

constexpr int kKeys = 128;  // keys per staged block (the MMA M of the score product)

// Instruction descriptor (kind::f16): D f32, M = 128, N = n; A and B both bf16
// (bf16 = true) or both f16; a_mn / b_mn = 1 for an MN-major A / B operand.
__host__ __device__ constexpr uint32_t idesc_f16kind(int n, int a_mn, int b_mn, bool bf16) {
  return (1u << 4) | (bf16 ? (1u << 7) | (1u << 10) : 0u) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(n >> 3) << 17) | ((128u >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc(int n, int a_mn, int b_mn) { return idesc_f16kind(n, a_mn, b_mn, true); }
// Instruction descriptor (kind::f8f6f4): D f32, M = 128, N = n, A and B e4m3
// (type code 0), both K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3(int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((128u >> 4) << 24);
}

// Byte offset of element column `col` (2-byte elements) of row `row` in a
// 128B-swizzled tile of 128-byte rows.
__device__ __forceinline__ uint32_t sw128_elem(int row, int col) {
  return (uint32_t)(row * 128 + ((((col >> 3) ^ (row & 7))) << 4) + (col & 7) * 2);
}
// Byte offset of 16-byte chunk `c` (0..7) of row `row` in the same layout.
__device__ __forceinline__ uint32_t sw128_chunk(int row, int c) {
  return (uint32_t)(row * 128 + ((c ^ (row & 7)) << 4));
}

// Bounded wait taken by a whole warp: every lane leaves with the same answer.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* status) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, status));
}

template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&v)[N]) {
  static_assert(N % 16 == 0 && N <= 64, "accumulator width");
#pragma unroll
  for (int c = 0; c < N / 32; ++c) tmem_ld32(taddr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
  if constexpr (N % 32 == 16) tmem_ld16(taddr + (N - 16), *reinterpret_cast<uint32_t(*)[16]>(&v[N - 16]));
}
template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&v)[N]) {
#pragma unroll
  for (int c = 0; c < N / 16; ++c) {
    uint32_t part[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) part[x] = v[16 * c + x];
    tmem_st16(taddr + 16 * c, part);
  }
}

// Warp maxima of H values per lane (H a power of two <= 32) in H - 1 + 5 -
// log2 H shuffles instead of 5 H: a reduce-scatter (at each step a lane keeps
// half of its values and takes the partner's maxima of that half), then a
// butterfly over the remaining lanes.  Afterwards lane l holds the maximum
// over the warp of value number l / (32 / H).
template <int N, int O>
struct MaxScatter {
  template <int H>
  static __device__ __forceinline__ void run(float (&v)[H], int lane) {
    const bool upper = (lane & O) != 0;
#pragma unroll
    for (int j = 0; j < N / 2; ++j) {
      const float keep = upper ? v[j + N / 2] : v[j];
      const float give = upper ? v[j] : v[j + N / 2];
      v[j] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, give, O));
    }
    MaxScatter<N / 2, O / 2>::run(v, lane);
  }
};
template <int O>
struct MaxScatter<1, O> {
  template <int H>
  static __device__ __forceinline__ void run(float (&v)[H], int) {
#pragma unroll
    for (int o = O; o > 0; o >>= 1) v[0] = fmaxf(v[0], __shfl_xor_sync(0xffffffffu, v[0], o));
  }
};
template <int H>
__device__ __forceinline__ float warp_max_scatter(const float (&x)[H], int lane) {
  static_assert(H >= 1 && H <= 32 && (H & (H - 1)) == 0, "a power of two");
  float v[H];
#pragma unroll
  for (int j = 0; j < H; ++j) v[j] = x[j];
  MaxScatter<H, 16>::run(v, lane);
  return v[0];
}
// The block maxima of H values: each of 4 warps wrote its row red[w][0..H)
// (16-byte aligned rows when H % 4 == 0).
template <int H>
__device__ __forceinline__ void block_max4(const float (&red)[4][H], float (&m)[H]) {
  if constexpr (H % 4 == 0) {
#pragma unroll
    for (int c = 0; c < H / 4; ++c) {
      const float4 a = reinterpret_cast<const float4*>(red[0])[c], b = reinterpret_cast<const float4*>(red[1])[c];
      const float4 e = reinterpret_cast<const float4*>(red[2])[c], f = reinterpret_cast<const float4*>(red[3])[c];
      m[4 * c + 0] = fmaxf(fmaxf(a.x, b.x), fmaxf(e.x, f.x));
      m[4 * c + 1] = fmaxf(fmaxf(a.y, b.y), fmaxf(e.y, f.y));
      m[4 * c + 2] = fmaxf(fmaxf(a.z, b.z), fmaxf(e.z, f.z));
      m[4 * c + 3] = fmaxf(fmaxf(a.w, b.w), fmaxf(e.w, f.w));
    }
  } else {
#pragma unroll
    for (int h = 0; h < H; ++h) m[h] = fmaxf(fmaxf(red[0][h], red[1][h]), fmaxf(red[2][h], red[3][h]));
  }
}

// What every role derives from a unit index: unit u covers KV heads
// kvh .. kvh + kPair - 1 of batch row b (bkv = b Hkv + kvh) over key chunk c.
struct Unit {
  int b, kvh, bkv, c, n, kbeg, kend, nch, nblk;
  bool bad;
};
// Batch row of unit u (units are chunk-major over the (b, KV-head group) pairs).
__device__ __forceinline__ int unit_row(long long u, int kPair, const DecodeArgs& a) {
  const int per_b = a.Hkv / kPair;
  return (int)(u % ((long long)a.B * per_b)) / per_b;
}
__device__ __forceinline__ Unit unit_of(long long u, int n, int kPair, const DecodeArgs& a) {
  const int per_b = a.Hkv / kPair, BU = a.B * per_b;
  Unit x;
  x.c = (int)(u / BU);
  const int bu = (int)(u - (long long)x.c * BU);
  x.b = bu / per_b;
  x.kvh = (bu - x.b * per_b) * kPair;
  x.bkv = x.b * a.Hkv + x.kvh;
  x.n = n;
  x.bad = x.n < 1 || x.n > a.L;
  // Keys lo..n-1 (lo > 0 only with a sliding window), cut into chunks.
  const int lo = (!x.bad && a.window > 0 && x.n > a.window) ? x.n - a.window : 0;
  x.kbeg = lo + x.c * a.chunk;
  x.kend = x.bad ? x.kbeg : min(x.kbeg + a.chunk, x.n);
  x.nblk = (!x.bad && x.kbeg < x.n) ? (x.kend - x.kbeg + kKeys - 1) / kKeys : 0;
  x.nch = x.bad ? 0 : (x.n - lo + a.chunk - 1) / a.chunk;
  return x;
}

}  // namespace dtc
}  // namespace plx
