// Per-head RMSNorm + rotate-half RoPE with the head split folded in, and the
// plain head split / merge transposes a layer forward needs.
//
// The agihunt.info summary of "Parallax: Parameterized Local Linear Attention
// for Language Modeling" says rho gets its own RMSNorm and that RoPE on it
// helps; q and k take the same Qwen-3-style treatment.  Readings adopted: unit
// RMSNorm weight, eps as given, frequencies base^(-2k/d), feature k paired with
// feature k + d/2, position = token index.
#include "plx_internal.cuh"

namespace plx {
namespace {

// RoPE frequencies base^(-2k/d) for k < d/2, computed once on the host.
struct RopeFreq {
  double f[64];
};

// Angle n * freq (up to ~10^4 rad) reduced modulo 2 pi in double, then its
// sine and cosine by the hardware approximation on [-pi, pi] (absolute error
// about 2^-21, far below the bf16 output's resolution).
__device__ __forceinline__ void rope_sincos(int n, double freq, float* sn, float* cs) {
  const double two_pi = 6.283185307179586476925286766559;
  const double inv_two_pi = 0.15915494309189533576888376337251;
  const double ang = (double)n * freq;
  const double red = fma(-rint(ang * inv_two_pi), two_pi, ang);
  __sincosf((float)red, sn, cs);
}

// One warp per (b, n, h) row, kRows rows in flight.  x: [B, N, H*d] bf16
// (token-major); y: [B, H, N, d].  Feature k is rotated with feature k + d/2.
// d = 128: lane l owns k = 2l, 2l+1 (and k + 64), read and written as bf16
// pairs; d = 64: lane l owns k = l.  Each lane's frequencies are fixed and
// computed once.
template <int D>
__global__ void __launch_bounds__(256) norm_rope_kernel(const __nv_bfloat16* __restrict__ x,
                                                        __nv_bfloat16* __restrict__ y, int B, int N,
                                                        int H, float eps, const RopeFreq fr) {
  constexpr int kRows = 4;
  constexpr int KPL = D / 64;  // pairs per lane: 2 (d = 128) or 1 (d = 64)
  constexpr int HALF = D / 2;
  const int lane = threadIdx.x & 31;
  // Index arithmetic in 32 bits (the host checks B*N*H < 2^31): 64-bit
  // division is emulated and would dominate this memory-bound kernel.
  const unsigned rows = (unsigned)B * N * H;
  const unsigned warps = (gridDim.x * blockDim.x) >> 5;
  double freq[KPL];
#pragma unroll
  for (int e = 0; e < KPL; ++e) freq[e] = fr.f[KPL * lane + e];
  for (unsigned r0 = ((blockIdx.x * blockDim.x + threadIdx.x) >> 5) * kRows; r0 < rows;
       r0 += warps * kRows) {
    float lo[kRows][KPL], hi[kRows][KPL];
#pragma unroll
    for (int q = 0; q < kRows; ++q) {
      const unsigned r = r0 + q;
      if (r < rows) {
        const __nv_bfloat16* src = x + (size_t)r * D;
        if constexpr (KPL == 2) {
          __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(src + 2 * lane);
          __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(src + HALF + 2 * lane);
          lo[q][0] = __low2float(a);
          lo[q][1] = __high2float(a);
          hi[q][0] = __low2float(b);
          hi[q][1] = __high2float(b);
        } else {
          lo[q][0] = __bfloat162float(src[lane]);
          hi[q][0] = __bfloat162float(src[HALF + lane]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < KPL; ++e) lo[q][e] = hi[q][e] = 0.f;
      }
    }
    // With H a multiple of kRows the warp's rows share one token position, so
    // the rotation factors are computed once for all of them.
    const bool shared_pos = (H % kRows) == 0;
    float sn0[KPL], cs0[KPL];
    if (shared_pos && r0 < rows) {
      const unsigned n0 = (r0 / (unsigned)H) % (unsigned)N;
#pragma unroll
      for (int e = 0; e < KPL; ++e) rope_sincos((int)n0, freq[e], &sn0[e], &cs0[e]);
    }
#pragma unroll
    for (int q = 0; q < kRows; ++q) {
      const unsigned r = r0 + q;
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < KPL; ++e) ss += lo[q][e] * lo[q][e] + hi[q][e] * hi[q][e];
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (r >= rows) continue;  // warp-uniform
      const float inv = rsqrtf(ss / (float)D + eps);
      const unsigned bn = r / (unsigned)H;
      const unsigned h = r - bn * (unsigned)H;
      const unsigned b = bn / (unsigned)N;
      const unsigned n = bn - b * (unsigned)N;
      __nv_bfloat16* dst = y + (((size_t)b * H + h) * N + n) * D;
      float o1[KPL], o2[KPL];
#pragma unroll
      for (int e = 0; e < KPL; ++e) {
        float sn = sn0[e], cs = cs0[e];
        if (!shared_pos) rope_sincos((int)n, freq[e], &sn, &cs);
        const float x1 = lo[q][e] * inv, x2 = hi[q][e] * inv;
        o1[e] = x1 * cs - x2 * sn;
        o2[e] = x2 * cs + x1 * sn;
      }
      if constexpr (KPL == 2) {
        *reinterpret_cast<__nv_bfloat162*>(dst + 2 * lane) = __floats2bfloat162_rn(o1[0], o1[1]);
        *reinterpret_cast<__nv_bfloat162*>(dst + HALF + 2 * lane) = __floats2bfloat162_rn(o2[0], o2[1]);
      } else {
        dst[lane] = __float2bfloat16_rn(o1[0]);
        dst[HALF + lane] = __float2bfloat16_rn(o2[0]);
      }
    }
  }
}

// [B, A1, A2, d] -> [B, A2, A1, d] in 16-byte pieces (head split and merge).
// 32-bit index arithmetic (the host checks the element count < 2^31).
__global__ void swap_axes_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int B,
                                 int A1, int A2, int vec_per_row) {
  const unsigned total = (unsigned)B * A1 * A2 * vec_per_row;
  for (unsigned i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const unsigned row = i / (unsigned)vec_per_row;
    const unsigned v = i - row * (unsigned)vec_per_row;
    const unsigned t = row / (unsigned)A2;
    const unsigned a2 = row - t * (unsigned)A2;
    const unsigned b = t / (unsigned)A1;
    const unsigned a1 = t - b * (unsigned)A1;
    dst[(((size_t)b * A2 + a2) * A1 + a1) * vec_per_row + v] = src[i];
  }
}

}  // namespace

cudaError_t launch_swap_axes(const void* src, void* dst, int B, int A1, int A2, int d,
                             cudaStream_t st) {
  int vpr = d * 2 / 16;
  long long total = (long long)B * A1 * A2 * vpr;
  long long blocks = (total + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  swap_axes_kernel<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const uint4*>(src),
                                                      reinterpret_cast<uint4*>(dst), B, A1, A2, vpr);
  return cudaGetLastError();
}

cudaError_t launch_qkr_norm_rope(const void* x, void* y, int B, int N, int H, int d, float eps,
                                 float base, cudaStream_t st) {
  long long rows = (long long)B * N * H;
  long long blocks = (rows + 31) / 32;  // 8 warps x 4 rows per block and step
  if (blocks > 148 * 16) blocks = 148 * 16;
  RopeFreq fr;
  for (int k = 0; k < 64; ++k) fr.f[k] = k < d / 2 ? pow((double)base, -2.0 * k / (double)d) : 0.0;
  auto xs = reinterpret_cast<const __nv_bfloat16*>(x);
  auto ys = reinterpret_cast<__nv_bfloat16*>(y);
  if (d == 128) {
    norm_rope_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(xs, ys, B, N, H, eps, fr);
  } else {
    norm_rope_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(xs, ys, B, N, H, eps, fr);
  }
  return cudaGetLastError();
}

}  // namespace plx
