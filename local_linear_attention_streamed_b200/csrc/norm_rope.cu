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

// One warp per (b, n, h) row.  x: [B, N, H*d] bf16 (token-major); y: [B, H, N, d].
__global__ void norm_rope_kernel(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ y,
                                 int B, int N, int H, int d, float eps, float base) {
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)B * N * H;
  const long long warps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int half = d >> 1;
  const int ppl = half >> 5;  // rotation pairs per lane (1 or 2 for d = 64, 128)
  for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += warps) {
    const int h = (int)(r % H);
    const long long bn = r / H;
    const int n = (int)(bn % N);
    const int b = (int)(bn / N);
    const __nv_bfloat16* src = x + r * d;  // row (b, n, h) is contiguous in [B, N, H*d]
    __nv_bfloat16* dst = y + (((long long)b * H + h) * N + n) * d;
    float lo[2], hi[2];
    float ss = 0.f;
    for (int e = 0; e < ppl; ++e) {
      int k = lane + 32 * e;
      lo[e] = __bfloat162float(src[k]);
      hi[e] = __bfloat162float(src[k + half]);
      ss += lo[e] * lo[e] + hi[e] * hi[e];
    }
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rsqrtf(ss / (float)d + eps);
    for (int e = 0; e < ppl; ++e) {
      int k = lane + 32 * e;
      // Angle in double: positions reach 10^4 radians, beyond fp32 resolution.
      double freq = pow((double)base, -2.0 * (double)k / (double)d);
      double sn, cs;
      sincos((double)n * freq, &sn, &cs);
      float x1 = lo[e] * inv, x2 = hi[e] * inv;
      float c = (float)cs, s = (float)sn;
      dst[k] = __float2bfloat16_rn(x1 * c - x2 * s);
      dst[k + half] = __float2bfloat16_rn(x2 * c + x1 * s);
    }
  }
}

// [B, A1, A2, d] -> [B, A2, A1, d] in 16-byte pieces (head split and merge).
__global__ void swap_axes_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int B,
                                 int A1, int A2, int vec_per_row) {
  const long long total = (long long)B * A1 * A2 * vec_per_row;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    int v = (int)(i % vec_per_row);
    long long row = i / vec_per_row;
    int a2 = (int)(row % A2);
    long long t = row / A2;
    int a1 = (int)(t % A1);
    int b = (int)(t / A1);
    dst[(((long long)b * A2 + a2) * A1 + a1) * vec_per_row + v] = src[i];
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
  long long blocks = (rows + 7) / 8;
  if (blocks > 148 * 64) blocks = 148 * 64;
  norm_rope_kernel<<<(unsigned)blocks, 256, 0, st>>>(
      reinterpret_cast<const __nv_bfloat16*>(x), reinterpret_cast<__nv_bfloat16*>(y), B, N, H, d,
      eps, base);
  return cudaGetLastError();
}

}  // namespace plx
