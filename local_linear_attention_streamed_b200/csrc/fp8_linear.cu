// Dynamic fp8 (e4m3) linear layers for the Parallax layer wrapper.
//
// The pages pretrain with the linear layers in dynamic fp8 ("Parallax:
// Parameterized Local Linear Attention for Language Modeling", rainbus.top
// reproduction notes: dynamic fp8 for the linear layers, bf16 for the LM head).
// Reading: one scale per tensor per call, s = max|a| / 448 (the largest e4m3
// value); each operand of a linear (activation and weight) is divided by its
// scale and rounded to e4m3 (nearest, ties to even, saturating), and the GEMM
// accumulates in fp32 and multiplies by s_a s_w.
//
// Kernels here: a per-tensor |max| reduction, a quantiser, and a quantiser
// that also transposes a weight into the operand layout the fp8 GEMM takes.
// The GEMM itself is a plain library call (cuBLASLt, e4m3 x e4m3 -> bf16 with
// device-side scale pointers, so no host synchronisation).
#include "plx_internal.cuh"

#include <cublasLt.h>
#include <cuda_fp8.h>

namespace plx {
namespace {

constexpr float kE4m3Max = 448.f;

__device__ __forceinline__ float scale_of(const unsigned* amax_bits) {
  const float amax = __uint_as_float(*amax_bits);
  return amax > 0.f ? amax / kE4m3Max : 1.f;
}

// max |x| over n bf16 values (n a multiple of 8, x 16-byte aligned) into
// *amax_bits, as float bits: non-negative floats order like their bit
// patterns, so an unsigned atomicMax reduces them (*amax_bits starts at 0).
__global__ void __launch_bounds__(256) amax_kernel(const __nv_bfloat16* __restrict__ x, size_t n,
                                                   unsigned* __restrict__ amax_bits) {
  float m = 0.f;
  const size_t stride = (size_t)gridDim.x * blockDim.x * 8;
  for (size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; i < n; i += stride) {
    const uint4 v = *reinterpret_cast<const uint4*>(x + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

// out[i] = e4m3(x[i] / s), s from *amax_bits; block 0 publishes s.
__global__ void __launch_bounds__(256) quant_kernel(const __nv_bfloat16* __restrict__ x, size_t n,
                                                    const unsigned* __restrict__ amax_bits,
                                                    __nv_fp8_e4m3* __restrict__ out, float* __restrict__ scale) {
  const float s = scale_of(amax_bits);
  if (blockIdx.x == 0 && threadIdx.x == 0) *scale = s;
  const size_t stride = (size_t)gridDim.x * blockDim.x * 8;
  for (size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; i < n; i += stride) {
    const uint4 v = *reinterpret_cast<const uint4*>(x + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint8_t q[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
      q[2 * j] = __nv_cvt_float_to_fp8(__fdiv_rn(f.x, s), __NV_SATFINITE, __NV_E4M3);
      q[2 * j + 1] = __nv_cvt_float_to_fp8(__fdiv_rn(f.y, s), __NV_SATFINITE, __NV_E4M3);
    }
    *reinterpret_cast<uint2*>(out + i) = *reinterpret_cast<const uint2*>(q);
  }
}

// Wt[c][r] = e4m3(W[r][c] / s) for W [rows][cols] bf16: 32 x 32 tiles through
// shared memory (rows and cols multiples of 32).
__global__ void __launch_bounds__(256) quant_t_kernel(const __nv_bfloat16* __restrict__ W, int rows, int cols,
                                                      const unsigned* __restrict__ amax_bits,
                                                      __nv_fp8_e4m3* __restrict__ Wt, float* __restrict__ scale) {
  __shared__ float tile[32][33];
  const float s = scale_of(amax_bits);
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 && threadIdx.y == 0) *scale = s;
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int y = threadIdx.y; y < 32; y += 8)
    tile[y][threadIdx.x] = __bfloat162float(W[(size_t)(r0 + y) * cols + c0 + threadIdx.x]);
  __syncthreads();
  for (int y = threadIdx.y; y < 32; y += 8) {
    const float v = tile[threadIdx.x][y];
    reinterpret_cast<uint8_t*>(Wt)[(size_t)(c0 + y) * rows + r0 + threadIdx.x] =
        __nv_cvt_float_to_fp8(__fdiv_rn(v, s), __NV_SATFINITE, __NV_E4M3);
  }
}

int grid_for(size_t n) {
  const size_t blocks = (n / 8 + 255) / 256;
  return (int)(blocks < 4096 ? (blocks > 0 ? blocks : 1) : 4096);
}

}  // namespace

cudaError_t launch_amax(const void* x, size_t n, unsigned* amax_bits, cudaStream_t st) {
  amax_kernel<<<grid_for(n), 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(x), n, amax_bits);
  return cudaGetLastError();
}

cudaError_t launch_quant(const void* x, size_t n, const unsigned* amax_bits, void* out, float* scale,
                         cudaStream_t st) {
  quant_kernel<<<grid_for(n), 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(x), n, amax_bits,
                                            reinterpret_cast<__nv_fp8_e4m3*>(out), scale);
  return cudaGetLastError();
}

cudaError_t launch_quant_t(const void* W, int rows, int cols, const unsigned* amax_bits, void* Wt, float* scale,
                           cudaStream_t st) {
  dim3 grid(cols / 32, rows / 32), block(32, 8);
  quant_t_kernel<<<grid, block, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(W), rows, cols, amax_bits,
                                         reinterpret_cast<__nv_fp8_e4m3*>(Wt), scale);
  return cudaGetLastError();
}

// Y[M, Dout] (bf16, row-major) = (X8[M, Din] Wt8[Dout, Din]^T) * sX * sW, both
// operands e4m3 row-major.  Column-major view for cuBLASLt: Y^T = Wt8 X8^T with
// A = Wt8 stored Din x Dout (transposed), B = X8 stored Din x M.
int fp8_gemm(void* lt_handle, const void* Wt8, const void* X8, void* Y, int Dout, int Din, long long M,
             const float* sW, const float* sX, void* ws, size_t ws_bytes, cudaStream_t st) {
  cublasLtHandle_t lt = static_cast<cublasLtHandle_t>(lt_handle);
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
  cublasLtMatmulPreference_t pref = nullptr;
  int rc = -1;
  do {
    if (cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS) break;
    const cublasOperation_t tA = CUBLAS_OP_T, tB = CUBLAS_OP_N;
    cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &tA, sizeof(tA));
    cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &tB, sizeof(tB));
    cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_A_SCALE_POINTER, &sW, sizeof(sW));
    cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_B_SCALE_POINTER, &sX, sizeof(sX));
    if (cublasLtMatrixLayoutCreate(&la, CUDA_R_8F_E4M3, Din, Dout, Din) != CUBLAS_STATUS_SUCCESS) break;
    if (cublasLtMatrixLayoutCreate(&lb, CUDA_R_8F_E4M3, Din, (uint64_t)M, Din) != CUBLAS_STATUS_SUCCESS) break;
    if (cublasLtMatrixLayoutCreate(&lc, CUDA_R_16BF, Dout, (uint64_t)M, Dout) != CUBLAS_STATUS_SUCCESS) break;
    if (cublasLtMatmulPreferenceCreate(&pref) != CUBLAS_STATUS_SUCCESS) break;
    cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &ws_bytes,
                                         sizeof(ws_bytes));
    cublasLtMatmulHeuristicResult_t heur;
    int found = 0;
    if (cublasLtMatmulAlgoGetHeuristic(lt, op, la, lb, lc, lc, pref, 1, &heur, &found) != CUBLAS_STATUS_SUCCESS ||
        found < 1)
      break;
    const float one = 1.f, zero = 0.f;
    if (cublasLtMatmul(lt, op, &one, Wt8, la, X8, lb, &zero, Y, lc, Y, lc, &heur.algo, ws, ws_bytes, st) !=
        CUBLAS_STATUS_SUCCESS)
      break;
    rc = 0;
  } while (false);
  if (pref) cublasLtMatmulPreferenceDestroy(pref);
  if (lc) cublasLtMatrixLayoutDestroy(lc);
  if (lb) cublasLtMatrixLayoutDestroy(lb);
  if (la) cublasLtMatrixLayoutDestroy(la);
  if (op) cublasLtMatmulDescDestroy(op);
  return rc;
}

}  // namespace plx
