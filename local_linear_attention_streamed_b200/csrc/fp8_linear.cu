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

#include <mutex>

#include <cublasLt.h>
#include <cuda_fp8.h>

namespace plx {
namespace {

constexpr float kE4m3Max = 448.f;

__device__ __forceinline__ float scale_of(const unsigned* amax_bits) {
  const float amax = __uint_as_float(*amax_bits);
  return amax > 0.f ? amax / kE4m3Max : 1.f;
}

// Up to five tensors of one launch (blockIdx.y picks one).
struct Tensors5 {
  const __nv_bfloat16* x[5];
  unsigned* amax_bits[5];
  __nv_fp8_e4m3* out[5];
  float* scale[5];
};

// max |x| over n bf16 values (n a multiple of 8, x 16-byte aligned) into
// *amax_bits, as float bits: non-negative floats order like their bit
// patterns, so an unsigned atomicMax reduces them (*amax_bits starts at 0).
// One atomic per block after a warp and a block reduction.
__global__ void __launch_bounds__(256) amax_kernel(Tensors5 t, size_t n) {
  const __nv_bfloat16* __restrict__ x = t.x[blockIdx.y];
  __shared__ float wmax[8];
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
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, wmax[w]);
    atomicMax(t.amax_bits[blockIdx.y], __float_as_uint(m));
  }
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

// Wt[c][r] = e4m3(W[r][c] / s) for W [rows][cols] bf16 (blockIdx.z picks the
// tensor): 64 x 64 tiles through shared memory, 16-byte loads and 4-byte
// stores (rows and cols multiples of 64).
__global__ void __launch_bounds__(256) quant_t_kernel(Tensors5 t, int rows, int cols) {
  __shared__ float tile[64][65];
  const int z = blockIdx.z;
  const float s = scale_of(t.amax_bits[z]);
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *t.scale[z] = s;
  const __nv_bfloat16* __restrict__ W = t.x[z];
  const int r0 = blockIdx.y * 64, c0 = blockIdx.x * 64;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int idx = threadIdx.x + 256 * k, r = idx >> 3, c8 = (idx & 7) * 8;
    const uint4 v = *reinterpret_cast<const uint4*>(W + (size_t)(r0 + r) * cols + c0 + c8);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
      tile[r][c8 + 2 * j] = f.x;
      tile[r][c8 + 2 * j + 1] = f.y;
    }
  }
  __syncthreads();
  uint8_t* __restrict__ out = reinterpret_cast<uint8_t*>(t.out[z]);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int idx = threadIdx.x + 256 * k, oc = idx >> 4, r4 = (idx & 15) * 4;
    uint32_t packed = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      packed |= (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(tile[r4 + e][oc], s), __NV_SATFINITE, __NV_E4M3)
                << (8 * e);
    *reinterpret_cast<uint32_t*>(out + (size_t)(c0 + oc) * rows + r0 + r4) = packed;
  }
}

int grid_for(size_t n) {
  const size_t blocks = (n / 8 + 255) / 256;
  return (int)(blocks < 1184 ? (blocks > 0 ? blocks : 1) : 1184);  // 8 blocks per SM at most
}

}  // namespace

cudaError_t launch_amax(const void* const* x, int count, size_t n, unsigned* amax_bits, cudaStream_t st) {
  if (count < 1 || count > 5) return cudaErrorInvalidValue;
  Tensors5 t{};
  for (int i = 0; i < count; ++i) {
    t.x[i] = reinterpret_cast<const __nv_bfloat16*>(x[i]);
    t.amax_bits[i] = amax_bits + i;
  }
  amax_kernel<<<dim3(grid_for(n), count), 256, 0, st>>>(t, n);
  return cudaGetLastError();
}

cudaError_t launch_quant(const void* x, size_t n, const unsigned* amax_bits, void* out, float* scale,
                         cudaStream_t st) {
  // Streaming conversion: enough blocks to keep every SM's memory pipe busy.
  const size_t blocks = (n / 8 + 255) / 256;
  quant_kernel<<<(int)(blocks < 4096 ? (blocks > 0 ? blocks : 1) : 4096), 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(x), n, amax_bits,
                                            reinterpret_cast<__nv_fp8_e4m3*>(out), scale);
  return cudaGetLastError();
}

cudaError_t launch_quant_t(const void* const* W, int count, int rows, int cols, const unsigned* amax_bits,
                           void* Wt, size_t wt_stride, float* scale, cudaStream_t st) {
  if (count < 1 || count > 5 || rows % 64 != 0 || cols % 64 != 0) return cudaErrorInvalidValue;
  Tensors5 t{};
  for (int i = 0; i < count; ++i) {
    t.x[i] = reinterpret_cast<const __nv_bfloat16*>(W[i]);
    t.amax_bits[i] = const_cast<unsigned*>(amax_bits) + i;
    t.out[i] = reinterpret_cast<__nv_fp8_e4m3*>(static_cast<char*>(Wt) + i * wt_stride);
    t.scale[i] = scale + i;
  }
  quant_t_kernel<<<dim3(cols / 64, rows / 64, count), 256, 0, st>>>(t, rows, cols);
  return cudaGetLastError();
}

// Y[M, Dout] (bf16, row-major) = (X8[M, Din] Wt8[Dout, Din]^T) * sX * sW, both
// operands e4m3 row-major.  Column-major view for cuBLASLt: Y^T = Wt8 X8^T with
// A = Wt8 stored Din x Dout (transposed), B = X8 stored Din x M.
//
// The matmul descriptor, the three layouts and the algorithm the heuristic
// picks depend only on the handle and the sizes, so they are built once per
// shape and kept (a layer step runs five GEMMs of two shapes); only the scale
// pointers, which may move with the caller's workspace, are set per call.
namespace {

struct Fp8Plan {
  void* lt = nullptr;
  int Dout = 0, Din = 0;
  long long M = 0;
  size_t ws_bytes = 0;
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
  cublasLtMatmulAlgo_t algo{};
};

constexpr int kPlans = 16;
std::mutex g_plan_mu;
Fp8Plan g_plans[kPlans];
int g_plan_next = 0;

void destroy_plan(Fp8Plan& p) {
  if (p.lc) cublasLtMatrixLayoutDestroy(p.lc);
  if (p.lb) cublasLtMatrixLayoutDestroy(p.lb);
  if (p.la) cublasLtMatrixLayoutDestroy(p.la);
  if (p.op) cublasLtMatmulDescDestroy(p.op);
  p = Fp8Plan{};
}

// The cached plan for these sizes, built on first use (nullptr on failure).
Fp8Plan* plan_for(void* lt_handle, int Dout, int Din, long long M, size_t ws_bytes) {
  for (Fp8Plan& p : g_plans)
    if (p.op && p.lt == lt_handle && p.Dout == Dout && p.Din == Din && p.M == M && p.ws_bytes == ws_bytes)
      return &p;
  Fp8Plan& p = g_plans[g_plan_next];
  g_plan_next = (g_plan_next + 1) % kPlans;
  destroy_plan(p);
  cublasLtHandle_t lt = static_cast<cublasLtHandle_t>(lt_handle);
  cublasLtMatmulPreference_t pref = nullptr;
  bool ok = false;
  do {
    if (cublasLtMatmulDescCreate(&p.op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS) break;
    const cublasOperation_t tA = CUBLAS_OP_T, tB = CUBLAS_OP_N;
    cublasLtMatmulDescSetAttribute(p.op, CUBLASLT_MATMUL_DESC_TRANSA, &tA, sizeof(tA));
    cublasLtMatmulDescSetAttribute(p.op, CUBLASLT_MATMUL_DESC_TRANSB, &tB, sizeof(tB));
    if (cublasLtMatrixLayoutCreate(&p.la, CUDA_R_8F_E4M3, Din, Dout, Din) != CUBLAS_STATUS_SUCCESS) break;
    if (cublasLtMatrixLayoutCreate(&p.lb, CUDA_R_8F_E4M3, Din, (uint64_t)M, Din) != CUBLAS_STATUS_SUCCESS) break;
    if (cublasLtMatrixLayoutCreate(&p.lc, CUDA_R_16BF, Dout, (uint64_t)M, Dout) != CUBLAS_STATUS_SUCCESS) break;
    if (cublasLtMatmulPreferenceCreate(&pref) != CUBLAS_STATUS_SUCCESS) break;
    cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &ws_bytes,
                                         sizeof(ws_bytes));
    cublasLtMatmulHeuristicResult_t heur;
    int found = 0;
    if (cublasLtMatmulAlgoGetHeuristic(lt, p.op, p.la, p.lb, p.lc, p.lc, pref, 1, &heur, &found) !=
            CUBLAS_STATUS_SUCCESS ||
        found < 1)
      break;
    p.algo = heur.algo;
    ok = true;
  } while (false);
  if (pref) cublasLtMatmulPreferenceDestroy(pref);
  if (!ok) {
    destroy_plan(p);
    return nullptr;
  }
  p.lt = lt_handle;
  p.Dout = Dout;
  p.Din = Din;
  p.M = M;
  p.ws_bytes = ws_bytes;
  return &p;
}

}  // namespace

int fp8_gemm(void* lt_handle, const void* Wt8, const void* X8, void* Y, int Dout, int Din, long long M,
             const float* sW, const float* sX, void* ws, size_t ws_bytes, cudaStream_t st) {
  std::lock_guard<std::mutex> lk(g_plan_mu);
  Fp8Plan* p = plan_for(lt_handle, Dout, Din, M, ws_bytes);
  if (!p) return -1;
  if (cublasLtMatmulDescSetAttribute(p->op, CUBLASLT_MATMUL_DESC_A_SCALE_POINTER, &sW, sizeof(sW)) !=
          CUBLAS_STATUS_SUCCESS ||
      cublasLtMatmulDescSetAttribute(p->op, CUBLASLT_MATMUL_DESC_B_SCALE_POINTER, &sX, sizeof(sX)) !=
          CUBLAS_STATUS_SUCCESS)
    return -1;
  const float one = 1.f, zero = 0.f;
  if (cublasLtMatmul(static_cast<cublasLtHandle_t>(lt_handle), p->op, &one, Wt8, p->la, X8, p->lb, &zero, Y, p->lc,
                     Y, p->lc, &p->algo, ws, ws_bytes, st) != CUBLAS_STATUS_SUCCESS)
    return -1;
  return 0;
}

}  // namespace plx
