// Exact-path Parallax kernels on the CUDA cores (FFMA, fp32 throughout,
// precise expf).  They serve fp32 tensors, where tensor cores have no fp32
// mode and the 1e-5 parity bar rules out TF32, and any head dim that the
// tensor-core kernels do not cover.
//
// Streamed form ("Parallax: Parameterized Local Linear Attention for Language
// Modeling", rainbus.top summary, "方法步骤详情"; agihunt.info summary, hardware
// paragraph): per chunk of 32 keys, S1 = q.k/sqrt(d) and S2 = rho.k; one
// running max m and one factor alpha rescale omega = sum w, T = sum w t,
// O1 = sum w v and O2 = sum w t v; at the end tbar = T/omega and
// out = ((1 + tbar) O1 - O2) / omega.
#include "plx_internal.cuh"

#include <math_constants.h>

namespace plx {
namespace {

constexpr int kChunk = 32;        // keys per shared-memory chunk (one per lane)
constexpr int kRowsPerWarp = 4;   // query rows each warp carries in prefill
constexpr int kWarps = 4;
constexpr int kRowsPerCta = kRowsPerWarp * kWarps;
constexpr int kMaxD = 128;
constexpr int kMaxDpl = kMaxD / 32;  // dims per lane

template <bool BF16>
__device__ __forceinline__ float ld(const void* p, long long i) {
  if constexpr (BF16) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  } else {
    return reinterpret_cast<const float*>(p)[i];
  }
}

template <bool BF16>
__device__ __forceinline__ void st(void* p, long long i, float v) {
  if constexpr (BF16) {
    reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  } else {
    reinterpret_cast<float*>(p)[i] = v;
  }
}

__device__ __forceinline__ float warp_max(float v) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Running state of one query row; lane owns dims lane + 32*e.
struct RowState {
  float m, omega, T;
  float O1[kMaxDpl], O2[kMaxDpl];
  __device__ void init() {
    m = -CUDART_INF_F;
    omega = 0.f;
    T = 0.f;
#pragma unroll
    for (int e = 0; e < kMaxDpl; ++e) O1[e] = O2[e] = 0.f;
  }
};

// One chunk of up to 32 keys for one row.  Ks is [32][d+1] (padded), Vs is
// [32][d]; q and rho rows live in shared memory.  `valid` says whether this
// lane's key is visible to the row.
__device__ __forceinline__ void row_update(RowState& s, const float* qrow, const float* rrow,
                                           const float* Ks, const float* Vs, int d, bool valid,
                                           float inv_sqrt_d, int lane) {
  const float* kr = Ks + lane * (d + 1);
  float s1 = 0.f, s2 = 0.f;
  for (int a = 0; a < d; ++a) {
    float kv = kr[a];
    s1 = fmaf(qrow[a], kv, s1);
    s2 = fmaf(rrow[a], kv, s2);
  }
  s1 = valid ? s1 * inv_sqrt_d : -CUDART_INF_F;
  float cmax = warp_max(s1);
  if (cmax == -CUDART_INF_F) return;  // no visible key in this chunk (warp-uniform)
  float m_new = fmaxf(s.m, cmax);
  float alpha = (s.m == -CUDART_INF_F) ? 0.f : expf(s.m - m_new);
  float w = valid ? expf(s1 - m_new) : 0.f;
  float wt = w * s2;
  s.omega = fmaf(alpha, s.omega, warp_sum(w));
  s.T = fmaf(alpha, s.T, warp_sum(wt));
  s.m = m_new;
  const int dpl = d >> 5;
#pragma unroll
  for (int e = 0; e < kMaxDpl; ++e) {
    if (e < dpl) {
      s.O1[e] *= alpha;
      s.O2[e] *= alpha;
    }
  }
  for (int j = 0; j < kChunk; ++j) {
    float wj = __shfl_sync(0xffffffffu, w, j);
    float wtj = __shfl_sync(0xffffffffu, wt, j);
    const float* vr = Vs + j * d + lane;
#pragma unroll
    for (int e = 0; e < kMaxDpl; ++e) {
      if (e < dpl) {
        float v = vr[32 * e];
        s.O1[e] = fmaf(wj, v, s.O1[e]);
        s.O2[e] = fmaf(wtj, v, s.O2[e]);
      }
    }
  }
}

template <bool BF16>
__device__ __forceinline__ void row_finish(const RowState& s, void* out, long long row_off, int d,
                                           int lane) {
  const int dpl = d >> 5;
  float inv = 1.f / s.omega;
  float one_plus_tbar = 1.f + s.T * inv;
#pragma unroll
  for (int e = 0; e < kMaxDpl; ++e) {
    if (e < dpl) {
      float o = (one_plus_tbar * s.O1[e] - s.O2[e]) * inv;
      st<BF16>(out, row_off + lane + 32 * e, o);
    }
  }
}

// Stage keys [k0, k0+32) of one (b, h) (rows beyond `nkeys` are zero).
template <bool BF16>
__device__ __forceinline__ void stage_kv(float* Ks, float* Vs, const void* K, const void* V,
                                         long long base, int k0, int nkeys, int d) {
  for (int idx = threadIdx.x; idx < kChunk * d; idx += blockDim.x) {
    int j = idx / d, a = idx - j * d;
    int key = k0 + j;
    float kv = 0.f, vv = 0.f;
    if (key < nkeys) {
      kv = ld<BF16>(K, base + (long long)key * d + a);
      vv = ld<BF16>(V, base + (long long)key * d + a);
    }
    Ks[j * (d + 1) + a] = kv;
    Vs[j * d + a] = vv;
  }
}

template <bool BF16>
__global__ void __launch_bounds__(kWarps * 32) prefill_simt_kernel(PrefillArgs a) {
  extern __shared__ float smem[];
  const int d = a.d;
  float* Qs = smem;                       // [16][d]
  float* Rs = Qs + kRowsPerCta * d;       // [16][d]
  float* Ks = Rs + kRowsPerCta * d;       // [32][d+1]
  float* Vs = Ks + kChunk * (d + 1);      // [32][d]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = (a.N + kRowsPerCta - 1) / kRowsPerCta;
  const int bh = blockIdx.x / tiles;
  const int row0 = (blockIdx.x - bh * tiles) * kRowsPerCta;
  const long long base = (long long)bh * a.N * d;
  const float inv_sqrt_d = 1.f / sqrtf((float)d);

  for (int idx = threadIdx.x; idx < kRowsPerCta * d; idx += blockDim.x) {
    int r = idx / d, c = idx - r * d;
    int i = row0 + r;
    float qv = 0.f, rv = 0.f;
    if (i < a.N) {
      qv = ld<BF16>(a.Q, base + (long long)i * d + c);
      rv = ld<BF16>(a.R, base + (long long)i * d + c);
    }
    Qs[idx] = qv;
    Rs[idx] = rv;
  }
  RowState s[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) s[r].init();

  int last_row = min(row0 + kRowsPerCta, a.N) - 1;
  int kend = a.causal ? last_row + 1 : a.N;
  // With a sliding window the tile's first row sees keys from row0 - window + 1.
  const int kfirst = a.window > 0 ? max(0, row0 - a.window + 1) / kChunk * kChunk : 0;
  for (int k0 = kfirst; k0 < kend; k0 += kChunk) {
    __syncthreads();
    stage_kv<BF16>(Ks, Vs, a.K, a.V, base, k0, a.N, d);
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      int lr = warp + kWarps * r;
      int i = row0 + lr;
      if (i >= a.N) continue;
      if (a.causal && k0 > i) continue;
      if (a.window > 0 && k0 + kChunk <= i - a.window + 1) continue;
      int key = k0 + lane;
      bool valid = key < a.N && (!a.causal || key <= i) && (a.window <= 0 || key > i - a.window);
      row_update(s[r], Qs + lr * d, Rs + lr * d, Ks, Vs, d, valid, inv_sqrt_d, lane);
    }
  }
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    int i = row0 + warp + kWarps * r;
    if (i < a.N) row_finish<BF16>(s[r], a.out, base + (long long)i * d, d, lane);
  }
}

// One warp per (b, h): the decode query at position seqlens[b]-1.
template <bool BF16>
__global__ void __launch_bounds__(32) decode_simt_kernel(DecodeArgs a) {
  extern __shared__ float smem[];
  const int d = a.d;
  float* Qs = smem;            // [d]
  float* Rs = Qs + d;          // [d]
  float* Ks = Rs + d;          // [32][d+1]
  float* Vs = Ks + kChunk * (d + 1);
  const int lane = threadIdx.x;
  const int bh = blockIdx.x;
  const int b = bh / a.H;
  const int n = a.seqlens[b];
  const long long qoff = (long long)bh * d;
  if (n < 1 || n > a.L) {
    for (int c = lane; c < d; c += 32) st<BF16>(a.out, qoff + c, 0.f);
    if (lane == 0) atomicOr(a.status, kStatusBadSeqlen);
    return;
  }
  for (int c = lane; c < d; c += 32) {
    Qs[c] = ld<BF16>(a.q, qoff + c);
    Rs[c] = ld<BF16>(a.r, qoff + c);
  }
  const long long base = (long long)bh * a.L * d;
  const float inv_sqrt_d = 1.f / sqrtf((float)d);
  RowState s;
  s.init();
  const int lo = (a.window > 0 && n > a.window) ? n - a.window : 0;  // sliding window
  for (int k0 = lo / kChunk * kChunk; k0 < n; k0 += kChunk) {
    __syncwarp();
    stage_kv<BF16>(Ks, Vs, a.K, a.V, base, k0, n, d);
    __syncwarp();
    row_update(s, Qs, Rs, Ks, Vs, d, k0 + lane < n && k0 + lane >= lo, inv_sqrt_d, lane);
  }
  row_finish<BF16>(s, a.out, qoff, d, lane);
}

}  // namespace

cudaError_t launch_prefill_simt(const PrefillArgs& a, bool bf16, cudaStream_t st) {
  size_t smem = sizeof(float) * (2 * kRowsPerCta * a.d + kChunk * (a.d + 1) + kChunk * a.d);
  long long tiles = (a.N + kRowsPerCta - 1) / kRowsPerCta;
  dim3 grid((unsigned)(tiles * a.B * a.H));
  if (bf16) {
    cudaFuncSetAttribute(prefill_simt_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    prefill_simt_kernel<true><<<grid, kWarps * 32, smem, st>>>(a);
  } else {
    cudaFuncSetAttribute(prefill_simt_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    prefill_simt_kernel<false><<<grid, kWarps * 32, smem, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_decode_simt(const DecodeArgs& a, bool bf16, cudaStream_t st) {
  size_t smem = sizeof(float) * (2 * a.d + kChunk * (a.d + 1) + kChunk * a.d);
  dim3 grid((unsigned)(a.B * a.H));
  if (bf16) {
    cudaFuncSetAttribute(decode_simt_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    decode_simt_kernel<true><<<grid, 32, smem, st>>>(a);
  } else {
    cudaFuncSetAttribute(decode_simt_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    decode_simt_kernel<false><<<grid, 32, smem, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace plx
