// Split-KV Parallax decode for bf16 caches, d in {64, 128}, on warp-level
// MMAs, and the split plan.  At d = 128 the launcher hands sizes whose units
// carry enough keys (decode_bf16_tc) to the tcgen05 decode of
// decode_gqa_tc.cu, with one KV head per query head.
//
// One decode query per (b, h) is HBM-bound: every cached key and value is read
// once (8d flops per key against 4d bytes).  The kernel therefore optimises the
// stream, not the math:
//
// * Work unit = (b, h, key chunk).  Persistent CTAs of 4 warps take units
//   from a global counter (chunk-major, so full chunks first; the last CTA to
//   finish resets the counter); the warps of a CTA take the chunk's 16-key
//   blocks round-robin.
// * K and V are read straight from HBM with coalesced 16-byte non-allocating
//   loads into registers, one block ahead of the math (software pipeline), so
//   each warp keeps 8 KB in flight.
// * S1 = q.K^T and S2 = rho.K^T come out of ONE warp-level tensor-core MMA
//   whose A tile carries q in row 0 and rho in row 1 (the pages' packing of the
//   QK and RK products into one MMA; agihunt.info summary, decode paragraph).
//   O1 and O2 come out of one MMA as well: V^T times [w ; w t] gives O1 and O2
//   as columns of one accumulator (each weight split into a bf16 hi + lo pair
//   that fills two of the MMA's otherwise idle columns).  The contraction dims and the key
//   order inside a block are permuted consistently on both operands, so the
//   16-byte vectors as loaded ARE the MMA fragments (V needs one byte-permute
//   per two elements to pair keys); no shared-memory transpose is needed.
// * One running max per warp, updated lazily: the max is raised only when a
//   block's max exceeds it by more than 2^8, which is exact because omega, T,
//   O1 and O2 are always scaled by the same factor.
// * Partial state (m, omega, T, O1, O2) is merged across the 4 warps in shared
//   memory, and across the chunks of one (b, h) by the last CTA to finish that
//   (b, h), found with an atomic arrival counter (no spin-waits); it resets the
//   counter for the next call ("persistent KV-loop split" and "in-kernel
//   reduction", rainbus.top reproduction notes).
//
// Formulas: rainbus.top summary "方法步骤详情" and the covariance form of the
// gist.science summary; out = ((1 + T/omega) O1 - O2) / omega.
#include "plx_internal.cuh"

#include <math_constants.h>

namespace plx {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr float kLazyTau = 8.f;  // log2 units: raise the max only when it grows by > 2^8

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t word(const uint4& v, int w) {
  return w == 0 ? v.x : (w == 1 ? v.y : (w == 2 ? v.z : v.w));
}

// Pair element `e` (0..7) of two 8-element bf16 vectors: low half from x, high from y.
__device__ __forceinline__ uint32_t pair(const uint4& x, const uint4& y, int e) {
  return __byte_perm(word(x, e >> 1), word(y, e >> 1), (e & 1) ? 0x7632 : 0x5410);
}

template <int D>
struct Frag {
  static constexpr int KLD = D / 32;  // 16-byte K loads per key per thread (4 threads per key)
  static constexpr int VLD = D / 64;  // 16-byte V loads per key per thread (8 threads per key)
  uint4 k[2][KLD];                    // [n-tile][load]
  uint4 v[4][VLD];                    // [key 4t+e][load]
};

// Lane (g = lane/4, t = lane%4).  S-MMA n-tile nt, column n holds key
// sigma_nt(n) = 2n - (n&1) + 2nt of the block, so the accumulator of lane (0,t)
// ends up holding keys 4t..4t+3 -- exactly the keys lane t supplies to the
// value MMA, whose k index 2t+e maps to key 4t+e and 2t+8+e to key 4t+2+e.
template <int D>
__device__ __forceinline__ void load_block(Frag<D>& f, const __nv_bfloat16* Kbh,
                                           const __nv_bfloat16* Vbh, int j0, int kend, int g,
                                           int t) {
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    int key = min(j0 + 2 * g - (g & 1) + 2 * nt, kend - 1);
    const __nv_bfloat16* row = Kbh + (long long)key * D + 8 * t;
#pragma unroll
    for (int i = 0; i < Frag<D>::KLD; ++i) f.k[nt][i] = ld_stream(row + 32 * i);
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    int key = min(j0 + 4 * t + e, kend - 1);
    const __nv_bfloat16* row = Vbh + (long long)key * D + 8 * g;
#pragma unroll
    for (int i = 0; i < Frag<D>::VLD; ++i) f.v[e][i] = ld_stream(row + 64 * i);
  }
}

template <int D>
struct WarpState {
  static constexpr int MT = D / 16;
  float O[MT][4];  // value-MMA accumulators: rows = dims, columns (0+1) = O1, (2+3) = O2
  float m;         // running max (log2 domain), warp-uniform
  float omega, T;  // partial sums held by lanes 0..3
};

template <int D>
__device__ __forceinline__ void compute_block(WarpState<D>& s, const Frag<D>& f,
                                              const uint32_t (&aq)[D / 16][2], int j0, int kend,
                                              int lane, float c_log2) {
  constexpr int KS = D / 16;
  const int g = lane >> 2, t = lane & 3;
  // ---- S = [q ; rho ; 0] x K^T, two n-tiles of 8 keys.
  float S[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    S[nt][0] = S[nt][1] = S[nt][2] = S[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const uint4& kv = f.k[nt][ks >> 1];
      uint32_t b0 = (ks & 1) ? kv.z : kv.x;
      uint32_t b1 = (ks & 1) ? kv.w : kv.y;
      mma_bf16(S[nt], aq[ks][0], 0u, aq[ks][1], 0u, b0, b1);
    }
  }
  // Lane t holds s1 (row 0) and lane 4+t holds s2 (row 1) of keys 4t..4t+3;
  // every lane fetches both for its own t.
  float s1[4], s2[4];
  float mloc = -CUDART_INF_F;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float own = (e < 2) ? S[0][e] : S[1][e - 2];
    float a = __shfl_sync(0xffffffffu, own, t);
    s2[e] = __shfl_sync(0xffffffffu, own, 4 + t);
    bool valid = j0 + 4 * t + e < kend;
    s1[e] = valid ? a * c_log2 : -CUDART_INF_F;
    mloc = fmaxf(mloc, s1[e]);
  }
  mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
  const float mblk = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));  // same in every lane
  if (mblk > s.m + kLazyTau) {  // warp-uniform; also taken on the first block (m = -inf)
    const float alpha = exp2f(s.m - mblk);
#pragma unroll
    for (int mt = 0; mt < WarpState<D>::MT; ++mt) {
#pragma unroll
      for (int r = 0; r < 4; ++r) s.O[mt][r] *= alpha;
    }
    s.omega *= alpha;
    s.T *= alpha;
    s.m = mblk;
  }
  float w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) w[e] = exp2f(s1[e] - s.m);
  if (g == 0) {
    s.omega += (w[0] + w[1]) + (w[2] + w[3]);
    s.T += (w[0] * s2[0] + w[1] * s2[1]) + (w[2] * s2[2] + w[3] * s2[3]);
  }
  // ---- [O1 O2] += V^T x [w_hi, w_lo, wt_hi, wt_lo]: column n comes from lanes
  // with g = n.  Each weight travels as a bf16 pair hi + lo (lo = the bf16 of
  // the remainder), so the products carry ~16 mantissa bits: the combine
  // (1 + tbar) O1 - O2 cancels by up to |t| on queries with few keys, and a
  // single bf16 rounding of w t would show through it.
  uint32_t b0 = 0u, b1 = 0u;
  if (g < 4) {
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float v = (g < 2) ? w[e] : w[e] * s2[e];
      if (g & 1) v -= __bfloat162float(__float2bfloat16_rn(v));
      x[e] = v;
    }
    b0 = pack_bf16(x[0], x[1]);
    b1 = pack_bf16(x[2], x[3]);
  }
#pragma unroll
  for (int mt = 0; mt < WarpState<D>::MT; ++mt) {
    // Rows g and g+8 of m-tile mt are dims 8g+mt and (D==128 ? 64+8g+mt : 8g+4+mt).
    uint32_t a0, a1, a2, a3;
    if constexpr (D == 128) {
      a0 = pair(f.v[0][0], f.v[1][0], mt);
      a1 = pair(f.v[0][1], f.v[1][1], mt);
      a2 = pair(f.v[2][0], f.v[3][0], mt);
      a3 = pair(f.v[2][1], f.v[3][1], mt);
    } else {
      a0 = pair(f.v[0][0], f.v[1][0], mt);
      a1 = pair(f.v[0][0], f.v[1][0], mt + 4);
      a2 = pair(f.v[2][0], f.v[3][0], mt);
      a3 = pair(f.v[2][0], f.v[3][0], mt + 4);
    }
    mma_bf16(s.O[mt], a0, a1, a2, a3, b0, b1);
  }
}

template <int D>
__device__ __forceinline__ int dim_row(int g, int mt, int half) {
  if constexpr (D == 128) return half ? 64 + 8 * g + mt : 8 * g + mt;
  return half ? 8 * g + 4 + mt : 8 * g + mt;
}

template <int D>
struct Smem {
  float O1[kWarps][D];
  float O2[kWarps][D];
  float m[kWarps], omega[kWarps], T[kWarps];
  int last;
  long long unit;
};

// Dynamic unit scheduler: the next unit to hand out and the number of CTAs
// that finished; the last CTA of a launch resets both for the next launch.
__device__ unsigned long long g_unit_next;
__device__ unsigned int g_cta_done;

template <int D>
__global__ void __launch_bounds__(kThreads) decode_bf16_kernel(DecodeArgs a) {
  __shared__ Smem<D> sm;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int BH = a.B * a.H;
  const long long units = (long long)BH * a.splits;
  const float c_log2 = 1.4426950408889634f / sqrtf((float)D);
  const __nv_bfloat16* Kall = reinterpret_cast<const __nv_bfloat16*>(a.K);
  const __nv_bfloat16* Vall = reinterpret_cast<const __nv_bfloat16*>(a.V);
  const __nv_bfloat16* qall = reinterpret_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* rall = reinterpret_cast<const __nv_bfloat16*>(a.r);
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);

  // Units in chunk-major order (every sequence's first chunk, then the second,
  // ...), so that the full-length chunks go first.  Each CTA starts with unit
  // blockIdx.x; further units come from a global counter, fetched at the start
  // of the current unit so that the atomic's latency hides behind its stream.
  long long u = blockIdx.x;
  while (u < units) {
    long long next = 0;
    if (threadIdx.x == 0) next = (long long)gridDim.x + (long long)atomicAdd(&g_unit_next, 1ull);
    do {  // one unit; `break` leaves it early
    const int c = (int)(u / BH);
    const int bh = (int)(u - (long long)c * BH);
    const int b = bh / a.H;
    const int n = a.seqlens[b];
    if (n < 1 || n > a.L) {
      if (c == 0) {
        for (int x = threadIdx.x; x < D; x += kThreads) out[(long long)bh * D + x] = __float2bfloat16(0.f);
        if (threadIdx.x == 0) atomicOr(a.status, kStatusBadSeqlen);
      }
      break;
    }
    // Keys lo..n-1 (lo > 0 only with a sliding window), cut into chunks.
    const int lo = a.window > 0 ? max(0, n - a.window) : 0;
    const int nch = (n - lo + a.chunk - 1) / a.chunk;
    if (c >= nch) break;
    const int kbeg = lo + c * a.chunk;
    const int kend = min(kbeg + a.chunk, n);

    // A fragments of [q ; rho]: row g (0 = q, 1 = rho), contraction dims of
    // k-step ks = 2i + hh are 32i + 8t + 4hh + {0,1} and + {2,3}.
    uint32_t aq[D / 16][2];
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      aq[ks][0] = aq[ks][1] = 0u;
      if (g < 2) {
        const __nv_bfloat16* src = (g == 0 ? qall : rall) + (long long)bh * D + 32 * (ks >> 1) +
                                   8 * t + 4 * (ks & 1);
        uint2 v = *reinterpret_cast<const uint2*>(src);
        aq[ks][0] = v.x;
        aq[ks][1] = v.y;
      }
    }

    WarpState<D> s;
#pragma unroll
    for (int mt = 0; mt < WarpState<D>::MT; ++mt) s.O[mt][0] = s.O[mt][1] = s.O[mt][2] = s.O[mt][3] = 0.f;
    s.m = -CUDART_INF_F;
    s.omega = 0.f;
    s.T = 0.f;

    const __nv_bfloat16* Kbh = Kall + (long long)bh * a.L * D;
    const __nv_bfloat16* Vbh = Vall + (long long)bh * a.L * D;
    const int stride = 16 * kWarps;
    int j0 = kbeg + 16 * warp;
    if (j0 < kend) {
      Frag<D> fa, fb;
      load_block<D>(fa, Kbh, Vbh, j0, kend, g, t);
      while (true) {
        int j1 = j0 + stride;
        bool has1 = j1 < kend;
        if (has1) load_block<D>(fb, Kbh, Vbh, j1, kend, g, t);
        compute_block<D>(s, fa, aq, j0, kend, lane, c_log2);
        if (!has1) break;
        j0 = j1 + stride;
        bool has0 = j0 < kend;
        if (has0) load_block<D>(fa, Kbh, Vbh, j0, kend, g, t);
        compute_block<D>(s, fb, aq, j1, kend, lane, c_log2);
        if (!has0) break;
      }
    }
    // ---- Warp partials to shared memory.
    s.omega += __shfl_xor_sync(0xffffffffu, s.omega, 1);
    s.omega += __shfl_xor_sync(0xffffffffu, s.omega, 2);
    s.T += __shfl_xor_sync(0xffffffffu, s.T, 1);
    s.T += __shfl_xor_sync(0xffffffffu, s.T, 2);
    if (lane == 0) {
      sm.m[warp] = s.m;
      sm.omega[warp] = s.omega;
      sm.T[warp] = s.T;
    }
    if (t < 2) {  // lane t = 0 holds columns 0, 1 (O1 hi + lo); t = 1 holds 2, 3 (O2)
      float* dst = (t == 0) ? sm.O1[warp] : sm.O2[warp];
#pragma unroll
      for (int mt = 0; mt < WarpState<D>::MT; ++mt) {
        dst[dim_row<D>(g, mt, 0)] = s.O[mt][0] + s.O[mt][1];
        dst[dim_row<D>(g, mt, 1)] = s.O[mt][2] + s.O[mt][3];
      }
    }
    __syncthreads();
    // ---- Merge the warps (thread x owns dim x).
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm.m[w]);
    float omega = 0.f, T = 0.f, o1 = 0.f, o2 = 0.f;
    const int x = threadIdx.x;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      float sc = (sm.m[w] == -CUDART_INF_F) ? 0.f : exp2f(sm.m[w] - M);
      omega += sc * sm.omega[w];
      T += sc * sm.T[w];
      if (x < D) {
        o1 += sc * sm.O1[w][x];
        o2 += sc * sm.O2[w][x];
      }
    }
    if (nch == 1) {
      if (x < D) {
        float inv = 1.f / omega;
        out[(long long)bh * D + x] = __float2bfloat16_rn(((1.f + T * inv) * o1 - o2) * inv);
      }
      break;
    }
    // ---- Publish this chunk's partial; the last chunk of (b, h) merges all.
    float* rec = a.partials + ((long long)bh * a.splits + c) * (2 * D + 4);
    if (x == 0) {
      rec[0] = M;
      rec[1] = omega;
      rec[2] = T;
    }
    if (x < D) {
      rec[4 + x] = o1;
      rec[4 + D + x] = o2;
    }
    __threadfence();
    __syncthreads();
    if (x == 0) sm.last = (atomicAdd(a.counters + bh, 1) == nch - 1);
    __syncthreads();
    if (sm.last) {
      __threadfence();
      const float* base = a.partials + (long long)bh * a.splits * (2 * D + 4);
      float Mg = -CUDART_INF_F;
      // Several chunks' loads in flight per round trip.
#pragma unroll 4
      for (int cc = 0; cc < nch; ++cc) Mg = fmaxf(Mg, __ldcg(base + (long long)cc * (2 * D + 4)));
      float om = 0.f, TT = 0.f, p1 = 0.f, p2 = 0.f;
#pragma unroll 4
      for (int cc = 0; cc < nch; ++cc) {
        const float* r = base + (long long)cc * (2 * D + 4);
        float mc = __ldcg(r);
        float sc = (mc == -CUDART_INF_F) ? 0.f : exp2f(mc - Mg);
        om += sc * __ldcg(r + 1);
        TT += sc * __ldcg(r + 2);
        if (x < D) {
          p1 += sc * __ldcg(r + 4 + x);
          p2 += sc * __ldcg(r + 4 + D + x);
        }
      }
      if (x < D) {
        float inv = 1.f / om;
        out[(long long)bh * D + x] = __float2bfloat16_rn(((1.f + TT * inv) * p1 - p2) * inv);
      }
      if (x == 0) a.counters[bh] = 0;
    }
    } while (false);
    __syncthreads();  // shared memory and sm.unit are reused by the next unit
    if (threadIdx.x == 0) sm.unit = next;
    __syncthreads();
    u = sm.unit;
  }
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&g_cta_done, 1u) == gridDim.x - 1) {
      atomicExch(&g_unit_next, 0ull);
      atomicExch(&g_cta_done, 0u);
    }
  }
}

}  // namespace

// Keys per (b, h) are cut into `splits` chunks.  Fewer, longer chunks stream
// better (each unit pays a fixed start-up and merge), but the last wave of
// units should be nearly full: take the fewest splits whose waves over the
// resident CTAs are at least 97 % used, with chunks of at least 256 keys.
void decode_split_plan(int B, int H, int L, int num_sms, int* splits, int* chunk, int ctas_per_sm) {
  const double bh = (double)B * H;
  const double resident = (double)num_sms * ctas_per_sm;  // CTAs the launcher keeps per SM
  long long smax = L / 256;
  if (smax < 1) smax = 1;
  if (smax > 256) smax = 256;
  long long best = 1;
  double best_eff = -1.0;
  for (long long S = 1; S <= smax; ++S) {
    const double waves = bh * (double)S / resident;
    const double eff = waves / ceil(waves);
    if (eff > best_eff + 0.02) {
      best_eff = eff;
      best = S;
    }
    if (eff >= 0.97) break;
  }
  long long c = (L + best - 1) / best;
  c = (c + 63) / 64 * 64;
  *chunk = (int)c;
  *splits = (int)((L + c - 1) / c);
}

cudaError_t launch_decode_bf16(const DecodeArgs& a, cudaStream_t st, int num_sms) {
  const int keys = (a.window > 0 && a.window < a.L) ? a.window : a.L;
  if (decode_bf16_tc_h(a.B, a.H, keys, a.d)) {  // the tensor-core decode, Hkv = H
    DecodeArgs g = a;
    g.Hkv = a.H;
    return launch_decode_gqa_tc(g, st, num_sms);
  }
  long long units = (long long)a.B * a.H * a.splits;
  int per_sm = 0;
  cudaError_t e;
  if (a.d == 128) {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_bf16_kernel<128>, kThreads, 0);
  } else {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_bf16_kernel<64>, kThreads, 0);
  }
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  long long grid = (long long)num_sms * per_sm;
  if (grid > units) grid = units;
  if (a.d == 128) {
    decode_bf16_kernel<128><<<(unsigned)grid, kThreads, 0, st>>>(a);
  } else {
    decode_bf16_kernel<64><<<(unsigned)grid, kThreads, 0, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace plx
