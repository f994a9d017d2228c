// Backward pass of causal (or full) Parallax prefill, bf16, d in {64, 128}, on
// sm_100a tensor cores (tcgen05 MMAs, TMA loads, TMEM accumulators).
//
// The forward output of query i is a weighted sum of values,
//   out_i = sum_j a_ij v_j,   a_ij = p_ij (1 - t_ij + tbar_i),
// with p_ij = softmax_j(q_i . k_j / sqrt(d)), t_ij = rho_i . k_j and
// tbar_i = sum_j p_ij t_ij (the covariance correction of "Parallax:
// Parameterized Local Linear Attention for Language Modeling", gist.science
// summary "Mecanismo central", written out per key; the rainbus.top summary's
// six-step forward has the same weights).  The pages train the layer end to
// end but print no backward pass; its gradients follow from that expression.
// With dO_i the output gradient, dA_ij = dO_i . v_j, u_ij = 1 - t_ij + tbar_i,
//   D_i = dO_i . vbar_i  (= sum_j p_ij dA_ij),   F_i = dO_i . out_i,
//   dV_j  = sum_i a_ij dO_i,
//   dt_ij = p_ij (D_i - dA_ij)                   -> dR_i = sum_j dt_ij k_j,
//   dl_ij = p_ij (u_ij (dA_ij - D_i) + D_i - F_i) (gradient of the logit),
//   dQ_i  = sum_j dl_ij k_j / sqrt(d),   dK_j = sum_i dl_ij q_i / sqrt(d) + dt_ij rho_i.
// Only centred quantities (u, dA - D, D - F) enter, so a large mean probe score
// costs no precision.
//
// Three launches:
//  1. prep: per query row, the statistics (-lse in log2 units, 1 + tbar, D,
//     F - D) from the forward's saved lse, tbar, vbar (fp32: D from a bf16
//     vbar would carry its rounding into every dt and dl of the row) and out,
//     into a per-head padded workspace (padding rows give p = 0), laid out
//     by 64-row blocks as four arrays of 64 floats (one 1 KB copy per block).
//  2. dK/dV: one CTA per 128-key block of a head.  K and V stay in shared
//     memory; 64-query blocks stream through a three-stage ring (Q and R
//     stacked as one 128-row operand, and dO).  Per block:
//       [S^T | T^T] = K [Q; R]^T   (one N = 128 MMA: keys are M, so Q and R
//                                   share it as the B operand)
//       dA^T        = V dO^T
//     the elementwise warps turn the scores into a^T (bf16, shared memory,
//     K-major) and dl^T/sqrt(d), dt^T (bf16 pairs in TMEM), then
//       dV += a^T dO,   dK += [dl^T | dt^T] [Q; R]   (one K = 128 MMA, A in TMEM)
//     accumulate in TMEM for the whole key block.  A stage is held until the
//     block's gradient MMAs complete, so the third stage lets the loads of
//     block i + 2 overlap block i's elementwise step and gradient MMAs.
//  3. dQ/dR: one CTA per 128-query block; 64-key blocks stream through a
//     three-stage ring.  Per block S = Q K^T, T = R K^T, dA = dO V^T; the
//     elementwise warps write dl/sqrt(d) and dt as bf16 into TMEM, and
//       dQ += dl K,   dR += dt K
//     accumulate in TMEM (A operands from TMEM).
// Splitting dQ/dR from dK/dV recomputes the scores once more (11 MMA tiles
// per score tile instead of 8) but needs no cross-CTA reduction: every
// gradient is written once, in bf16, with no atomics and no fp32 workspace.
//
// Warp roles in both kernels: warp 0 TMA producer, warp 1 TMEM owner and MMA
// issuer (one elected thread), warps 4..19 four elementwise warpgroups that
// split each block's columns (every TMEM lane is read by one warp of each).
// Every wait is bounded in time; one that runs out sets the device status
// word and the CTA's abort flag, and every role unwinds.
#include "sm100.cuh"

#include <math_constants.h>

#include <cstdlib>
#include <cstring>

namespace plx {
namespace {

using namespace sm100;

// Four elementwise warpgroups, each taking 16 of a block's 64 columns for every
// TMEM lane: the per-pair arithmetic is latency-bound, so more warps per
// scheduler hide more of it.
constexpr int kEwGroups = 4;
constexpr int kEwCols = 64 / kEwGroups;  // columns per elementwise thread
constexpr int kThreads = 128 * (1 + kEwGroups);
constexpr int kFirstEwWarp = 4;
constexpr float kLog2e = 1.4426950408889634f;

// Instruction descriptor (kind::f16): D f32, A and B bf16, M = 128, N = n;
// b_mn = 1 when B is MN-major (A is always K-major here).
__host__ __device__ constexpr uint32_t idesc(int n, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn << 16) | ((uint32_t)(n >> 3) << 17) |
         ((128u >> 4) << 24);
}

// Byte offset of the 16-byte chunk `chunk` of row `row` in a 128B-swizzled
// tile of 128-byte rows (the layout TMA writes and the MMA descriptors read).
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// ---------------------------------------------------------------------------
// 1. Per-row statistics.
// ---------------------------------------------------------------------------

// Float index of statistic k (0..3) of row i of head bh: 64-row blocks of
// four 64-float arrays.
__host__ __device__ __forceinline__ size_t stat_index(int bh, int Npad, int i, int k) {
  return ((size_t)bh * (Npad / 64) + (size_t)(i / 64)) * 256 + (size_t)k * 64 + (size_t)(i % 64);
}

// Statistics of row i: (-lse_i log2(e), 1 + tbar_i, D_i, F_i - D_i) for i < N;
// (-inf, 1, 0, 0) for the padding rows i in [N, Npad).  One warp per row.
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ out,
                                                       const float* __restrict__ vbar,
                                                       const __nv_bfloat16* __restrict__ dO,
                                                       const float* __restrict__ lse,
                                                       const float* __restrict__ tbar,
                                                       float* __restrict__ stats, int BH, int N, int Npad,
                                                       int d) {
  const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= (long long)BH * Npad) return;
  const int bh = (int)(r / Npad), i = (int)(r % Npad);
  if (i >= N) {
    if (lane < 4) stats[stat_index(bh, Npad, i, lane)] = lane == 0 ? -CUDART_INF_F : (lane == 1 ? 1.f : 0.f);
    return;
  }
  const long long g = (long long)bh * N + i;
  float dv = 0.f, df = 0.f;
  for (int c = 2 * lane; c < d; c += 64) {
    const float2 go = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dO + g * d + c));
    const float2 vb = *reinterpret_cast<const float2*>(vbar + g * d + c);
    const float2 o = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(out + g * d + c));
    dv = fmaf(go.x, vb.x, fmaf(go.y, vb.y, dv));
    df = fmaf(go.x, o.x, fmaf(go.y, o.y, df));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    dv += __shfl_xor_sync(0xffffffffu, dv, o);
    df += __shfl_xor_sync(0xffffffffu, df, o);
  }
  const float v = lane == 0 ? -lse[g] * kLog2e : (lane == 1 ? 1.f + tbar[g] : (lane == 2 ? dv : df - dv));
  if (lane < 4) stats[stat_index(bh, Npad, i, lane)] = v;
}

struct BwdParams {
  int B, H, N, Npad, causal;
  int Hkv;           // KV heads (H a multiple of it): query head h read KV head h / (H / Hkv)
  int window;        // sliding window (0: none): query i saw keys i - window + 1 .. i
  int inject_stall;  // failure-detection test: CTA 0 of the dK/dV kernel never loads its K/V
  int chunk_heads;  // heads whose blocks are launched together (L2 reuse of their tiles)
  const float* stats;
  __nv_bfloat16* g0;  // dV (key-block kernel) or dQ (query-block kernel)
  __nv_bfloat16* g1;  // dK or dR
  int* status;
};

// Block t of the launch order: heads in chunks of `ch`, and within a chunk the
// blocks with the most causal work first (rank 0 = most), across the chunk's
// heads.  Blocks start roughly in index order, so the few heads whose blocks
// run at one time keep their streamed tiles in L2 for all of those blocks.
struct BlockOrder {
  int bh, rank;
};
__device__ __forceinline__ BlockOrder block_order(int t, int BH, int nblk, int ch) {
  const int per_chunk = ch * nblk;
  const int chunk = t / per_chunk;
  const int nh = min(ch, BH - chunk * ch);
  const int pos = t - chunk * per_chunk;
  BlockOrder o;
  o.rank = pos / nh;
  o.bh = chunk * ch + pos % nh;
  return o;
}

// Bounded wait taken by a whole warp: every lane leaves with the same answer,
// so the warp-collective TMEM accesses that follow are reached by all or none.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* status) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, status));
}

// Elementwise step shared by both kernels, for two neighbouring (query, key)
// pairs at once in packed f32x2 arithmetic: raw scores s = q . k, probe scores
// t, dA = dO . v, and the pairs' statistics nl = -lse log2 e, c0 = 1 + tbar,
// dd = D, fd = F - D; keep0/keep1 clear masked pairs.  With p the softmax
// weight, u = c0 - t and x = D - dA, it packs bf16 pairs of
//   a = p u,   dt = p x,   dl = p (D - F - u x) / sqrt(d) = p (u (dA - D) + D - F) / sqrt(d).
struct GradPairs {
  uint32_t a, dt, dl;
};
__device__ __forceinline__ uint32_t pack2(uint64_t v) {
  float lo, hi;
  uf2(v, lo, hi);
  return pack_bf16(lo, hi);
}
__device__ __forceinline__ GradPairs grad_pairs(uint32_t s0, uint32_t s1, uint32_t t0, uint32_t t1, uint32_t a0,
                                                uint32_t a1, uint64_t nl, uint64_t c0, uint64_t dd, uint64_t fd,
                                                uint64_t sc2, uint64_t nisd2, bool keep0, bool keep1) {
  const uint64_t m1 = f2(-1.f, -1.f);
  float e0, e1;
  uf2(fma2(f2(__uint_as_float(s0), __uint_as_float(s1)), sc2, nl), e0, e1);
  float p0 = ex2(e0), p1 = ex2(e1);
  p0 = keep0 ? p0 : 0.f;
  p1 = keep1 ? p1 : 0.f;
  const uint64_t p2 = f2(p0, p1);
  const uint64_t u2 = fma2(f2(__uint_as_float(t0), __uint_as_float(t1)), m1, c0);
  const uint64_t x2 = fma2(f2(__uint_as_float(a0), __uint_as_float(a1)), m1, dd);
  GradPairs g;
  g.a = pack2(mul2(p2, u2));
  g.dt = pack2(mul2(p2, x2));
  // u x - (D - F) = u x + fd; times -p / sqrt(d).
  g.dl = pack2(mul2(mul2(p2, nisd2), fma2(u2, x2, fd)));
  return g;
}

// Writes 8 * NC bf16 values (4 * NC packed pairs) as 16-byte chunks
// c0..c0+NC-1 of a 128B-swizzled row.
template <int NC>
__device__ __forceinline__ void st_row_chunks(uint8_t* tile, int row, int c0, const uint32_t (&v)[4 * NC]) {
#pragma unroll
  for (int j = 0; j < NC; ++j)
    *reinterpret_cast<uint4*>(tile + sw128(row, c0 + j)) = make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
}

// 8 consecutive TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]));
}

// Loads NC fp32 TMEM columns of this thread's lane from `taddr` and stores
// them as bf16 at dst (nullptr: load only, every lane takes part).
template <int NC>
__device__ __forceinline__ void tmem_row_to_global(uint32_t taddr, __nv_bfloat16* dst) {
#pragma unroll 1
  for (int c0 = 0; c0 < NC; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(taddr + c0, v);
    tc_wait_ld();
    if (dst != nullptr) {
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) pk[c] = pack_bf16(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1]));
      uint4* o = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
      for (int c = 0; c < 4; ++c) o[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
    }
  }
}

// ---------------------------------------------------------------------------
// 2. dK and dV: one CTA per 128-key block of a head.
// ---------------------------------------------------------------------------
constexpr int kKB = 128;  // keys per CTA (MMA M)
constexpr int kQB = 64;   // queries per streamed block
constexpr int kQStages = 3;

template <int D>
struct KvSmem {
  static constexpr int kHalves = D / 64;
  // 128B-swizzled tiles, every one 1024-byte aligned; a "half" is 64 dims.
  uint8_t k[kHalves][kKB * 128];
  uint8_t v[kHalves][kKB * 128];
  uint8_t qr[kQStages][kHalves][2 * kQB * 128];  // per half: Q rows 0..63, then R rows 0..63
  uint8_t dout[kQStages][kHalves][kQB * 128];
  uint8_t a[kKB * 128];  // a^T [128 keys][64 queries] bf16, K-major
  uint64_t kv_full, q_full[kQStages], q_empty[kQStages];
  uint64_t s_full, s_free, p_full, ag_free, done, drain, drain_g;
  uint32_t tmem_base;
  int abort;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmR,
                   const __grid_constant__ CUtensorMap tmdO, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, BwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  using Sm = KvSmem<D>;
  constexpr int kHalves = D / 64;
  // TMEM columns: dV and dK accumulators, the score stage, then the bf16
  // pairs of dl^T / sqrt(d) (32 columns) and dt^T (32): the A operand of dK.
  constexpr uint32_t kColDV = 0, kColDK = D, kColS = 2 * D, kColT = 2 * D + 64, kColDA = 2 * D + 128,
                     kColG = 2 * D + 192;
  Sm& sm = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // One CTA per key block of a KV head (bh indexes KV heads); its gradients
  // sum over the query blocks of every query head of the head's group, taken
  // head by head: step i is query block q0 + i % nq1 of group member i / nq1.
  const int G = p.H / p.Hkv;
  const BlockOrder bo = block_order(blockIdx.x, p.B * p.Hkv, (p.N + kKB - 1) / kKB, p.chunk_heads);
  const int kb = bo.rank, bh = bo.bh;
  const int qbh0 = (bh / p.Hkv) * p.H + (bh % p.Hkv) * G;  // first query head of the group
  const int nqb = (p.N + kQB - 1) / kQB;
  const int q0 = p.causal ? (kb * kKB) / kQB : 0;
  // With a window, the block's last key is seen by queries up to kb kKB + kKB - 1 + window - 1.
  const int qend = p.window > 0 ? min(nqb, (kb * kKB + kKB + p.window - 2) / kQB + 1) : nqb;
  const int nq1 = qend - q0;  // >= 1: key block kb starts below N
  const int nq = G * nq1;
  volatile int* abort = &sm.abort;

  if (threadIdx.x == 0) {
    mbar_init(&sm.kv_full, 1);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&sm.q_full[s], 1);
      mbar_init(&sm.q_empty[s], 1);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.s_free, 4 * kEwGroups);    // lane 0 of each elementwise warp
    mbar_init(&sm.p_full, 128 * kEwGroups);  // every elementwise thread
    mbar_init(&sm.ag_free, 1);
    mbar_init(&sm.done, 1);
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.drain_g, 1);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&sm.tmem_base)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const int krow = bh * p.N + kb * kKB;
      // The failure-detection test withholds CTA 0's K/V: the score issuer's
      // bounded wait runs out and every role unwinds through the abort path.
      if (!(p.inject_stall && blockIdx.x == 0)) {
        mbar_expect_tx(&sm.kv_full, 2 * kKB * D * 2);
        for (int h = 0; h < kHalves; ++h) {
          tma_load_2d(sm.k[h], &tmK, &sm.kv_full, 64 * h, krow);
          tma_load_2d(sm.v[h], &tmV, &sm.kv_full, 64 * h, krow);
        }
      }
      int last_use[kQStages] = {-1, -1, -1};
      int qh = qbh0, qb = q0;  // query head and block of step i
      for (int i = 0; i < nq && !*abort; ++i, qb = qb + 1 < qend ? qb + 1 : (++qh, q0)) {
        const int st = i % kQStages, u = i / kQStages;
        if (u > 0 && !mbar_wait(&sm.q_empty[st], (u - 1) & 1, abort, p.status)) break;
        mbar_expect_tx(&sm.q_full[st], 3 * kQB * D * 2);
        last_use[st] = u;
        const int qrow = qh * p.N + qb * kQB;
        for (int h = 0; h < kHalves; ++h) {
          tma_load_2d(sm.qr[st][h], &tmQ, &sm.q_full[st], 64 * h, qrow);
          tma_load_2d(sm.qr[st][h] + kQB * 128, &tmR, &sm.q_full[st], 64 * h, qrow);
          tma_load_2d(sm.dout[st][h], &tmdO, &sm.q_full[st], 64 * h, qrow);
        }
        // The block's statistics (1 KB, read by every elementwise thread)
        // into L1 ahead of use.
        const float* stp = p.stats + stat_index(qh, p.Npad, qb * kQB, 0);
#pragma unroll
        for (int l = 0; l < 8; ++l) asm volatile("prefetch.global.L1 [%0];" ::"l"(stp + 32 * l));
      }
      if (*abort) {  // let every copy issued here land before the CTA exits
        mbar_drain(&sm.kv_full, 0);
        for (int s = 0; s < kQStages; ++s)
          if (last_use[s] >= 0) mbar_drain(&sm.q_full[s], (uint32_t)(last_use[s] & 1));
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ---------------- MMA issuers ----------------
    // Warp 1 issues the scores of every block, warp 2 its gradient MMAs: an
    // issue returns only once the tensor pipe has taken the MMA, so one
    // thread for both would hold the gradients of block i behind the scores
    // of block i + 1 (and those behind the wait for block i + 1's operands).
    if (lane == 0) {
      const uint64_t aK = sdesc(smem_u32(sm.k[0]), 16, 1024), aV = sdesc(smem_u32(sm.v[0]), 16, 1024);
      const uint64_t aA = sdesc(smem_u32(sm.a), 16, 1024);
      auto issue_grads = [&](int b) {
        const int st = b % kQStages;
        // dO and [Q; R] as MN-major B operands: 64-dim halves apart by LBO,
        // 8-row groups by 1024 bytes, 16 rows (one K step) by 2048.
        const uint64_t bdo = sdesc(smem_u32(sm.dout[st][0]), kQB * 128, 1024);
        const uint64_t bqr = sdesc(smem_u32(sm.qr[st][0]), 2 * kQB * 128, 1024);
#pragma unroll
        for (int ks = 0; ks < kQB / 16; ++ks)
          mma_ss(tmem + kColDV, aA + (uint64_t)((ks * 32) >> 4), bdo + (uint64_t)((ks * 2048) >> 4), idesc(D, 1),
                 (b > 0 || ks > 0) ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < 2 * kQB / 16; ++ks)
          mma_ts(tmem + kColDK, tmem + kColG + ks * 8, bqr + (uint64_t)((ks * 2048) >> 4), idesc(D, 1),
                 (b > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&sm.ag_free);
        mma_commit(&sm.q_empty[st]);
      };
      if (warp == 1) {
        bool ok = mbar_wait(&sm.kv_full, 0, abort, p.status);
        for (int i = 0; ok && i < nq; ++i) {
          const int st = i % kQStages;
          if (!(ok = mbar_wait(&sm.q_full[st], (i / kQStages) & 1, abort, p.status))) break;
          if (i > 0 && !(ok = mbar_wait(&sm.s_free, (i - 1) & 1, abort, p.status))) break;
          tc_fence_after();
          const uint64_t bqr = sdesc(smem_u32(sm.qr[st][0]), 16, 1024);
          const uint64_t bdo = sdesc(smem_u32(sm.dout[st][0]), 16, 1024);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t ka = (ks >> 2) * (kKB * 128) + (ks & 3) * 32;
            mma_ss(tmem + kColS, aK + (uint64_t)(ka >> 4),
                   bqr + (uint64_t)((((ks >> 2) * 2 * kQB * 128) + (ks & 3) * 32) >> 4), idesc(2 * kQB, 0),
                   ks > 0 ? 1u : 0u);
            mma_ss(tmem + kColDA, aV + (uint64_t)(ka >> 4),
                   bdo + (uint64_t)((((ks >> 2) * kQB * 128) + (ks & 3) * 32) >> 4), idesc(kQB, 0),
                   ks > 0 ? 1u : 0u);
          }
          mma_commit(&sm.s_full);
        }
        // Every MMA issued here completes before TMEM is freed.
        mma_commit(&sm.drain);
        mbar_drain(&sm.drain, 0);
      } else {
        bool ok = true;
        for (int i = 0; ok && i < nq; ++i) {
          if (!(ok = mbar_wait(&sm.p_full, i & 1, abort, p.status))) break;
          tc_fence_after();
          issue_grads(i);
        }
        if (ok) mma_commit(&sm.done);
        mma_commit(&sm.drain_g);
        mbar_drain(&sm.drain_g, 0);
      }
    }
  } else if (warp >= kFirstEwWarp) {
    // ---------------- elementwise warpgroups ----------------
    // Thread = one key (TMEM lane) x 16 of the block's 64 queries (wg picks which).
    const int wg = (warp - kFirstEwWarp) >> 2, quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const uint32_t lb = tmem + ((uint32_t)(32 * quarter) << 16);
    const int kk = kb * kKB + row;  // key position
    const float isd = rsqrtf((float)D), scale2 = kLog2e * isd;
    bool ok = true;
    int qh = qbh0, qb = q0;  // query head and block of step i
    for (int i = 0; i < nq; ++i, qb = qb + 1 < qend ? qb + 1 : (++qh, q0)) {
      if (!(ok = warp_wait(&sm.s_full, i & 1, abort, p.status))) break;
      tc_fence_after();
      uint32_t s[kEwCols], t[kEwCols], da[kEwCols];
      tmem_ld16(lb + kColS + kEwCols * wg, s);
      tmem_ld16(lb + kColT + kEwCols * wg, t);
      tmem_ld16(lb + kColDA + kEwCols * wg, da);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.s_free);
      const int i0 = qb * kQB + kEwCols * wg;  // query of column 0
      // Masks only where some pair of the warp is masked: the causal diagonal
      // (query before key) and queries past N.
      const bool edge = __any_sync(0xffffffffu, (p.causal && i0 < kk) || i0 + kEwCols - 1 >= p.N ||
                                                    (p.window > 0 && i0 + kEwCols - 1 >= kk + p.window));
      // The statistics of this thread's 16 queries (read by every lane: cached).
      const float* sts = p.stats + stat_index(qh, p.Npad, qb * kQB, 0) + kEwCols * wg;
      const uint64_t sc2 = f2(scale2, scale2), nisd2 = f2(-isd, -isd);
      uint32_t pa[kEwCols / 2], pl[kEwCols / 2], pt[kEwCols / 2];
#pragma unroll
      for (int c4 = 0; c4 < kEwCols / 4; ++c4) {
        // Statistics of four consecutive queries (broadcast loads).
        const float4 L = __ldg(reinterpret_cast<const float4*>(sts + 4 * c4));
        const float4 C = __ldg(reinterpret_cast<const float4*>(sts + 64 + 4 * c4));
        const float4 Dv = __ldg(reinterpret_cast<const float4*>(sts + 128 + 4 * c4));
        const float4 Fd = __ldg(reinterpret_cast<const float4*>(sts + 192 + 4 * c4));
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int e = 4 * c4 + 2 * h;
          const bool k0 = !edge || ((!p.causal || i0 + e >= kk) && i0 + e < p.N &&
                                    (p.window <= 0 || i0 + e < kk + p.window));
          const bool k1 = !edge || ((!p.causal || i0 + e + 1 >= kk) && i0 + e + 1 < p.N &&
                                    (p.window <= 0 || i0 + e + 1 < kk + p.window));
          const GradPairs g = grad_pairs(
              s[e], s[e + 1], t[e], t[e + 1], da[e], da[e + 1], h ? f2(L.z, L.w) : f2(L.x, L.y),
              h ? f2(C.z, C.w) : f2(C.x, C.y), h ? f2(Dv.z, Dv.w) : f2(Dv.x, Dv.y),
              h ? f2(Fd.z, Fd.w) : f2(Fd.x, Fd.y), sc2, nisd2, k0, k1);
          pa[2 * c4 + h] = g.a;
          pl[2 * c4 + h] = g.dl;
          pt[2 * c4 + h] = g.dt;
        }
      }
      // The operands are free once the gradient MMAs of block i - 1 completed.
      if (i > 0) {
        if (!(ok = warp_wait(&sm.ag_free, (i - 1) & 1, abort, p.status))) break;
        tc_fence_after();
      }
      st_row_chunks<kEwCols / 8>(sm.a, row, (kEwCols / 8) * wg, pa);
      tmem_st8(lb + kColG + (kEwCols / 2) * wg, pl);
      tmem_st8(lb + kColG + 32 + (kEwCols / 2) * wg, pt);
      fence_async_smem();
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full);
    }
    if (ok && warp_wait(&sm.done, 0, abort, p.status)) {
      tc_fence_after();
      // Warpgroups 0, 1: the two halves of dV; 2, 3: of dK.
      const int half = (wg & 1) * (D / 2);
      __nv_bfloat16* dst = kk < p.N ? (wg < 2 ? p.g0 : p.g1) + ((long long)bh * p.N + kk) * D + half : nullptr;
      tmem_row_to_global<D / 2>(lb + (wg < 2 ? kColDV : kColDK) + half, dst);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

// ---------------------------------------------------------------------------
// 3. dQ and dR: one CTA per 128-query block of a head.
// ---------------------------------------------------------------------------
constexpr int kQM = 128;  // queries per CTA (MMA M)
constexpr int kKN = 64;   // keys per streamed block
constexpr int kKVStages = 3;

template <int D>
struct QSmem {
  static constexpr int kHalves = D / 64;
  uint8_t q[kHalves][kQM * 128];
  uint8_t r[kHalves][kQM * 128];
  uint8_t dout[kHalves][kQM * 128];
  uint8_t k[kKVStages][kHalves][kKN * 128];
  uint8_t v[kKVStages][kHalves][kKN * 128];
  uint64_t q_full, kv_full[kKVStages], kv_empty[kKVStages];
  uint64_t s_full, s_free, p_full, pv_done, done, drain, drain_g;
  uint32_t tmem_base;
  int abort;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmR,
                  const __grid_constant__ CUtensorMap tmdO, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, BwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  using Sm = QSmem<D>;
  constexpr int kHalves = D / 64;
  // TMEM columns: the score stage, the bf16 pairs of dl (32 columns) and dt
  // (32), then the dQ and dR accumulators.
  constexpr uint32_t kColS = 0, kColT = 64, kColDA = 128, kColP = 192, kColDQ = 256, kColDR = 256 + D;
  Sm& sm = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = p.B * p.H;
  const int nmb = (p.N + kQM - 1) / kQM;
  // The last query block sees every key (causal): rank r is query block nmb - 1 - r.
  const BlockOrder bo = block_order(blockIdx.x, BH, nmb, p.chunk_heads);
  const int m = nmb - 1 - bo.rank, bh = bo.bh;
  const int kvbh = (bh / p.H) * p.Hkv + (bh % p.H) / (p.H / p.Hkv);  // the KV head this query head reads
  // Key blocks j0 .. j0 + nk - 1 (a window hides the keys before m kQM - window + 1).
  const int j0 = p.window > 0 ? max(0, m * kQM - p.window + 1) / kKN : 0;
  const int nk = (p.causal ? (min(m * kQM + kQM - 1, p.N - 1) / kKN + 1) : (p.N + kKN - 1) / kKN) - j0;
  volatile int* abort = &sm.abort;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kKVStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.s_free, 4 * kEwGroups);
    mbar_init(&sm.p_full, 128 * kEwGroups);
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.done, 1);
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.drain_g, 1);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&sm.tmem_base)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const int qrow = bh * p.N + m * kQM;
      mbar_expect_tx(&sm.q_full, 3 * kQM * D * 2);
      for (int h = 0; h < kHalves; ++h) {
        tma_load_2d(sm.q[h], &tmQ, &sm.q_full, 64 * h, qrow);
        tma_load_2d(sm.r[h], &tmR, &sm.q_full, 64 * h, qrow);
        tma_load_2d(sm.dout[h], &tmdO, &sm.q_full, 64 * h, qrow);
      }
      int last_use[kKVStages] = {-1, -1, -1};
      for (int j = 0; j < nk && !*abort; ++j) {
        const int st = j % kKVStages, u = j / kKVStages;
        if (u > 0 && !mbar_wait(&sm.kv_empty[st], (u - 1) & 1, abort, p.status)) break;
        mbar_expect_tx(&sm.kv_full[st], 2 * kKN * D * 2);
        last_use[st] = u;
        const int krow = kvbh * p.N + (j0 + j) * kKN;
        for (int h = 0; h < kHalves; ++h) {
          tma_load_2d(sm.k[st][h], &tmK, &sm.kv_full[st], 64 * h, krow);
          tma_load_2d(sm.v[st][h], &tmV, &sm.kv_full[st], 64 * h, krow);
        }
      }
      if (*abort) {
        mbar_drain(&sm.q_full, 0);
        for (int s = 0; s < kKVStages; ++s)
          if (last_use[s] >= 0) mbar_drain(&sm.kv_full[s], (uint32_t)(last_use[s] & 1));
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ---------------- MMA issuers: scores (warp 1) and gradients (warp 2) ----------------
    if (lane == 0) {
      const uint64_t aQ = sdesc(smem_u32(sm.q[0]), 16, 1024), aR = sdesc(smem_u32(sm.r[0]), 16, 1024);
      const uint64_t aO = sdesc(smem_u32(sm.dout[0]), 16, 1024);
      auto issue_grads = [&](int b) {
        const int st = b % kKVStages;
        // K as the MN-major B operand ([keys][dims]: halves apart by LBO).
        const uint64_t bk = sdesc(smem_u32(sm.k[st][0]), kKN * 128, 1024);
#pragma unroll
        for (int ks = 0; ks < kKN / 16; ++ks) {
          const uint32_t acc = (b > 0 || ks > 0) ? 1u : 0u;
          const uint64_t bks = bk + (uint64_t)((ks * 2048) >> 4);
          mma_ts(tmem + kColDQ, tmem + kColP + ks * 8, bks, idesc(D, 1), acc);
          mma_ts(tmem + kColDR, tmem + kColP + 32 + ks * 8, bks, idesc(D, 1), acc);
        }
        mma_commit(&sm.kv_empty[st]);
        mma_commit(&sm.pv_done);
      };
      if (warp == 1) {
      bool ok = mbar_wait(&sm.q_full, 0, abort, p.status);
      for (int j = 0; ok && j < nk; ++j) {
        const int st = j % kKVStages;
        if (!(ok = mbar_wait(&sm.kv_full[st], (j / kKVStages) & 1, abort, p.status))) break;
        if (j > 0 && !(ok = mbar_wait(&sm.s_free, (j - 1) & 1, abort, p.status))) break;
        tc_fence_after();
        const uint64_t bk = sdesc(smem_u32(sm.k[st][0]), 16, 1024);
        const uint64_t bv = sdesc(smem_u32(sm.v[st][0]), 16, 1024);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t ao = (uint64_t)((((ks >> 2) * kQM * 128) + (ks & 3) * 32) >> 4);
          const uint64_t bo = (uint64_t)((((ks >> 2) * kKN * 128) + (ks & 3) * 32) >> 4);
          const uint32_t acc = ks > 0 ? 1u : 0u;
          mma_ss(tmem + kColS, aQ + ao, bk + bo, idesc(kKN, 0), acc);
          mma_ss(tmem + kColT, aR + ao, bk + bo, idesc(kKN, 0), acc);
          mma_ss(tmem + kColDA, aO + ao, bv + bo, idesc(kKN, 0), acc);
        }
        mma_commit(&sm.s_full);
      }
      mma_commit(&sm.drain);
      mbar_drain(&sm.drain, 0);
      } else {
        bool ok = true;
        for (int j = 0; ok && j < nk; ++j) {
          if (!(ok = mbar_wait(&sm.p_full, j & 1, abort, p.status))) break;
          tc_fence_after();
          issue_grads(j);
        }
        if (ok) mma_commit(&sm.done);
        mma_commit(&sm.drain_g);
        mbar_drain(&sm.drain_g, 0);
      }
    }
  } else if (warp >= kFirstEwWarp) {
    // ---------------- elementwise warpgroups ----------------
    // Thread = one query (TMEM lane) x 16 of the block's 64 keys (wg picks which).
    const int wg = (warp - kFirstEwWarp) >> 2, quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const uint32_t lb = tmem + ((uint32_t)(32 * quarter) << 16);
    const int i = m * kQM + row;  // query position
    const float isd = rsqrtf((float)D), scale2 = kLog2e * isd;
    // This query's statistics, as f32x2 pairs for the packed arithmetic.
    const float* sp = p.stats + stat_index(bh, p.Npad, i, 0);
    const uint64_t nl2 = f2(sp[0], sp[0]), c02 = f2(sp[64], sp[64]), dd2 = f2(sp[128], sp[128]),
                   fd2 = f2(sp[192], sp[192]);
    const uint64_t sc2 = f2(scale2, scale2), nisd2 = f2(-isd, -isd);
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      if (!(ok = warp_wait(&sm.s_full, j & 1, abort, p.status))) break;
      tc_fence_after();
      uint32_t s[kEwCols], t[kEwCols], da[kEwCols];
      tmem_ld16(lb + kColS + kEwCols * wg, s);
      tmem_ld16(lb + kColT + kEwCols * wg, t);
      tmem_ld16(lb + kColDA + kEwCols * wg, da);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.s_free);
      const int k0 = (j0 + j) * kKN + kEwCols * wg;  // key of column 0
      const bool edge = __any_sync(0xffffffffu, (p.causal && k0 + kEwCols - 1 > i) || k0 + kEwCols - 1 >= p.N ||
                                                    (p.window > 0 && k0 <= i - p.window));
      uint32_t pl[kEwCols / 2], pt[kEwCols / 2];
#pragma unroll
      for (int c = 0; c < kEwCols / 2; ++c) {
        const int e = 2 * c;
        const bool keep0 = !edge || ((!p.causal || k0 + e <= i) && k0 + e < p.N &&
                                     (p.window <= 0 || k0 + e > i - p.window));
        const bool keep1 = !edge || ((!p.causal || k0 + e + 1 <= i) && k0 + e + 1 < p.N &&
                                     (p.window <= 0 || k0 + e + 1 > i - p.window));
        const GradPairs g = grad_pairs(s[e], s[e + 1], t[e], t[e + 1], da[e], da[e + 1], nl2, c02, dd2, fd2, sc2,
                                       nisd2, keep0, keep1);
        pl[c] = g.dl;
        pt[c] = g.dt;
      }
      // The bf16 buffer is free once the gradient MMAs of block j - 1 completed.
      if (j > 0) {
        if (!(ok = warp_wait(&sm.pv_done, (j - 1) & 1, abort, p.status))) break;
        tc_fence_after();
      }
      tmem_st8(lb + kColP + (kEwCols / 2) * wg, pl);
      tmem_st8(lb + kColP + 32 + (kEwCols / 2) * wg, pt);
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full);
    }
    if (ok && warp_wait(&sm.done, 0, abort, p.status)) {
      tc_fence_after();
      // Warpgroups 0, 1: the two halves of dQ; 2, 3: of dR.
      const int half = (wg & 1) * (D / 2);
      __nv_bfloat16* dst = i < p.N ? (wg < 2 ? p.g0 : p.g1) + ((long long)bh * p.N + i) * D + half : nullptr;
      tmem_row_to_global<D / 2>(lb + (wg < 2 ? kColDQ : kColDR) + half, dst);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

// The step of the last backward launch that failed in this thread.
thread_local const char* t_bwd_fail = "";

cudaError_t fail_at(const char* where, cudaError_t e) {
  t_bwd_fail = where;
  return e;
}

template <int D>
cudaError_t launch_bwd_d(const BwdArgs& a, cudaStream_t st, int num_sms) {
  const long long rows = (long long)a.B * a.H * a.N;
  if (rows >= (1ll << 31)) return cudaErrorInvalidValue;
  const int BH = a.B * a.H;
  const int Hkv = a.Hkv > 0 ? a.Hkv : a.H;
  const long long kv_rows = (long long)a.B * Hkv * a.N;
  const int Npad = (int)bwd_padded_rows(a.N);
  CUtensorMap mQ64, mR64, mO64, mK128, mV128, mQ128, mR128, mO128, mK64, mV64;
  if (!make_map(&mQ64, a.Q, rows, kQB, D) || !make_map(&mR64, a.R, rows, kQB, D) ||
      !make_map(&mO64, a.dO, rows, kQB, D) || !make_map(&mK128, a.K, kv_rows, kKB, D) ||
      !make_map(&mV128, a.V, kv_rows, kKB, D) || !make_map(&mQ128, a.Q, rows, kQM, D) ||
      !make_map(&mR128, a.R, rows, kQM, D) || !make_map(&mO128, a.dO, rows, kQM, D) ||
      !make_map(&mK64, a.K, kv_rows, kKN, D) || !make_map(&mV64, a.V, kv_rows, kKN, D))
    return fail_at("tensor map", cudaErrorInvalidValue);
  float* stats = reinterpret_cast<float*>(a.stats);
  const long long srows = (long long)BH * Npad;
  bwd_prep_kernel<<<(unsigned)((srows + 7) / 8), 256, 0, st>>>(
      reinterpret_cast<const __nv_bfloat16*>(a.out), reinterpret_cast<const float*>(a.vbar),
      reinterpret_cast<const __nv_bfloat16*>(a.dO), a.lse, a.tbar, stats, BH, a.N, Npad, D);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail_at("statistics kernel", e);
  const int nblk = (a.N + 127) / 128;  // 128-key blocks = 128-query blocks
  // About two waves of blocks per chunk of heads.
  int ch = (2 * num_sms + nblk - 1) / nblk;
  ch = ch < 1 ? 1 : (ch > BH ? BH : ch);
  // A dK/dV CTA of a KV head streams the query tiles of its G query heads:
  // chunks of ch / G KV heads keep the same query-tile footprint in L2.
  const int BHkv = a.B * Hkv, G = a.H / Hkv;
  int chkv = (ch + G - 1) / G;
  chkv = chkv > BHkv ? BHkv : chkv;
  // PLX_FAULT_INJECT=bwd_stall makes one CTA's bounded waits run out (tests of
  // the timeout status only).
  const char* fi = getenv("PLX_FAULT_INJECT");
  const int inject = (fi != nullptr && strcmp(fi, "bwd_stall") == 0) ? 1 : 0;
  BwdParams pk{a.B, a.H, a.N, Npad, a.causal, Hkv, a.window, inject, chkv, stats, reinterpret_cast<__nv_bfloat16*>(a.dV),
               reinterpret_cast<__nv_bfloat16*>(a.dK), a.status};
  size_t smem = sizeof(KvSmem<D>) + 1024;
  if ((e = cudaFuncSetAttribute(bwd_dkv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
      cudaSuccess)
    return fail_at("dK/dV shared-memory attribute", e);
  bwd_dkv_kernel<D><<<BHkv * nblk, kThreads, smem, st>>>(mQ64, mR64, mO64, mK128, mV128, pk);
  if ((e = cudaGetLastError()) != cudaSuccess) return fail_at("dK/dV kernel", e);
  BwdParams pq{a.B, a.H, a.N, Npad, a.causal, Hkv, a.window, 0, ch, stats, reinterpret_cast<__nv_bfloat16*>(a.dQ),
               reinterpret_cast<__nv_bfloat16*>(a.dR), a.status};
  // At least 116 KB so that one CTA (and its 512 TMEM columns) holds an SM.
  smem = sizeof(QSmem<D>) + 1024;
  if (smem < 116 * 1024) smem = 116 * 1024;
  if ((e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
      cudaSuccess)
    return fail_at("dQ/dR shared-memory attribute", e);
  bwd_dq_kernel<D><<<BH * nblk, kThreads, smem, st>>>(mQ128, mR128, mO128, mK64, mV64, pq);
  if ((e = cudaGetLastError()) != cudaSuccess) return fail_at("dQ/dR kernel", e);
  return cudaSuccess;
}

}  // namespace

size_t bwd_padded_rows(int N) { return ((size_t)N + 127) / 128 * 128; }

const char* bwd_last_failure() { return t_bwd_fail; }

cudaError_t launch_prefill_bwd(const BwdArgs& a, cudaStream_t st, int num_sms) {
  if (a.d == 128) return launch_bwd_d<128>(a, st, num_sms);
  if (a.d == 64) return launch_bwd_d<64>(a, st, num_sms);
  return cudaErrorInvalidValue;
}

}  // namespace plx
