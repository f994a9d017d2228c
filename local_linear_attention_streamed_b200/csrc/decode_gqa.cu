// Split-KV Parallax decode with grouped KV heads, bf16 caches, d in {64, 128}.
//
// G = H / Hkv consecutive query heads read one KV head.  The pages' decode
// packs the q and rho rows into one tensor-core tile so that one stream of K
// feeds both score products (agihunt.info summary, decode paragraph); with
// grouped heads the same tile carries the q and rho rows of several heads, so
// one pass over a KV head's cache serves the whole group.
//
// * Work unit = (b, KV head, key chunk), in chunk-major order; persistent CTAs
//   take units from a global counter (the first one statically).
// * Warp 4 is a TMA producer: it publishes the units to a small ring and
//   stages 64-key K and V blocks (128B-swizzled, the layout ldmatrix reads
//   without bank conflicts) in a 3-stage ring.  HBM is read once per KV head.
// * Warps 0..3 each own one or two query heads of the group (and, for G = 2, a
//   half of the keys).  Per 16-key slice: one m16n8k16 MMA per k-step whose A
//   rows are [q_h0; rho_h0; q_h1; rho_h1] gives S1 and S2 of the warp's heads;
//   the value MMA V^T x [w_hi, w_lo, wt_hi, wt_lo] per head gives O1 and O2 as
//   columns (each weight a bf16 hi + lo pair, as in the ungrouped decode).
// * One lazily raised running max per head (raised only when a block's max
//   exceeds it by more than 2^8), omega = sum w, T = sum w t in fp32.
// * Partials merge across the key-split warps in shared memory and across the
//   chunks of a KV head by the last CTA to finish it (one arrival counter per
//   (b, KV head) covers the group's heads); it leaves the counter at zero.
//
// Formulas: rainbus.top summary "方法步骤详情"; out = ((1 + T/omega) O1 - O2) / omega.
#include "plx_internal.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <math_constants.h>

namespace plx {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;  // + the TMA producer warp
constexpr int kBlk = 64;                             // keys per staged block
constexpr int kStages = 3;
constexpr int kUnitRing = 4;
constexpr float kLazyTau = 8.f;
constexpr unsigned long long kWaitNs = 2000000000ull;  // 2 s bound on every wait

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase of `parity`; false (with the CTA's abort flag and
// the device timeout status raised) if it ran out, or at once after an abort.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int* status) {
  if (mbar_test(bar, parity)) return true;
  const unsigned long long t0 = now_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_test(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (now_ns() - t0 > kWaitNs) {
        *abort = 1;
        atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
}
// Bounded wait that ignores the abort flag (lets issued copies land before exit).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = now_ns();
  while (!mbar_test(bar, parity) && now_ns() - t0 < kWaitNs) {
  }
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
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

// Byte offset of (row r, 16-byte chunk c) in a staged [64 rows x 128 B] tile
// with the 128B swizzle (what a TMA box of 64 bf16 columns writes).
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

template <int D>
struct Smem {
  static constexpr int KH = D / 64;  // 64-dim halves per row
  uint8_t k[kStages][KH * 8192];
  uint8_t v[kStages][KH * 8192];
  uint64_t full[kStages], empty[kStages];
  uint64_t unit_full[kUnitRing], unit_empty[kUnitRing];
  uint64_t csync;  // consumer-warp rendezvous (one lane per warp)
  long long unit_ring[kUnitRing];
  float O1[kConsumerWarps][2][D], O2[kConsumerWarps][2][D];
  float m[kConsumerWarps][2], omega[kConsumerWarps][2], T[kConsumerWarps][2];
  int last;
  int abort;
};

__device__ unsigned long long g_gqa_unit_next;
__device__ unsigned int g_gqa_cta_done;

// Per-warp softmax state of one head slot.
template <int D>
struct HeadState {
  float m;          // running max (log2 domain), warp-uniform
  float omega, T;   // partial sums over this lane's keys (equal in the eight lanes of one t)
};


template <int D, int G>
__global__ void __launch_bounds__(kThreads, 2)
    decode_gqa_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      DecodeArgs a) {
  constexpr int KH = D / 64;              // 64-dim halves of a row
  constexpr int KS = D / 16;              // k-steps of the score MMA
  constexpr int MT = D / 16;              // m-tiles (16 dims) of the value MMA
  constexpr int HPW = (G == 8) ? 2 : 1;   // query heads per consumer warp
  constexpr int NHG = G / HPW;            // head groups
  constexpr int KG = kConsumerWarps / NHG;  // key groups (warps that split a block's keys)
  static_assert(NHG * KG == kConsumerWarps, "warp split");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BKV = a.B * a.Hkv;
  const long long units = (long long)BKV * a.splits;
  volatile int* abort = &sm.abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    for (int s = 0; s < kUnitRing; ++s) {
      mbar_init(&sm.unit_full[s], 1);
      mbar_init(&sm.unit_empty[s], kConsumerWarps);
    }
    mbar_init(&sm.csync, kConsumerWarps);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------- TMA producer: units, then their K and V blocks ----------------
    if (lane == 0) {
      long long u = blockIdx.x;  // first unit static, the rest from the counter
      uint32_t pos = 0;          // K/V ring position
      long long issued[kStages];
      for (int s = 0; s < kStages; ++s) issued[s] = -1;
      for (int ui = 0;; ++ui) {
        const int slot = ui % kUnitRing;
        if (!mbar_wait(&sm.unit_empty[slot], ((ui / kUnitRing) & 1) ^ 1, abort, a.status)) break;
        const long long uu = u < units ? u : -1;
        sm.unit_ring[slot] = uu;
        mbar_arrive(&sm.unit_full[slot]);
        if (uu < 0) break;
        const long long next = (long long)gridDim.x + (long long)atomicAdd(&g_gqa_unit_next, 1ull);
        const int c = (int)(u / BKV);
        const int bkv = (int)(u - (long long)c * BKV);
        const int n = a.seqlens[bkv / a.Hkv];
        const int kbeg = c * a.chunk;
        const int nblk = (n >= 1 && n <= a.L && kbeg < n) ? (min(kbeg + a.chunk, n) - kbeg + kBlk - 1) / kBlk : 0;
        const int row0 = bkv * a.L + kbeg;  // < 2^31 (checked by the launcher)
        bool ok = true;
        for (int i = 0; i < nblk; ++i, ++pos) {
          const int st = pos % kStages;
          if (!(ok = mbar_wait(&sm.empty[st], ((pos / kStages) & 1) ^ 1, abort, a.status))) break;
          mbar_expect_tx(&sm.full[st], 2 * KH * 8192);
          issued[st] = pos / kStages;
#pragma unroll
          for (int h = 0; h < KH; ++h) {
            tma_load_2d(sm.k[st] + h * 8192, &tmK, &sm.full[st], 64 * h, row0 + kBlk * i);
            tma_load_2d(sm.v[st] + h * 8192, &tmV, &sm.full[st], 64 * h, row0 + kBlk * i);
          }
        }
        if (!ok) break;
        u = next;
      }
      // After an abort, let the issued copies land before the CTA exits.
      if (*abort) {
        for (int s = 0; s < kStages; ++s)
          if (issued[s] >= 0) mbar_drain(&sm.full[s], (uint32_t)(issued[s] & 1));
      }
    }
  } else {
    // ---------------- consumers ----------------
    const int g = lane >> 2, t = lane & 3;
    const int hg = warp % NHG, kg = warp / NHG;
    const float c_log2 = 1.4426950408889634f / sqrtf((float)D);
    const __nv_bfloat16* qall = reinterpret_cast<const __nv_bfloat16*>(a.q);
    const __nv_bfloat16* rall = reinterpret_cast<const __nv_bfloat16*>(a.r);
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
    uint32_t pos = 0, cs_phase = 0;
    // Rendezvous of the four consumer warps (bounded like every wait).
    auto csync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.csync);
      const bool r = mbar_wait(&sm.csync, cs_phase & 1, abort, a.status);
      ++cs_phase;
      return r;
    };
    for (int ui = 0;; ++ui) {
      const int slot = ui % kUnitRing;
      if (!mbar_wait(&sm.unit_full[slot], (ui / kUnitRing) & 1, abort, a.status)) break;
      const long long u = *reinterpret_cast<volatile long long*>(&sm.unit_ring[slot]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.unit_empty[slot]);
      if (u < 0) break;
      const int c = (int)(u / BKV);
      const int bkv = (int)(u - (long long)c * BKV);
      const int b = bkv / a.Hkv, kvh = bkv - b * a.Hkv;
      const int n = a.seqlens[b];
      if (n < 1 || n > a.L) {
        if (c == 0 && warp == 0) {
          __nv_bfloat16* o = out + ((long long)b * a.H + (long long)kvh * G) * D;
          for (int x = lane; x < G * D; x += 32) o[x] = __float2bfloat16(0.f);
          if (lane == 0) atomicOr(a.status, kStatusBadSeqlen);
        }
        continue;
      }
      const int kbeg = c * a.chunk;
      if (kbeg >= n) continue;
      const int kend = min(kbeg + a.chunk, n);
      const int nch = (n + a.chunk - 1) / a.chunk;
      const int nblk = (kend - kbeg + kBlk - 1) / kBlk;

      // A fragments: row 2s holds q and row 2s+1 rho of the warp's head slot s.
      uint32_t aq[KS][2];
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) aq[ks][0] = aq[ks][1] = 0u;
      if (g < 2 * HPW) {
        const int h = kvh * G + hg * HPW + (g >> 1);
        const __nv_bfloat16* src = ((g & 1) ? rall : qall) + ((long long)b * a.H + h) * D;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          aq[ks][0] = *reinterpret_cast<const uint32_t*>(src + 16 * ks + 2 * t);
          aq[ks][1] = *reinterpret_cast<const uint32_t*>(src + 16 * ks + 8 + 2 * t);
        }
      }
      float O[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) O[mt][0] = O[mt][1] = O[mt][2] = O[mt][3] = 0.f;
      HeadState<D> hs[HPW];
#pragma unroll
      for (int s = 0; s < HPW; ++s) {
        hs[s].m = -CUDART_INF_F;
        hs[s].omega = 0.f;
        hs[s].T = 0.f;
      }
      bool ok = true;
      for (int i = 0; i < nblk; ++i, ++pos) {
        const int stg = pos % kStages;
        if (!(ok = mbar_wait(&sm.full[stg], (pos / kStages) & 1, abort, a.status))) break;
        const uint32_t kb = smem_u32(sm.k[stg]), vb = smem_u32(sm.v[stg]);
        for (int sb = kg; sb < kBlk / 16; sb += KG) {
          const int j0 = kbeg + kBlk * i + 16 * sb;  // first key of this 16-key slice
          if (j0 >= kend) break;
          // ---- S = [q; rho; ...] K^T for 16 keys (two n-tiles of 8).
          float S[2][4];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) S[nt][0] = S[nt][1] = S[nt][2] = S[nt][3] = 0.f;
          {
            const int mi = lane >> 3;
            const int r = 16 * sb + 8 * (mi >> 1) + (lane & 7);
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
              const int d0 = 16 * ks + 8 * (mi & 1);
              uint32_t b00, b01, b10, b11;
              ldsm_x4(kb + (uint32_t)((d0 >> 6) * 8192) + swz(r, (d0 & 63) >> 3), b00, b01, b10, b11);
              mma_bf16(S[0], aq[ks][0], 0u, aq[ks][1], 0u, b00, b01);
              mma_bf16(S[1], aq[ks][0], 0u, aq[ks][1], 0u, b10, b11);
            }
          }
          // Lane (g, t) holds row g at keys 8nt + 2t + {0, 1}; every lane takes
          // s1 and s2 of each of the warp's heads at its own keys (e4 = 2nt + e).
          float s1[HPW][4], s2[HPW][4];
#pragma unroll
          for (int e4 = 0; e4 < 4; ++e4) {
            const float own = S[e4 >> 1][e4 & 1];
            const bool valid = j0 + 8 * (e4 >> 1) + 2 * t + (e4 & 1) < kend;
#pragma unroll
            for (int s = 0; s < HPW; ++s) {
              const float x1 = __shfl_sync(0xffffffffu, own, 8 * s + t);
              const float x2 = __shfl_sync(0xffffffffu, own, 8 * s + 4 + t);
              s1[s][e4] = valid ? x1 * c_log2 : -CUDART_INF_F;
              s2[s][e4] = valid ? x2 : 0.f;
            }
          }
          float w[HPW][4];
#pragma unroll
          for (int s = 0; s < HPW; ++s) {
            float ml = fmaxf(fmaxf(s1[s][0], s1[s][1]), fmaxf(s1[s][2], s1[s][3]));
            ml = fmaxf(ml, __shfl_xor_sync(0xffffffffu, ml, 1));
            const float mblk = fmaxf(ml, __shfl_xor_sync(0xffffffffu, ml, 2));  // warp-uniform
            if (mblk > hs[s].m + kLazyTau) {  // also on the slot's first slice (m = -inf)
              const float alpha = exp2f(hs[s].m - mblk);
              if ((t >> 1) == s) {  // this lane's value columns 2t, 2t+1 belong to slot t/2
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
                  for (int q = 0; q < 4; ++q) O[mt][q] *= alpha;
                }
              }
              hs[s].omega *= alpha;
              hs[s].T *= alpha;
              hs[s].m = mblk;
            }
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4) w[s][e4] = exp2f(s1[s][e4] - hs[s].m);
            hs[s].omega += (w[s][0] + w[s][1]) + (w[s][2] + w[s][3]);
            hs[s].T += (w[s][0] * s2[s][0] + w[s][1] * s2[s][1]) + (w[s][2] * s2[s][2] + w[s][3] * s2[s][3]);
          }
          // ---- [O1 O2] += V^T x [w_hi, w_lo, wt_hi, wt_lo] per head slot:
          // value column n = 4s + kind comes from the lanes with g = n.
          uint32_t b0 = 0u, b1 = 0u;
          if (g < 4 * HPW) {
            const bool s0 = (g >> 2) == 0;
            const int kind = g & 3;
            float x[4];
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4) {
              const float ww = s0 ? w[0][e4] : w[HPW - 1][e4];
              const float tt = s0 ? s2[0][e4] : s2[HPW - 1][e4];
              float v = (kind < 2) ? ww : ww * tt;
              if (kind & 1) v -= __bfloat162float(__float2bfloat16_rn(v));
              x[e4] = v;
            }
            b0 = pack_bf16(x[0], x[1]);  // keys 2t, 2t+1
            b1 = pack_bf16(x[2], x[3]);  // keys 8+2t, 9+2t
          }
          {
            const int mi = lane >> 3;
            const int r = 16 * sb + 8 * (mi >> 1) + (lane & 7);
            // Keys past the end of the sequence carry zero weight; their V rows
            // (whatever the cache holds there) are zeroed so that they cannot
            // turn into NaN in the product.
            const bool edge = j0 + 16 > kend;
            const int k0 = j0 + 2 * t, k8 = j0 + 8 + 2 * t;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              const int d0 = 16 * mt + 8 * (mi & 1);
              uint32_t a0, a1, a2, a3;
              ldsm_x4_t(vb + (uint32_t)((d0 >> 6) * 8192) + swz(r, (d0 & 63) >> 3), a0, a1, a2, a3);
              if (edge) {
                const uint32_t m0 = (k0 < kend ? 0x0000FFFFu : 0u) | (k0 + 1 < kend ? 0xFFFF0000u : 0u);
                const uint32_t m8 = (k8 < kend ? 0x0000FFFFu : 0u) | (k8 + 1 < kend ? 0xFFFF0000u : 0u);
                a0 &= m0;
                a1 &= m0;
                a2 &= m8;
                a3 &= m8;
              }
              mma_bf16(O[mt], a0, a1, a2, a3, b0, b1);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[stg]);
      }
      if (!ok) break;
      // ---- Warp partials to shared memory.
#pragma unroll
      for (int s = 0; s < HPW; ++s) {
        float om = hs[s].omega, tt = hs[s].T;
        om += __shfl_xor_sync(0xffffffffu, om, 1);
        om += __shfl_xor_sync(0xffffffffu, om, 2);
        tt += __shfl_xor_sync(0xffffffffu, tt, 1);
        tt += __shfl_xor_sync(0xffffffffu, tt, 2);
        if (lane == 0) {
          sm.m[warp][s] = hs[s].m;
          sm.omega[warp][s] = om;
          sm.T[warp][s] = tt;
        }
      }
      if ((t >> 1) < HPW) {  // lane t: columns 2t, 2t+1 = slot t/2, O1 (t even) or O2 (t odd), hi + lo
        float* dst = (t & 1) ? sm.O2[warp][t >> 1] : sm.O1[warp][t >> 1];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          dst[16 * mt + g] = O[mt][0] + O[mt][1];
          dst[16 * mt + 8 + g] = O[mt][2] + O[mt][3];
        }
      }
      if (!csync()) break;
      // ---- Merge the key groups per head; finish or publish the chunk's partials.
      const int x = threadIdx.x;  // 0..127: output dim
#pragma unroll 1
      for (int hh = 0; hh < G; ++hh) {
        const int hgg = hh / HPW, s = hh % HPW;
        float M = -CUDART_INF_F;
#pragma unroll
        for (int kk = 0; kk < KG; ++kk) M = fmaxf(M, sm.m[hgg + NHG * kk][s]);
        float om = 0.f, TT = 0.f, o1 = 0.f, o2 = 0.f;
#pragma unroll
        for (int kk = 0; kk < KG; ++kk) {
          const int w2 = hgg + NHG * kk;
          const float sc = (sm.m[w2][s] == -CUDART_INF_F) ? 0.f : exp2f(sm.m[w2][s] - M);
          om += sc * sm.omega[w2][s];
          TT += sc * sm.T[w2][s];
          if (x < D) {
            o1 += sc * sm.O1[w2][s][x];
            o2 += sc * sm.O2[w2][s][x];
          }
        }
        const long long bh = (long long)b * a.H + (long long)kvh * G + hh;
        if (nch == 1) {
          if (x < D) {
            const float inv = 1.f / om;
            out[bh * D + x] = __float2bfloat16_rn(((1.f + TT * inv) * o1 - o2) * inv);
          }
        } else {
          float* rec = a.partials + (bh * a.splits + c) * (2 * D + 4);
          if (x == 0) {
            rec[0] = M;
            rec[1] = om;
            rec[2] = TT;
          }
          if (x < D) {
            rec[4 + x] = o1;
            rec[4 + D + x] = o2;
          }
        }
      }
      if (nch > 1) {
        __threadfence();
        if (!csync()) break;
        if (x == 0) sm.last = (atomicAdd(a.counters + bkv, 1) == nch - 1);
        if (!csync()) break;
        if (sm.last) {
          __threadfence();
#pragma unroll 1
          for (int hh = 0; hh < G; ++hh) {
            const long long bh = (long long)b * a.H + (long long)kvh * G + hh;
            const float* base = a.partials + bh * a.splits * (2 * D + 4);
            float Mg = -CUDART_INF_F;
            for (int cc = 0; cc < nch; ++cc) Mg = fmaxf(Mg, __ldcg(base + (long long)cc * (2 * D + 4)));
            float om = 0.f, TT = 0.f, p1 = 0.f, p2 = 0.f;
            for (int cc = 0; cc < nch; ++cc) {
              const float* r = base + (long long)cc * (2 * D + 4);
              const float mc = __ldcg(r);
              const float sc = (mc == -CUDART_INF_F) ? 0.f : exp2f(mc - Mg);
              om += sc * __ldcg(r + 1);
              TT += sc * __ldcg(r + 2);
              if (x < D) {
                p1 += sc * __ldcg(r + 4 + x);
                p2 += sc * __ldcg(r + 4 + D + x);
              }
            }
            if (x < D) {
              const float inv = 1.f / om;
              out[bh * D + x] = __float2bfloat16_rn(((1.f + TT * inv) * p1 - p2) * inv);
            }
          }
          if (x == 0) a.counters[bkv] = 0;
        }
      }
      if (!csync()) break;  // shared memory is reused by the next unit
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Every CTA fetched its last unit before this point; the last CTA to get
    // here leaves the scheduler at zero for the next launch.
    __threadfence();
    if (atomicAdd(&g_gqa_cta_done, 1u) == gridDim.x - 1) {
      atomicExch(&g_gqa_unit_next, 0ull);
      atomicExch(&g_gqa_cta_done, 0u);
    }
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 2-D view [rows, d] of a bf16 cache [B, Hkv, L, d]: boxes of 64 dims x 64 keys, 128B swizzle.
bool make_cache_map(CUtensorMap* m, const void* base, long long rows, int d) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kBlk};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int G>
cudaError_t launch_gqa(const DecodeArgs& a, const CUtensorMap& mK, const CUtensorMap& mV, cudaStream_t st,
                       int num_sms) {
  const size_t smem = sizeof(Smem<D>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(decode_gqa_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_gqa_kernel<D, G>, kThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const long long units = (long long)a.B * a.Hkv * a.splits;
  long long grid = (long long)num_sms * per_sm;
  if (grid > units) grid = units;
  decode_gqa_kernel<D, G><<<(unsigned)grid, kThreads, smem, st>>>(mK, mV, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_gqa(const DecodeArgs& a, cudaStream_t st, int num_sms) {
  if (a.Hkv < 1 || a.H % a.Hkv != 0) return cudaErrorInvalidValue;
  const long long rows = (long long)a.B * a.Hkv * a.L;
  if (rows + kBlk >= (1ll << 31)) return cudaErrorInvalidValue;
  CUtensorMap mK, mV;
  if (!make_cache_map(&mK, a.K, rows, a.d) || !make_cache_map(&mV, a.V, rows, a.d)) return cudaErrorInvalidValue;
  const int G = a.H / a.Hkv;
  if (a.d == 128) {
    if (G == 2) return launch_gqa<128, 2>(a, mK, mV, st, num_sms);
    if (G == 4) return launch_gqa<128, 4>(a, mK, mV, st, num_sms);
    if (G == 8) return launch_gqa<128, 8>(a, mK, mV, st, num_sms);
  } else if (a.d == 64) {
    if (G == 2) return launch_gqa<64, 2>(a, mK, mV, st, num_sms);
    if (G == 4) return launch_gqa<64, 4>(a, mK, mV, st, num_sms);
    if (G == 8) return launch_gqa<64, 8>(a, mK, mV, st, num_sms);
  }
  return cudaErrorInvalidValue;
}

}  // namespace plx
