// Split-KV Parallax decode with grouped KV heads on warp-level MMAs, bf16
// caches, d = 64 with an odd number of KV heads (the launcher hands d = 128,
// and d = 64 with Hkv even, to the tcgen05 decode of decode_gqa_tc.cu; the
// kernel template still takes D in {64, 128}).
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
//   without bank conflicts) in a 3- or 6-stage ring.  HBM is read once per KV head.
// * Warps 0..3 each take one 16-key slice of every staged block, for all G
//   heads of the group, so each K and V byte is read from shared memory once:
//   one m16n8k16 MMA per k-step whose A rows are [q_0; rho_0; q_1; rho_1; ...]
//   gives S1 and S2 of every head of the group; the value MMA
//   V^T x [w_hi, w_lo, wt_hi, wt_lo] per head (two heads per n-tile) gives O1
//   and O2 as columns, one V fragment feeding every n-tile (each weight a bf16
//   hi + lo pair, as in the ungrouped decode).
// * One lazily raised running max per head (raised only when a block's max
//   exceeds it by more than 2^8), omega = sum w, T = sum w t in fp32.
// * Partials merge across the four warps in shared memory and across the
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

constexpr int kSlices = 4;  // 16-key slices of a staged block
constexpr int kBlk = 64;                             // keys per staged block
// Consumer warps: one per (16-key slice, share of the group's heads).  A group
// of 8 is split into two halves of 4 heads, so that a warp's accumulators
// (D/16 m-tiles x 2 n-tiles x 4 fp32 per lane) and its serial per-head work
// stay small; that configuration runs one CTA of 8 consumer warps per SM with
// a deeper staging ring, the others two CTAs of 4 consumer warps and 3 stages.
template <int D, int G>
struct Cfg {
  static constexpr int kHeadSplits = (G == 8) ? 2 : 1;
  static constexpr int kHeadsPerWarp = G / kHeadSplits;
  static constexpr int kConsumerWarps = kSlices * kHeadSplits;
  static constexpr int kThreads = (kConsumerWarps + 1) * 32;  // + the TMA producer warp
  static constexpr int kMinCtas = G == 8 ? 1 : 2;  // = decode_gqa_ctas_per_sm(G, 64)
  static constexpr int kStages = kMinCtas == 1 ? 6 : 3;
};
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

template <int D, int G>
struct Smem {
  static constexpr int kStages = Cfg<D, G>::kStages;
  static constexpr int KH = D / 64;  // 64-dim halves per row
  uint8_t k[kStages][KH * 8192];
  uint8_t v[kStages][KH * 8192];
  uint64_t full[kStages], empty[kStages];
  uint64_t unit_full[kUnitRing], unit_empty[kUnitRing];
  uint64_t csync;  // consumer-warp rendezvous (one lane per warp)
  long long unit_ring[kUnitRing];
  // The unit's A tile: row 2j = q and row 2j+1 = rho of the group's head j
  // (rows past 2G stay zero); rows padded by 16 bytes against bank conflicts.
  alignas(16) __nv_bfloat16 qr[16][D + 8];
  // Running merge of the four warps' partials per head of the group.
  float O1[G][D], O2[G][D];
  float m[G], omega[G], T[G];
  int last;
  int abort;
};

// 16-byte vector stores and ldmatrix rows need the A tile 16-byte aligned
// (its row pitch, 2 (D + 8) bytes, is a multiple of 16).
using SmemD128G8 = Smem<128, 8>;
using SmemD128G2 = Smem<128, 2>;
using SmemD64G8 = Smem<64, 8>;
using SmemD64G2 = Smem<64, 2>;
static_assert(offsetof(SmemD128G8, qr) % 16 == 0 && offsetof(SmemD128G2, qr) % 16 == 0 &&
                  offsetof(SmemD64G8, qr) % 16 == 0 && offsetof(SmemD64G2, qr) % 16 == 0,
              "A tile alignment");

__device__ unsigned long long g_gqa_unit_next;
__device__ unsigned int g_gqa_cta_done;



template <int D, int G>
__global__ void __launch_bounds__(Cfg<D, G>::kThreads, Cfg<D, G>::kMinCtas)
    decode_gqa_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      DecodeArgs a) {
  constexpr int kStages = Cfg<D, G>::kStages;
  constexpr int KH = D / 64;   // 64-dim halves of a row
  constexpr int KS = D / 16;   // k-steps of the score MMA
  constexpr int MT = D / 16;   // m-tiles (16 dims) of the value MMA
  constexpr int HW = Cfg<D, G>::kHeadsPerWarp;
  constexpr int NT = HW / 2;   // n-tiles (8 columns = 2 heads) of the value MMA
  constexpr int kConsumerWarps = Cfg<D, G>::kConsumerWarps;
  static_assert(G == 2 || G == 4 || G == 8, "group size");
  static_assert(kBlk / 16 == kSlices, "16-key slices");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem<D, G>& sm =
      *reinterpret_cast<Smem<D, G>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
    for (int x = 0; x < 16 * (D + 8); ++x) (&sm.qr[0][0])[x] = __float2bfloat16(0.f);
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
        // Keys lo..n-1 (lo > 0 only with a sliding window), cut into chunks.
        const int lo = (a.window > 0 && n > a.window) ? n - a.window : 0;
        const int kbeg = lo + c * a.chunk;
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
    const int sb = warp % kSlices;  // this warp's 16-key slice of every staged block
    const int h0 = (warp / kSlices) * HW;  // its first head within the group
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
      const int lo = (a.window > 0 && n > a.window) ? n - a.window : 0;
      const int kbeg = lo + c * a.chunk;
      if (kbeg >= n) continue;
      const int kend = min(kbeg + a.chunk, n);
      const int nch = (n - lo + a.chunk - 1) / a.chunk;
      const int nblk = (kend - kbeg + kBlk - 1) / kBlk;

      // The group's q and rho rows into the A tile (the previous unit's readers
      // finished at its closing rendezvous).
      for (int x = threadIdx.x; x < 2 * G * (D / 8); x += kConsumerWarps * 32) {
        const int row = x / (D / 8), col = (x % (D / 8)) * 8;
        const long long bh = (long long)b * a.H + (long long)kvh * G + (row >> 1);
        *reinterpret_cast<uint4*>(&sm.qr[row][col]) =
            *reinterpret_cast<const uint4*>(((row & 1) ? rall : qall) + bh * D + col);
      }
      if (!csync()) break;
      float O[MT][NT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) O[mt][nt][0] = O[mt][nt][1] = O[mt][nt][2] = O[mt][nt][3] = 0.f;
      }
      // Per head of the warp: running max (warp-uniform) and this lane's partial sums.
      float hm[HW], hom[HW], hT[HW];
#pragma unroll
      for (int j = 0; j < HW; ++j) {
        hm[j] = -CUDART_INF_F;
        hom[j] = 0.f;
        hT[j] = 0.f;
      }
      const uint32_t qa = smem_u32(&sm.qr[0][0]);
      bool ok = true;
      for (int i = 0; i < nblk; ++i, ++pos) {
        const int stg = pos % kStages;
        if (!(ok = mbar_wait(&sm.full[stg], (pos / kStages) & 1, abort, a.status))) break;
        const uint32_t kb = smem_u32(sm.k[stg]), vb = smem_u32(sm.v[stg]);
        const int j0 = kbeg + kBlk * i + 16 * sb;  // first key of this warp's slice
        if (j0 < kend) {
          const int mi = lane >> 3;
          // ---- S = [q_0; rho_0; q_1; ...] K^T for 16 keys (two n-tiles of 8).
          float S[2][4];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) S[nt][0] = S[nt][1] = S[nt][2] = S[nt][3] = 0.f;
          {
            const int ra = 8 * (mi & 1) + (lane & 7);             // A rows of matrices 0..3
            const int rk = 16 * sb + 8 * (mi >> 1) + (lane & 7);  // K rows (keys)
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
              uint32_t a0, a1, a2, a3, b00, b01, b10, b11;
              ldsm_x4(qa + (uint32_t)(ra * (D + 8) + 16 * ks + 8 * (mi >> 1)) * 2u, a0, a1, a2, a3);
              const int d0 = 16 * ks + 8 * (mi & 1);
              ldsm_x4(kb + (uint32_t)((d0 >> 6) * 8192) + swz(rk, (d0 & 63) >> 3), b00, b01, b10, b11);
              mma_bf16(S[0], a0, a1, a2, a3, b00, b01);
              mma_bf16(S[1], a0, a1, a2, a3, b10, b11);
            }
          }
          // Lane (g, t) holds rows g (S[nt][0..1]) and g + 8 (S[nt][2..3]) at
          // keys 8nt + 2t + {0, 1}.  Per head j: s1 = row 2j, s2 = row 2j + 1.
          // Value column n of n-tile nt is head 2nt + n/4, kind n % 4 (w_hi,
          // w_lo, wt_hi, wt_lo); lane (g, t) supplies column g of every n-tile.
          uint32_t bw0[NT], bw1[NT];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) bw0[nt] = bw1[nt] = 0u;
          // Phase 1 (all heads, no branches): scores at this lane's keys, the
          // block max and the lazy raise.  Head j of the warp is head h0 + j of
          // the group: rows 2(h0 + j) and 2(h0 + j) + 1, in S[..][0..1] (rows
          // 0..7) or S[..][2..3] (rows 8..15).
          float s1[HW][4], s2[HW][4], alpha[HW];
          const bool hi_rows = 2 * h0 >= 8;  // a warp's heads never straddle rows 7 | 8 (HW divides 4)
#pragma unroll
          for (int j = 0; j < HW; ++j) {
            const int src1 = ((2 * (h0 + j)) & 7) * 4 + t, src2 = ((2 * (h0 + j) + 1) & 7) * 4 + t;
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4) {
              const float own = hi_rows ? S[e4 >> 1][2 + (e4 & 1)] : S[e4 >> 1][e4 & 1];
              const float x1 = __shfl_sync(0xffffffffu, own, src1);
              const float x2 = __shfl_sync(0xffffffffu, own, src2);
              const bool valid = j0 + 8 * (e4 >> 1) + 2 * t + (e4 & 1) < kend;
              s1[j][e4] = valid ? x1 * c_log2 : -CUDART_INF_F;
              s2[j][e4] = valid ? x2 : 0.f;
            }
          }
          bool raised = false;
#pragma unroll
          for (int j = 0; j < HW; ++j) {
            float ml = fmaxf(fmaxf(s1[j][0], s1[j][1]), fmaxf(s1[j][2], s1[j][3]));
            ml = fmaxf(ml, __shfl_xor_sync(0xffffffffu, ml, 1));
            const float mblk = fmaxf(ml, __shfl_xor_sync(0xffffffffu, ml, 2));  // warp-uniform
            const bool up = mblk > hm[j] + kLazyTau;  // also on the head's first slice (m = -inf)
            alpha[j] = up ? exp2f(hm[j] - mblk) : 1.f;
            hm[j] = up ? mblk : hm[j];
            hom[j] *= alpha[j];
            hT[j] *= alpha[j];
            raised |= up;
          }
          if (raised) {  // warp-uniform; rare after a head's first slice
            // Columns 2t, 2t+1 of n-tile nt belong to the warp's head 2nt + t/2.
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const float al = (t >> 1) ? alpha[2 * nt + 1] : alpha[2 * nt];
#pragma unroll
              for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
                for (int q = 0; q < 4; ++q) O[mt][nt][q] *= al;
              }
            }
          }
          // Phase 2: weights, sums and the value MMA's B fragment.  Value column
          // n of n-tile nt is head 2nt + n/4, kind n % 4 (w_hi, w_lo, wt_hi,
          // wt_lo); lane (g, t) supplies column g of every n-tile.
#pragma unroll
          for (int j = 0; j < HW; ++j) {
            float w[4];
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4) w[e4] = exp2f(s1[j][e4] - hm[j]);
            hom[j] += (w[0] + w[1]) + (w[2] + w[3]);
            hT[j] += (w[0] * s2[j][0] + w[1] * s2[j][1]) + (w[2] * s2[j][2] + w[3] * s2[j][3]);
            if ((g >> 2) == (j & 1)) {
              const int kind = g & 3;
              float x[4];
#pragma unroll
              for (int e4 = 0; e4 < 4; ++e4) {
                float v = (kind < 2) ? w[e4] : w[e4] * s2[j][e4];
                if (kind & 1) v -= __bfloat162float(__float2bfloat16_rn(v));
                x[e4] = v;
              }
              bw0[j >> 1] = pack_bf16(x[0], x[1]);  // keys 2t, 2t+1
              bw1[j >> 1] = pack_bf16(x[2], x[3]);  // keys 8+2t, 9+2t
            }
          }
          // ---- [O1 O2] += V^T x weights; one V fragment feeds all n-tiles.
          const int rv = 16 * sb + 8 * (mi >> 1) + (lane & 7);
          // Keys past the end of the sequence carry zero weight; their V rows
          // (whatever the cache holds there) are zeroed so that they cannot
          // turn into NaN in the product.
          const bool edge = j0 + 16 > kend;
          const int k0 = j0 + 2 * t, k8 = j0 + 8 + 2 * t;
          const uint32_t m0 = (k0 < kend ? 0x0000FFFFu : 0u) | (k0 + 1 < kend ? 0xFFFF0000u : 0u);
          const uint32_t m8 = (k8 < kend ? 0x0000FFFFu : 0u) | (k8 + 1 < kend ? 0xFFFF0000u : 0u);
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            const int d0 = 16 * mt + 8 * (mi & 1);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(vb + (uint32_t)((d0 >> 6) * 8192) + swz(rv, (d0 & 63) >> 3), a0, a1, a2, a3);
            if (edge) {
              a0 &= m0;
              a1 &= m0;
              a2 &= m8;
              a3 &= m8;
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16(O[mt][nt], a0, a1, a2, a3, bw0[nt], bw1[nt]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[stg]);
      }
      if (!ok) break;
      // ---- Merge the slice warps' partials of each head, one slice after
      // another, into shared memory.
#pragma unroll
      for (int j = 0; j < HW; ++j) {
        hom[j] += __shfl_xor_sync(0xffffffffu, hom[j], 1);
        hom[j] += __shfl_xor_sync(0xffffffffu, hom[j], 2);
        hT[j] += __shfl_xor_sync(0xffffffffu, hT[j], 1);
        hT[j] += __shfl_xor_sync(0xffffffffu, hT[j], 2);
      }
      for (int w2 = 0; w2 < kSlices && ok; ++w2) {
        if (sb == w2) {
          // Lane (g, t): columns 2t, 2t+1 of n-tile nt = the warp's head
          // 2nt + t/2, O1 (t even) or O2 (t odd) as a hi + lo pair, dims
          // 16mt + g and + 8.
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const int jl = 2 * nt + (t >> 1);
            const int h = h0 + jl;
            const float mh = (t >> 1) ? hm[2 * nt + 1] : hm[2 * nt];
            float* dst = (t & 1) ? sm.O2[h] : sm.O1[h];
            float so = 1.f, ss = 0.f;
            if (w2 > 0) {
              const float M = fmaxf(sm.m[h], mh);
              ss = (sm.m[h] == -CUDART_INF_F) ? 0.f : exp2f(sm.m[h] - M);
              so = (mh == -CUDART_INF_F) ? 0.f : exp2f(mh - M);
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              const float v0 = O[mt][nt][0] + O[mt][nt][1], v8 = O[mt][nt][2] + O[mt][nt][3];
              float* p0 = dst + 16 * mt + g;
              p0[0] = w2 > 0 ? so * v0 + ss * p0[0] : v0;
              p0[8] = w2 > 0 ? so * v8 + ss * p0[8] : v8;
            }
          }
          __syncwarp();
          if (lane < HW) {
            const int h = h0 + lane;
            float mh = hm[0], oh = hom[0], th = hT[0];
#pragma unroll
            for (int j = 1; j < HW; ++j) {
              if (lane == j) {
                mh = hm[j];
                oh = hom[j];
                th = hT[j];
              }
            }
            if (w2 == 0) {
              sm.m[h] = mh;
              sm.omega[h] = oh;
              sm.T[h] = th;
            } else {
              const float M = fmaxf(sm.m[h], mh);
              const float ss = (sm.m[h] == -CUDART_INF_F) ? 0.f : exp2f(sm.m[h] - M);
              const float so = (mh == -CUDART_INF_F) ? 0.f : exp2f(mh - M);
              sm.omega[h] = ss * sm.omega[h] + so * oh;
              sm.T[h] = ss * sm.T[h] + so * th;
              sm.m[h] = M;
            }
          }
        }
        ok = csync();
      }
      if (!ok) break;
      // ---- Finish or publish the chunk's partials (thread x owns dim x).
      const int x = threadIdx.x;
#pragma unroll 1
      for (int hh = 0; hh < G; ++hh) {
        const float M = sm.m[hh], om = sm.omega[hh], TT = sm.T[hh];
        const long long bh = (long long)b * a.H + (long long)kvh * G + hh;
        if (nch == 1) {
          if (x < D) {
            const float inv = 1.f / om;
            out[bh * D + x] = __float2bfloat16_rn(((1.f + TT * inv) * sm.O1[hh][x] - sm.O2[hh][x]) * inv);
          }
        } else {
          float* rec = a.partials + (bh * a.splits + c) * (2 * D + 4);
          if (x == 0) {
            rec[0] = M;
            rec[1] = om;
            rec[2] = TT;
          }
          if (x < D) {
            rec[4 + x] = sm.O1[hh][x];
            rec[4 + D + x] = sm.O2[hh][x];
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
            // Several chunks' loads in flight per round trip.
#pragma unroll 4
            for (int cc = 0; cc < nch; ++cc) Mg = fmaxf(Mg, __ldcg(base + (long long)cc * (2 * D + 4)));
            float om = 0.f, TT = 0.f, p1 = 0.f, p2 = 0.f;
#pragma unroll 4
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
  const size_t smem = sizeof(Smem<D, G>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(decode_gqa_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_gqa_kernel<D, G>, Cfg<D, G>::kThreads,
                                                    smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const long long units = (long long)a.B * a.Hkv * a.splits;
  long long grid = (long long)num_sms * per_sm;
  if (grid > units) grid = units;
  decode_gqa_kernel<D, G><<<(unsigned)grid, Cfg<D, G>::kThreads, smem, st>>>(mK, mV, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_gqa(const DecodeArgs& a, cudaStream_t st, int num_sms) {
  if (a.Hkv < 1 || a.H % a.Hkv != 0) return cudaErrorInvalidValue;
  if (decode_gqa_tc(a.Hkv, a.d)) return launch_decode_gqa_tc(a, st, num_sms);
  const long long rows = (long long)a.B * a.Hkv * a.L;
  if (rows + kBlk >= (1ll << 31)) return cudaErrorInvalidValue;
  CUtensorMap mK, mV;
  if (!make_cache_map(&mK, a.K, rows, a.d) || !make_cache_map(&mV, a.V, rows, a.d)) return cudaErrorInvalidValue;
  const int G = a.H / a.Hkv;
  if (a.d == 64) {
    if (G == 2) return launch_gqa<64, 2>(a, mK, mV, st, num_sms);
    if (G == 4) return launch_gqa<64, 4>(a, mK, mV, st, num_sms);
    if (G == 8) return launch_gqa<64, 8>(a, mK, mV, st, num_sms);
  }
  return cudaErrorInvalidValue;
}

}  // namespace plx
