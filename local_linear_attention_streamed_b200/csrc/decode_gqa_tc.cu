// Split-KV Parallax decode on the tensor cores (tcgen05 MMAs with TMEM
// accumulators, TMA staging), bf16 caches, d = 128 with one KV head per query
// head (G = 1) or grouped KV heads (G = H / Hkv in {2, 4, 8}), and d = 64
// with grouped KV heads taken two KV heads at a time (see "d = 64" below).
//
// G consecutive query heads read one KV head, so one pass over a KV head's
// cache serves the whole group: the pages' decode packs the q and rho rows
// into one tensor-core tile so that a single stream of K feeds both score
// products (agihunt.info summary, decode paragraph), and grouping fills that
// tile with the rows of every head of the group.
//
// Per staged block of 128 keys (one CTA per SM, persistent, units from a
// global counter, unit = (b, KV head, key chunk)):
//   * scores, keys as the MMA's M:  S^T [128 keys x 16] = K_blk [Q; R]^T
//     (B rows 0..G-1 = q of the group's heads, rows 8..8+G-1 = rho);
//   * one thread per key (TMEM lane) forms, per head, the weight
//     w = 2^(s c - m) (lazy running max m, raised only when a block's max
//     exceeds it by more than 2^8) and w t, each as a bf16 hi + lo pair, into
//     a shared-memory tile W [128 keys x 4G];
//   * value product, dims as the MMA's M:  O^T [128 dims x 4G] += V_blk^T W,
//     with V read in place as an MN-major operand; the columns of head h are
//     sum w_hi v, sum w_lo v, sum wt_hi v, sum wt_lo v, so O1 and O2 come out
//     with about 16 bits of weight precision (the hi + lo split of the
//     ungrouped decode).
// omega = sum w and T = sum w t are kept per thread in fp32 and reduced at
// the end of the unit.  Chunks of one (b, KV head) merge through fp32
// partial records, by the last CTA to finish one (an arrival counter per
// (b, KV head), left at zero).
//
// d = 64.  The value product needs 128 dims as its M, so a unit takes a pair
// of KV heads (Hkv even): their 64-dim K (and V) blocks sit side by side as
// the two 64-dim halves of one 128-dim tile, the q / rho operand is
// block-diagonal (member p's rows 16p.. carry its heads' q and rho in half p
// and zeros in the other half), so one score MMA (N = 32) gives both members'
// scores, and the value product's lanes 0..63 / 64..127 are the two members'
// dims, each reading its own member's weight columns.
//
// Formulas: rainbus.top summary "方法步骤详情"; out = ((1 + T/omega) O1 - O2) / omega.
#include "plx_internal.cuh"
#include "sm100.cuh"
#include "decode_tc_common.cuh"

#include <math_constants.h>

#include <cstdlib>
#include <cstring>

namespace plx {
namespace {

using namespace sm100;
using namespace dtc;

constexpr int kUnitRing = 4;
constexpr int kFirstEw = 4;  // warp 0 TMA, warp 1 MMA, warps 4.. the key warpgroup(s)
constexpr float kLazyTau = 8.f;
constexpr float kLog2e = 1.4426950408889634f;

// Geometry per head dim D (the staged tiles are 128 dims wide either way):
// KV heads per unit, rows of the q / rho operand (the score MMA's N), query
// heads per unit, value-product columns ((w_hi, w_lo, wt_hi, wt_lo) per query
// head, at least the MMA's minimum N of 16; spare rows of W stay zero), K/V
// stages (64 KB each; two where the weight tiles are largest), and TMEM:
// two score stages, then two value accumulators.
template <int D, int G>
struct Geo {
  static constexpr int kPair = D == 64 ? 2 : 1;
  static constexpr int kRows = 16 * kPair;
  static constexpr int kHeads = G * kPair;
  static constexpr int NW = 4 * kHeads < 16 ? 16 : 4 * kHeads;
  // K/V stages.  Where shared memory is short (the weight tiles of groups of
  // 8 at d = 64) K and V travel in separate rings: a K stage is free once the
  // block's scores are computed, a V stage only after its value product, so
  // V gets the deeper ring.  Elsewhere one ring carries both (measured 3 %
  // faster for the ungrouped decode than two rings of equal depth).
  static constexpr int kKS = (D == 64 && G == 8) ? 2 : 3, kVS = 3;
  static constexpr bool kSepKV = kKS != kVS;
  static constexpr uint32_t kColS = 0, kColO = 2 * kRows;
  static constexpr uint32_t kTmemCols = D == 64 ? 256 : 128;
  // Key warpgroups: with 8 or more query heads a unit, two warpgroups split
  // the heads (each thread still owns one key, and one dim at the end), so
  // the per-key work of a block is done by twice the threads.  Warpgroup kg
  // takes kHW heads; its weight rows and accumulator columns are the block
  // 4 kHW kg .. 4 kHW (kg + 1) - 1.
  static constexpr int kKW = kHeads >= 8 ? 2 : 1;
  static constexpr int kHW = kHeads / kKW;
  static constexpr int kWCols = kKW == 1 ? NW : 4 * kHW;
  static constexpr int kThreads = 128 * (1 + kKW);
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(kColO + 2 * NW <= kTmemCols, "TMEM columns");
};

template <int D, int G>
struct Smem {
  using Gm = Geo<D, G>;
  static constexpr int NW = Gm::NW, kKS = Gm::kKS, kVS = Gm::kVS;
  uint8_t k[kKS][2][kKeys * 128];  // [128 keys x 64 dims] per 64-dim half (d = 64: per member)
  uint8_t v[kVS][2][kKeys * 128];
  uint8_t qr[2][2][Gm::kRows * 128];   // per unit slot: [rows x 64 dims] per half
  uint8_t w[2][2][NW * 128];           // per block slot: [NW rows x 64 keys] per 64-key half
  uint64_t k_full[kKS], k_empty[kKS], v_full[kVS], v_empty[kVS];
  uint64_t qr_full[2], qr_empty[2];
  uint64_t unit_full[kUnitRing], unit_empty[kUnitRing];
  uint64_t s_full[2], s_free[2], w_full[2], w_free[2];
  uint64_t o_full[2], o_free[2];
  uint64_t vote[Gm::kKW][2];  // block-max exchange among a warpgroup's four key warps
  uint64_t rdv;               // rendezvous of the key warps at the end of a unit
  uint64_t drain;
  long long unit_ring[kUnitRing];
  int unit_n[kUnitRing];  // seqlens of the unit's batch row, read once by the producer
  alignas(16) float red[Gm::kKW][2][4][Gm::kHW];  // per-warp block maxima of each head
  float sums[Gm::kKW][4][2 * Gm::kHW];             // per-warp omega and T of each head
  int last;
  uint32_t tmem_base;
  int abort;
};

static_assert(sizeof(Smem<128, 8>) + 1024 <= 227 * 1024 && sizeof(Smem<64, 8>) + 1024 <= 227 * 1024 &&
                  sizeof(Smem<64, 4>) + 1024 <= 227 * 1024 && sizeof(Smem<64, 2>) + 1024 <= 227 * 1024,
              "shared memory of one CTA");

__device__ unsigned long long g_tc_unit_next;
__device__ unsigned int g_tc_cta_done;

template <int D, int G>
__global__ void __launch_bounds__(Geo<D, G>::kThreads, 1)
    decode_gqa_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmR,
                         DecodeArgs a) {
  using Gm = Geo<D, G>;
  constexpr int NW = Gm::NW, kKS = Gm::kKS, kVS = Gm::kVS, kPair = Gm::kPair, kRows = Gm::kRows;
  constexpr bool kSepKV = Gm::kSepKV;
  constexpr int kKW = Gm::kKW, kHW = Gm::kHW, kWCols = Gm::kWCols;
  constexpr int kThreads = Gm::kThreads;
  constexpr uint32_t kColS = Gm::kColS, kColO = Gm::kColO, kTmemCols = Gm::kTmemCols;
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem<D, G>& sm =
      *reinterpret_cast<Smem<D, G>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long units = (long long)a.B * (a.Hkv / kPair) * a.splits;
  volatile int* abort = &sm.abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kKS; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < kVS; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int s = 0; s < kUnitRing; ++s) {
      mbar_init(&sm.unit_full[s], 1);
      mbar_init(&sm.unit_empty[s], 1 + 4 * kKW);  // the MMA thread and the key warps
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.qr_full[s], 1);
      mbar_init(&sm.qr_empty[s], 1);
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.s_free[s], 4 * kKW);
      mbar_init(&sm.w_full[s], 4 * kKW);  // one arrival per key warp
      mbar_init(&sm.w_free[s], 1);
      mbar_init(&sm.o_full[s], 1);
      mbar_init(&sm.o_free[s], 4 * kKW);
      for (int g = 0; g < kKW; ++g) mbar_init(&sm.vote[g][s], 4);
    }
    mbar_init(&sm.rdv, 4 * kKW);
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // Operand rows that no copy and no thread writes stay zero: the q / rho
  // tile's rows G..7 and 8+G..15, and the weight tile's rows past 4G.
  for (int x = threadIdx.x; x < (int)(sizeof(sm.qr) / 16); x += kThreads)
    reinterpret_cast<uint4*>(&sm.qr[0][0][0])[x] = make_uint4(0u, 0u, 0u, 0u);
  for (int x = threadIdx.x; x < (int)(sizeof(sm.w) / 16); x += kThreads)
    reinterpret_cast<uint4*>(&sm.w[0][0][0])[x] = make_uint4(0u, 0u, 0u, 0u);
  fence_async_smem();
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&sm.tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer: units, the group's q / rho rows, K and V blocks ----------------
    if (lane == 0) {
      long long u = blockIdx.x;  // first unit static, the rest from the counter
      uint32_t pos = 0;          // block count: position in both rings
      int last_k[kKS], last_v[kVS], last_qr[2] = {-1, -1};
      for (int s = 0; s < kKS; ++s) last_k[s] = -1;
      for (int s = 0; s < kVS; ++s) last_v[s] = -1;
      for (int ui = 0;; ++ui) {
        const int slot = ui % kUnitRing;
        if (!mbar_wait(&sm.unit_empty[slot], ((ui / kUnitRing) & 1) ^ 1, abort, a.status)) break;
        const long long uu = u < units ? u : -1;
        const int n = uu < 0 ? 0 : a.seqlens[unit_row(uu, kPair, a)];
        sm.unit_ring[slot] = uu;
        sm.unit_n[slot] = n;
        mbar_arrive(&sm.unit_full[slot]);
        if (uu < 0) break;
        const long long next = (long long)gridDim.x + (long long)atomicAdd(&g_tc_unit_next, 1ull);
        const Unit x = unit_of(uu, n, kPair, a);
        const int qs = ui & 1;
        if (!mbar_wait(&sm.qr_empty[qs], ((ui >> 1) & 1) ^ 1, abort, a.status)) break;
        mbar_expect_tx(&sm.qr_full[qs], 2 * 2 * G * 128);
        last_qr[qs] = ui >> 1;
        // Two boxes of G rows x 64 dims each for q and for rho: the two
        // 64-dim halves of one KV head's group (d = 128), or one box per
        // member of the pair into its own half, at rows 16p (d = 64).
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int mem = kPair == 2 ? h : 0;
          const int qrow = x.b * a.H + (x.kvh + mem) * G;
          uint8_t* dst = sm.qr[qs][h] + 16 * mem * 128;
          tma_load_2d(dst, &tmQ, &sm.qr_full[qs], kPair == 2 ? 0 : 64 * h, qrow);
          tma_load_2d(dst + 8 * 128, &tmR, &sm.qr_full[qs], kPair == 2 ? 0 : 64 * h, qrow);
        }
        bool ok = true;
        for (int i = 0; i < x.nblk; ++i, ++pos) {
          const int ks = pos % kKS, vs = pos % kVS;
          if constexpr (!kSepKV) {
            // One ring: K and V of the block on the V stage's barriers.
            if (!(ok = mbar_wait(&sm.v_empty[vs], ((pos / kVS) & 1) ^ 1, abort, a.status))) break;
            if (a.inject_stall && blockIdx.x == 0) continue;
            mbar_expect_tx(&sm.v_full[vs], 4 * kKeys * 128);
            last_v[vs] = (int)(pos / kVS);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int row = (x.bkv + (kPair == 2 ? h : 0)) * a.L + x.kbeg + kKeys * i;
              tma_load_2d(sm.k[ks][h], &tmK, &sm.v_full[vs], kPair == 2 ? 0 : 64 * h, row);
              tma_load_2d(sm.v[vs][h], &tmV, &sm.v_full[vs], kPair == 2 ? 0 : 64 * h, row);
            }
            continue;
          }
          if (!(ok = mbar_wait(&sm.k_empty[ks], ((pos / kKS) & 1) ^ 1, abort, a.status))) break;
          // The failure-detection test withholds CTA 0's K/V: the MMA thread's
          // bounded wait runs out and every role unwinds through the abort path.
          if (a.inject_stall && blockIdx.x == 0) continue;
          mbar_expect_tx(&sm.k_full[ks], 2 * kKeys * 128);
          last_k[ks] = (int)(pos / kKS);
          // The two 64-dim halves of the block: of one KV head (d = 128), or
          // one per member of the pair (d = 64).  Rows < 2^31 (launcher check).
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int row = (x.bkv + (kPair == 2 ? h : 0)) * a.L + x.kbeg + kKeys * i;
            tma_load_2d(sm.k[ks][h], &tmK, &sm.k_full[ks], kPair == 2 ? 0 : 64 * h, row);
          }
          if (!(ok = mbar_wait(&sm.v_empty[vs], ((pos / kVS) & 1) ^ 1, abort, a.status))) break;
          mbar_expect_tx(&sm.v_full[vs], 2 * kKeys * 128);
          last_v[vs] = (int)(pos / kVS);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int row = (x.bkv + (kPair == 2 ? h : 0)) * a.L + x.kbeg + kKeys * i;
            tma_load_2d(sm.v[vs][h], &tmV, &sm.v_full[vs], kPair == 2 ? 0 : 64 * h, row);
          }
        }
        if (!ok) break;
        u = next;
      }
      if (*abort) {  // let every copy issued here land before the CTA exits
        for (int s = 0; s < kKS; ++s)
          if (last_k[s] >= 0) mbar_drain(&sm.k_full[s], (uint32_t)(last_k[s] & 1));
        for (int s = 0; s < kVS; ++s)
          if (last_v[s] >= 0) mbar_drain(&sm.v_full[s], (uint32_t)(last_v[s] & 1));
        for (int s = 0; s < 2; ++s)
          if (last_qr[s] >= 0) mbar_drain(&sm.qr_full[s], (uint32_t)(last_qr[s] & 1));
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t pos = 0, blk = 0, ou = 0;
      bool ok = true;
      for (int ui = 0; ok; ++ui) {
        const int slot = ui % kUnitRing;
        if (!(ok = mbar_wait(&sm.unit_full[slot], (ui / kUnitRing) & 1, abort, a.status))) break;
        const long long uu = *reinterpret_cast<volatile long long*>(&sm.unit_ring[slot]);
        const int n = *reinterpret_cast<volatile int*>(&sm.unit_n[slot]);
        mbar_arrive(&sm.unit_empty[slot]);
        if (uu < 0) break;
        const Unit x = unit_of(uu, n, kPair, a);
        const int qs = ui & 1;
        if (!(ok = mbar_wait(&sm.qr_full[qs], (ui >> 1) & 1, abort, a.status))) break;
        if (x.nblk == 0) {
          mbar_arrive(&sm.qr_empty[qs]);
          continue;
        }
        const int ob = ou & 1;
        // The accumulator of two units back has been read out.
        if (!(ok = mbar_wait(&sm.o_free[ob], ((ou >> 1) & 1) ^ 1, abort, a.status))) break;
        const uint64_t bq = sdesc(smem_u32(sm.qr[qs][0]), 16, 1024);
        // Scores of block bb (ring position p): S^T = K [Q; R]^T, both K-major.
        auto issue_scores = [&](uint32_t p, uint32_t bb) -> bool {
          const int st = p % kKS, sb = bb & 1;
          if (!(kSepKV ? mbar_wait(&sm.k_full[st], (p / kKS) & 1, abort, a.status)
                       : mbar_wait(&sm.v_full[p % kVS], (p / kVS) & 1, abort, a.status)))
            return false;
          if (!mbar_wait(&sm.s_free[sb], ((bb >> 1) & 1) ^ 1, abort, a.status)) return false;
          tc_fence_after();
          const uint64_t ak = sdesc(smem_u32(sm.k[st][0]), 16, 1024);
#pragma unroll
          for (int ks = 0; ks < 128 / 16; ++ks) {  // the staged tiles are 128 dims wide
            const uint32_t oa = (ks >> 2) * (kKeys * 128) + (ks & 3) * 32;
            const uint32_t ob2 = (ks >> 2) * (kRows * 128) + (ks & 3) * 32;
            mma_ss(tmem + kColS + kRows * sb, ak + (uint64_t)(oa >> 4), bq + (uint64_t)(ob2 >> 4), idesc(kRows, 0, 0),
                   ks > 0 ? 1u : 0u);
          }
          mma_commit(&sm.s_full[sb]);
          if constexpr (kSepKV) mma_commit(&sm.k_empty[st]);  // the K block is read
          return true;
        };
        if (!(ok = issue_scores(pos, blk))) break;
        for (int i = 0; i < x.nblk; ++i) {
          const uint32_t p = pos + i, bb = blk + i;
          // The next block's scores go ahead of this block's value product.
          if (i + 1 < x.nblk) {
            if (!(ok = issue_scores(p + 1, bb + 1))) break;
          } else {
            mma_commit(&sm.qr_empty[qs]);  // every score MMA of the unit is issued
          }
          const int st = p % kVS, sb = bb & 1;
          if (!(ok = mbar_wait(&sm.v_full[st], (p / kVS) & 1, abort, a.status))) break;
          if (!(ok = mbar_wait(&sm.w_full[sb], (bb >> 1) & 1, abort, a.status))) break;
          tc_fence_after();
          // V^T as an MN-major A operand: the two 64-dim halves LBO apart,
          // 8-key groups 1024 bytes apart, 16 keys (one K step) 2048 bytes.
          const uint64_t av = sdesc(smem_u32(sm.v[st][0]), kKeys * 128, 1024);
          const uint64_t bw = sdesc(smem_u32(sm.w[sb][0]), 16, 1024);
#pragma unroll
          for (int ks = 0; ks < kKeys / 16; ++ks) {
            const uint32_t ow = (ks >> 2) * (NW * 128) + (ks & 3) * 32;
            mma_ss(tmem + kColO + NW * ob, av + (uint64_t)((ks * 2048) >> 4), bw + (uint64_t)(ow >> 4),
                   idesc(NW, 1, 0), (i > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(&sm.v_empty[st]);
          mma_commit(&sm.w_free[sb]);
        }
        if (!ok) break;
        mma_commit(&sm.o_full[ob]);
        pos += x.nblk;
        blk += x.nblk;
        ++ou;
      }
      // Every MMA issued here completes before TMEM is freed.
      mma_commit(&sm.drain);
      mbar_drain(&sm.drain, 0);
    }
  } else if (warp >= kFirstEw) {
    // ---------------- one key of every block (scores), one dim of the accumulator ----------------
    // Key warpgroup kg (warps 4 + 4 kg ..) takes kHW of the unit's heads: its
    // local head j is head hh(j) = member * G + kg * hpm + j % hpm of the unit
    // (member j / hpm), with hpm = G / kKW heads of each member.
    const int kg = (warp - kFirstEw) >> 2, q = warp & 3, r = 32 * q + lane;
    constexpr int hpm = G / kKW;
    auto hh_of = [&](int j) { return (j / hpm) * G + kg * hpm + j % hpm; };
    const uint32_t lb = tmem + ((uint32_t)(32 * q) << 16);
    const uint32_t wcol = kColO + (uint32_t)(kWCols * kg);  // this warpgroup's accumulator columns (plus NW ob)
    const float c_log2 = kLog2e / sqrtf((float)D);
    // Thread r is key r of every block and, at the end of a unit, dim
    // r % D of member r / D of the pair (d = 64) or dim r (d = 128).
    const int mem = r / D, dim = r % D;
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
    uint32_t pos = 0, blk = 0, ou = 0, rv = 0;
    // Rendezvous of all key warps (bounded like every wait).
    auto rendezvous = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.rdv);
      const bool ok = warp_wait(&sm.rdv, rv & 1, abort, a.status);
      ++rv;
      return ok;
    };
    bool ok = true;
    for (int ui = 0; ok; ++ui) {
      const int slot = ui % kUnitRing;
      if (!(ok = warp_wait(&sm.unit_full[slot], (ui / kUnitRing) & 1, abort, a.status))) break;
      const long long uu = *reinterpret_cast<volatile long long*>(&sm.unit_ring[slot]);
      const int n = *reinterpret_cast<volatile int*>(&sm.unit_n[slot]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.unit_empty[slot]);
      if (uu < 0) break;
      const Unit x = unit_of(uu, n, kPair, a);
      if (x.bad) {
        if (x.c == 0 && kg == 0) {
          const long long bh0 = (long long)x.b * a.H + (long long)(x.kvh + mem) * G;
#pragma unroll
          for (int h = 0; h < G; ++h) out[(bh0 + h) * D + dim] = __float2bfloat16(0.f);
          if (r == 0) atomicOr(a.status, kStatusBadSeqlen);
        }
        continue;
      }
      if (x.nblk == 0) continue;
      const int ob = ou & 1;
      // Per local head j: running max, omega and T of this thread's keys.
      float hm[kHW], hom[kHW], hT[kHW];
#pragma unroll
      for (int j = 0; j < kHW; ++j) {
        hm[j] = -CUDART_INF_F;
        hom[j] = 0.f;
        hT[j] = 0.f;
      }
      for (int i = 0; i < x.nblk; ++i) {
        const uint32_t p = pos + i, bb = blk + i;
        const int st = p % kVS, sb = bb & 1;
        if (!(ok = warp_wait(&sm.s_full[sb], (bb >> 1) & 1, abort, a.status))) break;
        tc_fence_after();
        uint32_t sv[kRows];
        tmem_ld_cols<kRows>(lb + kColS + kRows * sb, sv);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_free[sb]);
        const int key = x.kbeg + kKeys * i + r;
        const bool valid = key < x.kend;
        float xs[kHW], tv[kHW];
#pragma unroll
        for (int j = 0; j < kHW; ++j) {  // q of head hh in column 16 (hh / G) + hh % G, rho 8 further
          // Warpgroup 1's heads sit hpm columns after warpgroup 0's (selected,
          // so that every register index stays a constant).
          const int c0 = 16 * (j / hpm) + j % hpm;
          const uint32_t sq = kg == 0 ? sv[c0] : sv[(c0 + hpm) % kRows];
          const uint32_t sr = kg == 0 ? sv[c0 + 8] : sv[(c0 + hpm + 8) % kRows];
          xs[j] = valid ? __uint_as_float(sq) * c_log2 : -CUDART_INF_F;
          tv[j] = valid ? __uint_as_float(sr) : 0.f;
        }
        // Block max of every head over the warpgroup's four warps' keys.
        {
          const float mx = warp_max_scatter<kHW>(xs, lane);  // local head lane / (32 / kHW)
          if ((lane & (32 / kHW - 1)) == 0) sm.red[kg][sb][q][lane / (32 / kHW)] = mx;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.vote[kg][sb]);
        if (!(ok = warp_wait(&sm.vote[kg][sb], (bb >> 1) & 1, abort, a.status))) break;
        bool raised = false;
        float alpha[kHW], mb[kHW];
        block_max4<kHW>(sm.red[kg][sb], mb);
#pragma unroll
        for (int j = 0; j < kHW; ++j) {
          const bool up = mb[j] > hm[j] + kLazyTau;  // always on the unit's first block (m = -inf)
          alpha[j] = up ? exp2f(hm[j] - mb[j]) : 1.f;
          hm[j] = up ? mb[j] : hm[j];
          hom[j] *= alpha[j];
          hT[j] *= alpha[j];
          raised |= up;
        }
        if (raised && i > 0) {  // uniform over the warpgroup; rare after the first block
          // Rescale this warpgroup's accumulator columns once the previous
          // block's value MMAs are done.
          const uint32_t pb = bb - 1;
          if (!(ok = warp_wait(&sm.w_free[pb & 1], (pb >> 1) & 1, abort, a.status))) break;
          tc_fence_after();
          uint32_t ov[kWCols];
          tmem_ld_cols<kWCols>(lb + wcol + NW * ob, ov);
          tc_wait_ld();
#pragma unroll
          for (int j = 0; j < kHW; ++j) {
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) ov[4 * j + k4] = __float_as_uint(__uint_as_float(ov[4 * j + k4]) * alpha[j]);
          }
          tmem_st_cols<kWCols>(lb + wcol + NW * ob, ov);
          tc_wait_st();
          tc_fence_before();
        }
        float wv[kHW];
#pragma unroll
        for (int j = 0; j < kHW; ++j) {
          wv[j] = exp2f(xs[j] - hm[j]);
          hom[j] += wv[j];
          hT[j] += wv[j] * tv[j];
        }
        // The weight tile of two blocks back has been consumed.
        if (!(ok = warp_wait(&sm.w_free[sb], ((bb >> 1) & 1) ^ 1, abort, a.status))) break;
        uint8_t* wt = sm.w[sb][r >> 6];
        const int kk = r & 63;
#pragma unroll
        for (int j = 0; j < kHW; ++j) {
          const int row = 4 * (kHW * kg + j);
          const float w = wv[j], wtv = wv[j] * tv[j];
          const __nv_bfloat16 whi = __float2bfloat16_rn(w), thi = __float2bfloat16_rn(wtv);
          const __nv_bfloat16 wlo = __float2bfloat16_rn(w - __bfloat162float(whi));
          const __nv_bfloat16 tlo = __float2bfloat16_rn(wtv - __bfloat162float(thi));
          *reinterpret_cast<__nv_bfloat16*>(wt + sw128_elem(row + 0, kk)) = whi;
          *reinterpret_cast<__nv_bfloat16*>(wt + sw128_elem(row + 1, kk)) = wlo;
          *reinterpret_cast<__nv_bfloat16*>(wt + sw128_elem(row + 2, kk)) = thi;
          *reinterpret_cast<__nv_bfloat16*>(wt + sw128_elem(row + 3, kk)) = tlo;
        }
        // Keys past the end of the sequence carry zero weight; their V rows
        // (whatever the cache holds there, even NaN) are zeroed so that they
        // cannot turn into NaN in the product.
        if (kg == 0 && key >= x.n) {
          // (the V block's copy was issued with this block's K, long read)
          if (!mbar_wait(&sm.v_full[st], (p / kVS) & 1, abort, a.status)) ok = false;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint4* row = reinterpret_cast<uint4*>(sm.v[st][h] + r * 128);
#pragma unroll
            for (int c16 = 0; c16 < 8; ++c16) row[c16] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.w_full[sb]);
      }
      if (!ok) break;
      // ---- End of the unit: the accumulator (thread r holds dim `dim` of
      // member `mem`) and the sums.
      if (!(ok = warp_wait(&sm.o_full[ob], (ou >> 1) & 1, abort, a.status))) break;
      tc_fence_after();
      uint32_t ov[kWCols];
      tmem_ld_cols<kWCols>(lb + wcol + NW * ob, ov);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.o_free[ob]);
#pragma unroll
      for (int j = 0; j < kHW; ++j) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          hom[j] += __shfl_xor_sync(0xffffffffu, hom[j], o);
          hT[j] += __shfl_xor_sync(0xffffffffu, hT[j], o);
        }
        if (lane == 0) {
          sm.sums[kg][q][2 * j] = hom[j];
          sm.sums[kg][q][2 * j + 1] = hT[j];
        }
      }
      if (!(ok = rendezvous())) break;
      // The unit's query heads are consecutive from bh0: head hh of the unit
      // is query head bh0 + hh (member hh / G).
      const long long bh0 = (long long)x.b * a.H + (long long)x.kvh * G;
#pragma unroll
      for (int j = 0; j < kHW; ++j) {
        if (j / hpm != mem) continue;  // this thread's member (warp-uniform)
        const float om = (sm.sums[kg][0][2 * j] + sm.sums[kg][1][2 * j]) + (sm.sums[kg][2][2 * j] + sm.sums[kg][3][2 * j]);
        const float TT = (sm.sums[kg][0][2 * j + 1] + sm.sums[kg][1][2 * j + 1]) +
                         (sm.sums[kg][2][2 * j + 1] + sm.sums[kg][3][2 * j + 1]);
        const float o1 = __uint_as_float(ov[4 * j]) + __uint_as_float(ov[4 * j + 1]);
        const float o2 = __uint_as_float(ov[4 * j + 2]) + __uint_as_float(ov[4 * j + 3]);
        const long long bh = bh0 + hh_of(j);
        if (x.nch == 1) {
          const float inv = 1.f / om;
          out[bh * D + dim] = __float2bfloat16_rn(((1.f + TT * inv) * o1 - o2) * inv);
        } else {
          float* rec = a.partials + (bh * a.splits + x.c) * (2 * D + 4);
          if (dim == 0) {
            rec[0] = hm[j];
            rec[1] = om;
            rec[2] = TT;
          }
          rec[4 + dim] = o1;
          rec[4 + D + dim] = o2;
        }
      }
      if (x.nch > 1) {
        __threadfence();
        if (!(ok = rendezvous())) break;
        if (kg == 0 && r == 0) sm.last = (atomicAdd(a.counters + x.bkv, 1) == x.nch - 1);
        if (!(ok = rendezvous())) break;
        if (sm.last) {
          __threadfence();
          // One pass over the chunks with a running max, every head's record
          // of a chunk loaded at once: one L2 round trip per chunk, not one
          // per value.  This thread merges its warpgroup's heads of its member.
          float Mg[hpm], om[hpm], TT[hpm], p1[hpm], p2[hpm];
#pragma unroll
          for (int h = 0; h < hpm; ++h) {
            Mg[h] = -CUDART_INF_F;
            om[h] = TT[h] = p1[h] = p2[h] = 0.f;
          }
          for (int cc = 0; cc < x.nch; ++cc) {
            float mc[hpm], oc[hpm], tcv[hpm], q1[hpm], q2[hpm];
#pragma unroll
            for (int h = 0; h < hpm; ++h) {
              const float* rc = a.partials + ((bh0 + mem * G + kg * hpm + h) * a.splits + cc) * (2 * D + 4);
              mc[h] = __ldcg(rc);
              oc[h] = __ldcg(rc + 1);
              tcv[h] = __ldcg(rc + 2);
              q1[h] = __ldcg(rc + 4 + dim);
              q2[h] = __ldcg(rc + 4 + D + dim);
            }
#pragma unroll
            for (int h = 0; h < hpm; ++h) {
              const float Mn = fmaxf(Mg[h], mc[h]);  // finite: every chunk holds a key
              const float so = exp2f(Mg[h] - Mn), sc = exp2f(mc[h] - Mn);  // 2^-inf = 0 on the first
              om[h] = so * om[h] + sc * oc[h];
              TT[h] = so * TT[h] + sc * tcv[h];
              p1[h] = so * p1[h] + sc * q1[h];
              p2[h] = so * p2[h] + sc * q2[h];
              Mg[h] = Mn;
            }
          }
#pragma unroll
          for (int h = 0; h < hpm; ++h) {
            const float inv = 1.f / om[h];
            out[(bh0 + mem * G + kg * hpm + h) * D + dim] =
                __float2bfloat16_rn(((1.f + TT[h] * inv) * p1[h] - p2[h]) * inv);
          }
          if (kg == 0 && r == 0) a.counters[x.bkv] = 0;
        }
      }
      if (!(ok = rendezvous())) break;  // the sums and the flag are reused by the next unit
      pos += x.nblk;
      blk += x.nblk;
      ++ou;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) {
    // Every CTA fetched its last unit before this point; the last CTA to get
    // here leaves the scheduler at zero for the next launch.
    __threadfence();
    if (atomicAdd(&g_tc_cta_done, 1u) == gridDim.x - 1) {
      atomicExch(&g_tc_unit_next, 0ull);
      atomicExch(&g_tc_cta_done, 0u);
    }
  }
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

template <int D, int G>
cudaError_t launch_g(const DecodeArgs& args, cudaStream_t st, int num_sms) {
  // PLX_FAULT_INJECT=decode_stall makes one CTA's bounded waits run out (tests
  // of the timeout status only).
  DecodeArgs a = args;
  const char* fi = getenv("PLX_FAULT_INJECT");
  a.inject_stall = (fi != nullptr && strcmp(fi, "decode_stall") == 0) ? 1 : 0;
  CUtensorMap mK, mV, mQ, mR;
  const long long kv_rows = (long long)a.B * a.Hkv * a.L, q_rows = (long long)a.B * a.H;
  if (!make_map(&mK, a.K, kv_rows, kKeys, D) || !make_map(&mV, a.V, kv_rows, kKeys, D) ||
      !make_map(&mQ, a.q, q_rows, G, D) || !make_map(&mR, a.r, q_rows, G, D))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem<D, G>) + 1024;
  static_assert(sizeof(Smem<D, G>) + 1024 <= 227 * 1024, "shared memory of one CTA");
  cudaError_t e =
      cudaFuncSetAttribute(decode_gqa_tc_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long units = (long long)a.B * (a.Hkv / Geo<D, G>::kPair) * a.splits;
  const long long grid = units < num_sms ? units : num_sms;
  decode_gqa_tc_kernel<D, G><<<(unsigned)grid, Geo<D, G>::kThreads, smem, st>>>(mK, mV, mQ, mR, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_gqa_tc(const DecodeArgs& a, cudaStream_t st, int num_sms) {
  if (a.Hkv < 1 || a.H % a.Hkv != 0 || !decode_gqa_tc(a.Hkv, a.d)) return cudaErrorInvalidValue;
  if ((long long)a.B * a.Hkv * a.L + kKeys >= (1ll << 31)) return cudaErrorInvalidValue;
  const int G = a.H / a.Hkv;
  if (a.d == 128) {
    if (G == 1) return launch_g<128, 1>(a, st, num_sms);
    if (G == 2) return launch_g<128, 2>(a, st, num_sms);
    if (G == 4) return launch_g<128, 4>(a, st, num_sms);
    if (G == 8) return launch_g<128, 8>(a, st, num_sms);
  } else {
    if (G == 1) return launch_g<64, 1>(a, st, num_sms);  // two heads a unit, one query head each
    if (G == 2) return launch_g<64, 2>(a, st, num_sms);
    if (G == 4) return launch_g<64, 4>(a, st, num_sms);
    if (G == 8) return launch_g<64, 8>(a, st, num_sms);
  }
  return cudaErrorInvalidValue;
}

}  // namespace plx
