// Split-KV Parallax decode over an e4m3 KV cache (d = 128, G = H / Hkv in
// {1, 2, 4, 8}), and the quantiser that writes such a cache.
//
// Cache format: every cached key and value row of a KV head carries its own
// fp32 scale s = max|x| / 448 and 128 e4m3 codes x / s (round to nearest,
// ties to even), written when the row is appended.  That is the reading of
// the pages' "dynamic fp8" (rainbus.top summary, 复现评估: dynamic fp8 for the
// linear layers) for a cache that grows one token at a time.  A row stands
// for code * s; the decode is the Parallax decode over those values.
//
// The decode streams half the bytes of the bf16 decode (128 + 4 bytes per
// cached row instead of 256), so the same HBM stream carries twice the keys.
// The score and value products keep the bf16 decode's precision:
//   * scores, keys as the MMA's M:  S^T [128 keys x N] = K_blk B^T as e4m3
//     MMAs (kind::f8f6f4, K = 32) straight from the staged codes, with no
//     conversion.  B holds each q and rho row as three e4m3 terms
//     (hi + mid + lo, each the rounding of what the previous ones left):
//     after the row is scaled by the power of two 2^-e that brings its
//     largest element into [2^7, 2^8), three terms represent every bf16
//     element exactly down to 2^-17 of the row's largest, so the three
//     score columns of a row add up to the f32 score of the unrounded
//     operand.  The softmax threads add them, undo 2^e and apply the key's
//     scale in fp32.  N = 6G rounded up to 16.
//   * values, dims as the MMA's M:  O^T [128 dims x 4G] += V_blk^T W in bf16:
//     e4m3 codes convert exactly to bf16 (integer bit moves and one
//     multiply by a power of two), and the value row's
//     scale is folded into that key's weights (w s_v and w t s_v, each a bf16
//     hi + lo pair), so omega and T stay plain sums of w and w t.
// Roles (one persistent CTA per SM, units = (b, KV head, key chunk) from a
// global counter, as in the bf16 decode): warp 0 stages raw e4m3 K and V
// blocks by TMA; for groups of 1 and 2 warp 1 issues the score MMAs and warp 3
// the value MMAs (one issuing thread each: an issue waits for the tensor pipe
// to take the MMA, and either thread's barrier waits then overlap the other's
// issues), for larger groups warp 1 issues both; warp 2 (with warp 3 where
// that warp issues nothing) builds the q / rho operand of each unit; warps 4-7
// own one key each (scores, weights) and at the end of a unit one dim each
// (output or partial record, merged by the last CTA of a (b, KV head)); warps 8-15, two per key
// (one per 64-dim half of its V row), convert the value rows into the bf16
// value tile.
//
// Formulas: rainbus.top summary "方法步骤详情"; out = ((1 + T/omega) O1 - O2) / omega.
#include "plx_internal.cuh"
#include "sm100.cuh"
#include "decode_tc_common.cuh"

#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <math_constants.h>

#include <cstdlib>
#include <cstring>

namespace plx {
namespace {

using namespace sm100;
using namespace dtc;

constexpr int D = 128;
constexpr int kThreads = 512;
constexpr int kQrWarp = 2, kPVWarp = 3, kFirstEw = 4, kFirstCv = 8;
constexpr int kCvWarps = 8;  // two per 32 keys, each converting half of every value row
// Register split (setmaxnreg, per warpgroup): the launch gives 512 x 128; the
// control warpgroup and the two converter warpgroups hand registers to the
// key warpgroup: 128 x 96 + 128 x 208 + 256 x 88 = 61,440 <= 65,536.
constexpr int kRegsControl = 96, kRegsKey = 208, kRegsConv = 88;
constexpr int kUnitRing = 4;
constexpr int kScaleBox = kKeys + 4;   // scales per staged box (128 keys + up to 3 before them)
constexpr int kScaleBoxPad = 160;      // box rounded up to 128 bytes (a tensor copy's destination alignment)
constexpr float kLazyTau = 8.f;
constexpr float kLog2e = 1.4426950408889634f;
// TMEM columns: two score stages (N columns each) from 0, two value
// accumulators (NW columns each) from 128.
constexpr uint32_t kColS = 0, kColO = 128, kTmemCols = 256;

// Row of the score operand B holding term `term` (0 hi, 1 mid, 2 lo) of the
// q (kind 0) or rho (kind 1) row of head h of the group.
template <int G>
__host__ __device__ constexpr int brow(int term, int kind, int h) {
  return term * 2 * G + kind * G + h;
}

template <int G>
struct SmemF {
  static constexpr int NW = 4 * G < 16 ? 16 : 4 * G;
  static constexpr int NB = (6 * G + 15) / 16 * 16;  // score operand rows (the MMA's N)
  static constexpr int kStages = 4;      // raw stages in flight (as many as shared memory holds)
  uint8_t raw[kStages][2][kKeys * 128];  // e4m3 [128 keys x 128 dims]: K, V
  uint8_t vc[2][2][kKeys * 128];         // bf16 V block per buffer: [128 keys x 64 dims] per half
  uint8_t qr[2][NB * 128];               // e4m3 q / rho terms per unit slot: [NB rows x 128 dims]
  uint8_t w[2][2][NW * 128];             // bf16 weights per block slot: [NW rows x 64 keys] per half
  // Per raw stage, the K and V scales of the block's keys: a box of kScaleBox
  // floats starting at the block's first key rounded down to a 16-byte boundary.
  alignas(128) float sc[kStages][2][kScaleBoxPad];
  uint64_t raw_full[kStages], raw_empty[kStages];
  uint64_t vc_full[2], vc_free[2];
  uint64_t qr_full[2], qr_empty[2];
  uint64_t unit_full[kUnitRing], unit_empty[kUnitRing];
  uint64_t s_full[2], s_free[2], w_full[2], w_free[2];
  uint64_t o_full[2], o_free[2];
  uint64_t vote[2];
  uint64_t rdv;
  uint64_t drain;
  long long unit_ring[kUnitRing];
  int unit_n[kUnitRing];
  int qexp[2][16];  // per unit slot: e of the q row of head h (h) and of its rho row (8 + h)
  alignas(16) float red[2][4][G];  // per-warp block maxima of each head
  float sums[4][2 * G];
  int last;
  uint32_t tmem_base;
  int abort;
};

static_assert(sizeof(SmemF<8>) + 1024 <= 227 * 1024 && sizeof(SmemF<4>) + 1024 <= 227 * 1024,
              "shared memory of one CTA");

__device__ unsigned long long g_f8_unit_next;
__device__ unsigned int g_f8_cta_done;

// 4 e4m3 codes (code 0 in the low byte) -> 2 bf16x2 words, exactly, on the
// integer and FMA pipes (the conversion instructions share the XU pipe with
// the exponentials and would bound the stream).  With a code in the high byte
// of a 16-bit lane, its sign bit is bf16's sign bit, and its 4 exponent and 3
// mantissa bits shifted right by 4 land in bf16's exponent and top mantissa
// bits: the lane then holds the code's value times 2^-120 (exponent bias 7
// against 127), subnormal codes included.  One bf16x2 multiply by 2^120
// restores the value exactly.
__device__ __forceinline__ uint32_t bf16x2_times_2p120(uint32_t v) {
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&v);
  const uint32_t k = 0x7B807B80u;  // 2^120 in both lanes (exponent field 247)
  const __nv_bfloat162 r = __hmul2(a, *reinterpret_cast<const __nv_bfloat162*>(&k));
  return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ void e4m3x4_to_bf16(uint32_t x, uint32_t& lo, uint32_t& hi) {
  const uint32_t w0 = __byte_perm(x, 0u, 0x1404);  // [code1, 0, code0, 0]
  const uint32_t w1 = __byte_perm(x, 0u, 0x3424);  // [code3, 0, code2, 0]
  lo = bf16x2_times_2p120((w0 & 0x80008000u) | ((w0 & 0x7F007F00u) >> 4));
  hi = bf16x2_times_2p120((w1 & 0x80008000u) | ((w1 & 0x7F007F00u) >> 4));
}

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
    decode_fp8kv_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmKs, const __grid_constant__ CUtensorMap tmVs,
                        DecodeArgs a) {
  using Sm = SmemF<G>;
  constexpr int NW = Sm::NW;
  constexpr int kStages = Sm::kStages;
  // Small groups issue scores and values from two threads; from 4 heads a
  // group, where the key warps bound the block period, one thread issues
  // both in the order the key warps consume them (measured faster there).
  constexpr bool kSplit = G <= 2;
  // The q / rho operand is built by warp 2, and by warp 3 as well when that
  // warp issues no MMAs: kQrParts threads per operand row.
  constexpr int kQrWarps = kSplit ? 1 : 2, kQrParts = 2 * kQrWarps, kQPT = 4 / kQrParts;
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Sm& sm = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long units = (long long)a.B * a.Hkv * a.splits;
  volatile int* abort = &sm.abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.raw_full[s], 1);
      mbar_init(&sm.raw_empty[s], kCvWarps + 5);  // the converters, the key warps, the score MMAs' commit
    }
    for (int s = 0; s < kUnitRing; ++s) {
      mbar_init(&sm.unit_full[s], 1);
      // The MMA thread(s), the q / rho warp(s), 4 key warps, the converters.
      mbar_init(&sm.unit_empty[s], 7 + kCvWarps);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.vc_full[s], kCvWarps);
      mbar_init(&sm.vc_free[s], 1);
      mbar_init(&sm.qr_full[s], kQrWarps);
      mbar_init(&sm.qr_empty[s], 5);  // the MMA thread's commit and the four key warps
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.s_free[s], 4);
      mbar_init(&sm.w_full[s], 4);  // one arrival per key warp
      mbar_init(&sm.w_free[s], 1);
      mbar_init(&sm.o_full[s], 1);
      mbar_init(&sm.o_free[s], 4);
      mbar_init(&sm.vote[s], 4);
    }
    mbar_init(&sm.rdv, 4);
    mbar_init(&sm.drain, kSplit ? 2 : 1);  // one commit from each MMA issuer
    sm.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // Operand rows no thread writes stay zero: the q / rho tile's rows past 6G
  // and the weight tile's rows past 4G.
  for (int x = threadIdx.x; x < (int)(sizeof(sm.qr) / 16); x += kThreads)
    reinterpret_cast<uint4*>(&sm.qr[0][0])[x] = make_uint4(0u, 0u, 0u, 0u);
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

  // Every role but the producer reads the units in the order it publishes them.
  auto take_unit = [&](int ui, long long& uu, int& n) -> bool {
    const int slot = ui % kUnitRing;
    if (!warp_wait(&sm.unit_full[slot], (ui / kUnitRing) & 1, abort, a.status)) return false;
    uu = *reinterpret_cast<volatile long long*>(&sm.unit_ring[slot]);
    n = *reinterpret_cast<volatile int*>(&sm.unit_n[slot]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.unit_empty[slot]);
    return true;
  };

  if (warp < kFirstEw) {
  // Each warpgroup sets its share once, at the head of its branch.
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
  if (warp == 0) {
    // ---------------- TMA producer: units and raw e4m3 K / V blocks ----------------
    if (lane == 0) {
      uint32_t pos = 0;
      int last_kv[kStages];
      for (int s = 0; s < kStages; ++s) last_kv[s] = -1;
      // Units are published one ahead of their loads, so the roles that
      // prepare a unit (the q / rho operand, read from global memory behind
      // the cache stream) have the whole previous unit to do it.
      auto publish = [&](int ui, long long uu, int& n) -> bool {
        const int slot = ui % kUnitRing;
        if (!mbar_wait(&sm.unit_empty[slot], ((ui / kUnitRing) & 1) ^ 1, abort, a.status)) return false;
        n = uu < 0 ? 0 : a.seqlens[unit_row(uu, 1, a)];
        sm.unit_ring[slot] = uu;
        sm.unit_n[slot] = n;
        mbar_arrive(&sm.unit_full[slot]);
        return true;
      };
      long long uu = blockIdx.x;  // the grid never exceeds the unit count
      int n = 0;
      bool live = publish(0, uu, n);
      for (int ui = 1; live; ++ui) {
        long long nx = (long long)gridDim.x + (long long)atomicAdd(&g_f8_unit_next, 1ull);
        if (nx >= units) nx = -1;
        int nn = 0;
        if (!publish(ui, nx, nn)) break;
        const Unit x = unit_of(uu, n, 1, a);
        bool ok = true;
        for (int i = 0; i < x.nblk; ++i, ++pos) {
          const int st = pos % kStages;
          if (!(ok = mbar_wait(&sm.raw_empty[st], ((pos / kStages) & 1) ^ 1, abort, a.status))) break;
          if (a.inject_stall && blockIdx.x == 0) continue;
          mbar_expect_tx(&sm.raw_full[st], 2 * kKeys * 128 + 2 * kScaleBox * 4);
          last_kv[st] = (int)(pos / kStages);
          const int row = x.bkv * a.L + x.kbeg + kKeys * i;  // < 2^31 (launcher check)
          tma_load_2d(sm.raw[st][0], &tmK, &sm.raw_full[st], 0, row);
          tma_load_2d(sm.raw[st][1], &tmV, &sm.raw_full[st], 0, row);
          // Scales: the 1-D box must start on a 16-byte boundary (a multiple of
          // 4 floats); the key threads index from the remainder.
          tma_load_1d(sm.sc[st][0], &tmKs, &sm.raw_full[st], row & ~3);
          tma_load_1d(sm.sc[st][1], &tmVs, &sm.raw_full[st], row & ~3);
        }
        if (!ok) break;
        uu = nx;
        n = nn;
        live = uu >= 0;
      }
      if (*abort) {
        for (int s = 0; s < kStages; ++s)
          if (last_kv[s] >= 0) mbar_drain(&sm.raw_full[s], (uint32_t)(last_kv[s] & 1));
      }
    }
  } else if (warp == 1) {
    if constexpr (kSplit) {
      // ---------------- score MMA issuer ----------------
      if (lane == 0) {
        uint32_t blk = 0;
        bool ok = true;
        for (int ui = 0; ok; ++ui) {
          const int slot = ui % kUnitRing;
          if (!(ok = mbar_wait(&sm.unit_full[slot], (ui / kUnitRing) & 1, abort, a.status))) break;
          const long long uu = *reinterpret_cast<volatile long long*>(&sm.unit_ring[slot]);
          const int n = *reinterpret_cast<volatile int*>(&sm.unit_n[slot]);
          mbar_arrive(&sm.unit_empty[slot]);
          if (uu < 0) break;
          const Unit x = unit_of(uu, n, 1, a);
          const int qs = ui & 1;
          if (!(ok = mbar_wait(&sm.qr_full[qs], (ui >> 1) & 1, abort, a.status))) break;
          if (x.nblk == 0) {
            mbar_arrive(&sm.qr_empty[qs]);
            continue;
          }
          const uint64_t bq = sdesc(smem_u32(sm.qr[qs]), 16, 1024);
          // Scores of block bb: S^T = K B^T, e4m3 x e4m3, K straight from its raw
          // stage (K-major, 128-byte rows, 128B swizzle; 32 codes per K step).
          for (int i = 0; i < x.nblk; ++i) {
            const uint32_t bb = blk + i;
            const int st = bb % kStages, sb = bb & 1;
            if (!(ok = mbar_wait(&sm.raw_full[st], (bb / kStages) & 1, abort, a.status))) break;
            if (!(ok = mbar_wait(&sm.s_free[sb], ((bb >> 1) & 1) ^ 1, abort, a.status))) break;
            tc_fence_after();
            const uint64_t ak = sdesc(smem_u32(sm.raw[st][0]), 16, 1024);
  #pragma unroll
            for (int ks = 0; ks < D / 32; ++ks)
              mma_ss_f8(tmem + kColS + Sm::NB * sb, ak + (uint64_t)((ks * 32) >> 4), bq + (uint64_t)((ks * 32) >> 4),
                        idesc_e4m3(Sm::NB), ks > 0 ? 1u : 0u);
            mma_commit(&sm.s_full[sb]);
            mma_commit(&sm.raw_empty[st]);  // the K codes are read
          }
          if (!ok) break;
          mma_commit(&sm.qr_empty[qs]);  // every score MMA of the unit is issued
          blk += x.nblk;
        }
        mma_commit(&sm.drain);
        mbar_drain(&sm.drain, 0);
      }
    } else {
      // ---------------- MMA issuer: the scores of block i + 1, then the values of block i ----------------
      if (lane == 0) {
        uint32_t blk = 0, ou = 0;
        bool ok = true;
        for (int ui = 0; ok; ++ui) {
          const int slot = ui % kUnitRing;
          if (!(ok = mbar_wait(&sm.unit_full[slot], (ui / kUnitRing) & 1, abort, a.status))) break;
          const long long uu = *reinterpret_cast<volatile long long*>(&sm.unit_ring[slot]);
          const int n = *reinterpret_cast<volatile int*>(&sm.unit_n[slot]);
          mbar_arrive(&sm.unit_empty[slot]);
          if (uu < 0) break;
          const Unit x = unit_of(uu, n, 1, a);
          const int qs = ui & 1;
          if (!(ok = mbar_wait(&sm.qr_full[qs], (ui >> 1) & 1, abort, a.status))) break;
          if (x.nblk == 0) {
            mbar_arrive(&sm.qr_empty[qs]);
            continue;
          }
          const int ob = ou & 1;
          if (!(ok = mbar_wait(&sm.o_free[ob], ((ou >> 1) & 1) ^ 1, abort, a.status))) break;
          const uint64_t bq = sdesc(smem_u32(sm.qr[qs]), 16, 1024);
          // Scores of block bb: S^T = K B^T, e4m3 x e4m3, K straight from its raw
          // stage (K-major, 128-byte rows, 128B swizzle; 32 codes per K step).
          auto issue_scores = [&](uint32_t bb) -> bool {
            const int st = bb % kStages, sb = bb & 1;
            if (!mbar_wait(&sm.raw_full[st], (bb / kStages) & 1, abort, a.status)) return false;
            if (!mbar_wait(&sm.s_free[sb], ((bb >> 1) & 1) ^ 1, abort, a.status)) return false;
            tc_fence_after();
            const uint64_t ak = sdesc(smem_u32(sm.raw[st][0]), 16, 1024);
  #pragma unroll
            for (int ks = 0; ks < D / 32; ++ks)
              mma_ss_f8(tmem + kColS + Sm::NB * sb, ak + (uint64_t)((ks * 32) >> 4), bq + (uint64_t)((ks * 32) >> 4),
                        idesc_e4m3(Sm::NB), ks > 0 ? 1u : 0u);
            mma_commit(&sm.s_full[sb]);
            mma_commit(&sm.raw_empty[st]);  // the K codes are read
            return true;
          };
          if (!(ok = issue_scores(blk))) break;
          for (int i = 0; i < x.nblk; ++i) {
            const uint32_t bb = blk + i;
            if (i + 1 < x.nblk) {
              if (!(ok = issue_scores(bb + 1))) break;
            } else {
              mma_commit(&sm.qr_empty[qs]);  // every score MMA of the unit is issued
            }
            const int sb = bb & 1, vb = bb & 1;
            if (!(ok = mbar_wait(&sm.w_full[sb], (bb >> 1) & 1, abort, a.status))) break;
            if (!(ok = mbar_wait(&sm.vc_full[vb], (bb >> 1) & 1, abort, a.status))) break;
            tc_fence_after();
            // V^T as an MN-major A operand: the two 64-dim halves LBO apart,
            // 8-key groups 1024 bytes apart, 16 keys (one K step) 2048 bytes.
            const uint64_t av = sdesc(smem_u32(sm.vc[vb][0]), kKeys * 128, 1024);
            const uint64_t bw = sdesc(smem_u32(sm.w[sb][0]), 16, 1024);
  #pragma unroll
            for (int ks = 0; ks < kKeys / 16; ++ks) {
              const uint32_t ow = (ks >> 2) * (NW * 128) + (ks & 3) * 32;
              mma_ss(tmem + kColO + NW * ob, av + (uint64_t)((ks * 2048) >> 4), bw + (uint64_t)(ow >> 4),
                     idesc(NW, 1, 0), (i > 0 || ks > 0) ? 1u : 0u);
            }
            mma_commit(&sm.w_free[sb]);
            mma_commit(&sm.vc_free[vb]);
          }
          if (!ok) break;
          mma_commit(&sm.o_full[ob]);
          blk += x.nblk;
          ++ou;
        }
        mma_commit(&sm.drain);
        mbar_drain(&sm.drain, 0);
      }
    }
  } else if (kSplit && warp == kPVWarp) {
    {
      // ---------------- value MMA issuer ----------------
      if (lane == 0) {
        uint32_t blk = 0, ou = 0;
        bool ok = true;
        for (int ui = 0; ok; ++ui) {
          const int slot = ui % kUnitRing;
          if (!(ok = mbar_wait(&sm.unit_full[slot], (ui / kUnitRing) & 1, abort, a.status))) break;
          const long long uu = *reinterpret_cast<volatile long long*>(&sm.unit_ring[slot]);
          const int n = *reinterpret_cast<volatile int*>(&sm.unit_n[slot]);
          mbar_arrive(&sm.unit_empty[slot]);
          if (uu < 0) break;
          const Unit x = unit_of(uu, n, 1, a);
          if (x.nblk == 0) continue;
          const int ob = ou & 1;
          if (!(ok = mbar_wait(&sm.o_free[ob], ((ou >> 1) & 1) ^ 1, abort, a.status))) break;
          for (int i = 0; i < x.nblk; ++i) {
            const uint32_t bb = blk + i;
            const int sb = bb & 1, vb = bb & 1;
            if (!(ok = mbar_wait(&sm.w_full[sb], (bb >> 1) & 1, abort, a.status))) break;
            if (!(ok = mbar_wait(&sm.vc_full[vb], (bb >> 1) & 1, abort, a.status))) break;
            tc_fence_after();
            // V^T as an MN-major A operand: the two 64-dim halves LBO apart,
            // 8-key groups 1024 bytes apart, 16 keys (one K step) 2048 bytes.
            const uint64_t av = sdesc(smem_u32(sm.vc[vb][0]), kKeys * 128, 1024);
            const uint64_t bw = sdesc(smem_u32(sm.w[sb][0]), 16, 1024);
  #pragma unroll
            for (int ks = 0; ks < kKeys / 16; ++ks) {
              const uint32_t ow = (ks >> 2) * (NW * 128) + (ks & 3) * 32;
              mma_ss(tmem + kColO + NW * ob, av + (uint64_t)((ks * 2048) >> 4), bw + (uint64_t)(ow >> 4),
                     idesc(NW, 1, 0), (i > 0 || ks > 0) ? 1u : 0u);
            }
            mma_commit(&sm.w_free[sb]);
            mma_commit(&sm.vc_free[vb]);
          }
          if (!ok) break;
          mma_commit(&sm.o_full[ob]);
          blk += x.nblk;
          ++ou;
        }
        mma_commit(&sm.drain);
        mbar_drain(&sm.drain, 0);
      }
    }
  } else {
    // ---------------- q / rho operand of each unit (three e4m3 terms, one power-of-two scale per row) ----------------
    // q rows 0..7, rho rows 8..15 (head = row & 7), kQrParts threads a row
    // (kQPT quarters of 32 dims each).
    const int t = threadIdx.x - 32 * kQrWarp;
    const int row = t / kQrParts, hf = t % kQrParts;
    const int kind = row >> 3, head = row & 7;
    const bool live = head < G;
    bool ok = true;
    for (int ui = 0; ok; ++ui) {
      long long uu;
      int n;
      if (!(ok = take_unit(ui, uu, n))) break;
      if (uu < 0) break;
      const Unit x = unit_of(uu, n, 1, a);
      const int qs = ui & 1;
      if (!(ok = warp_wait(&sm.qr_empty[qs], ((ui >> 1) & 1) ^ 1, abort, a.status))) break;
      // The row's largest magnitude first; the conversion reads the row again
      // (from L1) a quarter at a time, which keeps this warpgroup's registers low.
      const uint4* src = reinterpret_cast<const uint4*>(
          reinterpret_cast<const __nv_bfloat16*>(kind == 0 ? a.q : a.r) +
          ((long long)x.b * a.H + (long long)x.kvh * G + head) * D + 32 * kQPT * hf);
      float m = 0.f;
      if (live) {
#pragma unroll
        for (int c = 0; c < 4 * kQPT; ++c) {
          const uint4 vc = __ldg(src + c);
          const uint32_t wd[4] = {vc.x, vc.y, vc.z, vc.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            m = fmaxf(m, fabsf(__uint_as_float(wd[k] << 16)));
            m = fmaxf(m, fabsf(__uint_as_float(wd[k] & 0xffff0000u)));
          }
        }
      }
#pragma unroll
      for (int o = 1; o < kQrParts; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      // 2^-e brings the largest element into [2^7, 2^8) (below e4m3's 448).
      const int e = (m > 0.f && m <= 3.4e38f) ? ilogbf(m) - 7 : 0;
      if (live) {
#pragma unroll
        for (int qq = 0; qq < kQPT; ++qq) {
          // Per term, the 32 codes (8 words of 4) of dims 32 (kQPT hf + qq) ..
          uint32_t tw[3][8];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 vc = __ldg(src + 4 * qq + c);
            const uint32_t wd[4] = {vc.x, vc.y, vc.z, vc.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              float2 y = make_float2(ldexpf(__uint_as_float(wd[k] << 16), -e),
                                     ldexpf(__uint_as_float(wd[k] & 0xffff0000u), -e));
#pragma unroll
              for (int term = 0; term < 3; ++term) {
                // Round what is left to e4m3 and keep the (exact) remainder.
                const __nv_fp8x2_storage_t p = __nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3);
                const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(p, __NV_E4M3);
                y.x -= __half2float(__ushort_as_half(hr.x));
                y.y -= __half2float(__ushort_as_half(hr.y));
                const int wi = 2 * c + (k >> 1);
                if ((k & 1) == 0) {
                  tw[term][wi] = (uint32_t)p;
                } else {
                  tw[term][wi] |= (uint32_t)p << 16;
                }
              }
            }
          }
          const int q4 = kQPT * hf + qq;  // 32-dim quarter: 16-byte chunks 2 q4, 2 q4 + 1
#pragma unroll
          for (int term = 0; term < 3; ++term) {
            uint8_t* dst = sm.qr[qs];
            const int rr = brow<G>(term, kind, head);
            *reinterpret_cast<uint4*>(dst + sw128_chunk(rr, 2 * q4)) =
                make_uint4(tw[term][0], tw[term][1], tw[term][2], tw[term][3]);
            *reinterpret_cast<uint4*>(dst + sw128_chunk(rr, 2 * q4 + 1)) =
                make_uint4(tw[term][4], tw[term][5], tw[term][6], tw[term][7]);
          }
        }
        if (hf == 0) sm.qexp[qs][row] = e;
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.qr_full[qs]);
    }
  }
  } else if (warp < kFirstCv) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsKey));
    // ---------------- one key of every block (scores, weights), one dim of the accumulator ----------------
    const int q = warp - kFirstEw, r = 32 * q + lane;
    const uint32_t lb = tmem + ((uint32_t)(32 * q) << 16);
    const float c_log2 = kLog2e / sqrtf((float)D);
    const int dim = r;
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
    uint32_t blk = 0, ou = 0, rv = 0;
    auto rendezvous = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.rdv);
      const bool ok = warp_wait(&sm.rdv, rv & 1, abort, a.status);
      ++rv;
      return ok;
    };
    bool ok = true;
    for (int ui = 0; ok; ++ui) {
      long long uu;
      int n;
      if (!(ok = take_unit(ui, uu, n))) break;
      if (uu < 0) break;
      const Unit x = unit_of(uu, n, 1, a);
      // The unit's row exponents (read before the operand slot is handed back).
      const int qs = ui & 1;
      if (!(ok = warp_wait(&sm.qr_full[qs], (ui >> 1) & 1, abort, a.status))) break;
      float fq[G], fr[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        fq[h] = c_log2 * ldexpf(1.f, sm.qexp[qs][h]);
        fr[h] = ldexpf(1.f, sm.qexp[qs][8 + h]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.qr_empty[qs]);
      if (x.bad) {
        if (x.c == 0) {
          const long long bh0 = (long long)x.b * a.H + (long long)x.kvh * G;
#pragma unroll
          for (int h = 0; h < G; ++h) out[(bh0 + h) * D + dim] = __float2bfloat16(0.f);
          if (r == 0) atomicOr(a.status, kStatusBadSeqlen);
        }
        continue;
      }
      if (x.nblk == 0) continue;
      const int ob = ou & 1;
      const long long srow = (long long)x.bkv * a.L;
      float hm[G], hom[G], hT[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        hm[h] = -CUDART_INF_F;
        hom[h] = 0.f;
        hT[h] = 0.f;
      }
      for (int i = 0; i < x.nblk; ++i) {
        const uint32_t bb = blk + i;
        const int sb = bb & 1, st = bb % kStages;
        const int key = x.kbeg + kKeys * i + r;
        const bool valid = key < x.kend, inside = key < x.n;
        // The key's scales from the raw stage (staged with the block's codes;
        // rows past the sequence get weight 0 whatever they hold).
        if (!(ok = warp_wait(&sm.raw_full[st], (bb / kStages) & 1, abort, a.status))) break;
        const int off = (int)((srow + x.kbeg + kKeys * i) & 3);
        const float sk = inside ? sm.sc[st][0][off + r] : 0.f;
        const float sv = inside ? sm.sc[st][1][off + r] : 0.f;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.raw_empty[st]);
        if (!(ok = warp_wait(&sm.s_full[sb], (bb >> 1) & 1, abort, a.status))) break;
        tc_fence_after();
        uint32_t sc[Sm::NB];
        tmem_ld_cols<Sm::NB>(lb + kColS + Sm::NB * sb, sc);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_free[sb]);
        float xs[G], tv[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          // hi + (mid + lo): the three terms' dot products with the key.
          const float sq = __uint_as_float(sc[brow<G>(0, 0, h)]) +
                           (__uint_as_float(sc[brow<G>(1, 0, h)]) + __uint_as_float(sc[brow<G>(2, 0, h)]));
          const float sr = __uint_as_float(sc[brow<G>(0, 1, h)]) +
                           (__uint_as_float(sc[brow<G>(1, 1, h)]) + __uint_as_float(sc[brow<G>(2, 1, h)]));
          xs[h] = valid ? sq * (sk * fq[h]) : -CUDART_INF_F;
          tv[h] = valid ? sr * (sk * fr[h]) : 0.f;
        }
        {
          const float mx = warp_max_scatter<G>(xs, lane);  // head lane / (32 / G)
          if ((lane & (32 / G - 1)) == 0) sm.red[sb][q][lane / (32 / G)] = mx;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.vote[sb]);
        if (!(ok = warp_wait(&sm.vote[sb], (bb >> 1) & 1, abort, a.status))) break;
        bool raised = false;
        float alpha[G], mb[G];
        block_max4<G>(sm.red[sb], mb);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float mblk = mb[h];
          const bool up = mblk > hm[h] + kLazyTau;
          alpha[h] = up ? exp2f(hm[h] - mblk) : 1.f;
          hm[h] = up ? mblk : hm[h];
          hom[h] *= alpha[h];
          hT[h] *= alpha[h];
          raised |= up;
        }
        if (raised && i > 0) {
          const uint32_t pb = bb - 1;
          if (!(ok = warp_wait(&sm.w_free[pb & 1], (pb >> 1) & 1, abort, a.status))) break;
          tc_fence_after();
          uint32_t ov[NW];
          tmem_ld_cols<NW>(lb + kColO + NW * ob, ov);
          tc_wait_ld();
#pragma unroll
          for (int h = 0; h < G; ++h) {
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) ov[4 * h + k4] = __float_as_uint(__uint_as_float(ov[4 * h + k4]) * alpha[h]);
          }
          tmem_st_cols<NW>(lb + kColO + NW * ob, ov);
          tc_wait_st();
          tc_fence_before();
        }
        float wv[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          wv[h] = exp2f(xs[h] - hm[h]);
          hom[h] += wv[h];
          hT[h] += wv[h] * tv[h];
        }
        if (!(ok = warp_wait(&sm.w_free[sb], ((bb >> 1) & 1) ^ 1, abort, a.status))) break;
        uint8_t* wt = sm.w[sb][r >> 6];
        const int kk = r & 63;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          // The value row's scale rides on the weights of the value product.
          const float w = wv[h] * sv, wtv = wv[h] * tv[h] * sv;
          const __nv_bfloat16 whi = __float2bfloat16_rn(w), thi = __float2bfloat16_rn(wtv);
          const __nv_bfloat16 wlo = __float2bfloat16_rn(w - __bfloat162float(whi));
          const __nv_bfloat16 tlo = __float2bfloat16_rn(wtv - __bfloat162float(thi));
          *reinterpret_cast<__nv_bfloat16*>(wt + sw128_elem(4 * h + 0, kk)) = whi;
          *reinterpret_cast<__nv_bfloat16*>(wt + sw128_elem(4 * h + 1, kk)) = wlo;
          *reinterpret_cast<__nv_bfloat16*>(wt + sw128_elem(4 * h + 2, kk)) = thi;
          *reinterpret_cast<__nv_bfloat16*>(wt + sw128_elem(4 * h + 3, kk)) = tlo;
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.w_full[sb]);
      }
      if (!ok) break;
      // ---- End of the unit: thread r holds dim r of the accumulator.
      if (!(ok = warp_wait(&sm.o_full[ob], (ou >> 1) & 1, abort, a.status))) break;
      tc_fence_after();
      uint32_t ov[NW];
      tmem_ld_cols<NW>(lb + kColO + NW * ob, ov);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.o_free[ob]);
#pragma unroll
      for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          hom[h] += __shfl_xor_sync(0xffffffffu, hom[h], o);
          hT[h] += __shfl_xor_sync(0xffffffffu, hT[h], o);
        }
        if (lane == 0) {
          sm.sums[q][2 * h] = hom[h];
          sm.sums[q][2 * h + 1] = hT[h];
        }
      }
      if (!(ok = rendezvous())) break;
      const long long bh0 = (long long)x.b * a.H + (long long)x.kvh * G;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float om = (sm.sums[0][2 * h] + sm.sums[1][2 * h]) + (sm.sums[2][2 * h] + sm.sums[3][2 * h]);
        const float TT =
            (sm.sums[0][2 * h + 1] + sm.sums[1][2 * h + 1]) + (sm.sums[2][2 * h + 1] + sm.sums[3][2 * h + 1]);
        const float o1 = __uint_as_float(ov[4 * h]) + __uint_as_float(ov[4 * h + 1]);
        const float o2 = __uint_as_float(ov[4 * h + 2]) + __uint_as_float(ov[4 * h + 3]);
        const long long bh = bh0 + h;
        if (x.nch == 1) {
          const float inv = 1.f / om;
          out[bh * D + dim] = __float2bfloat16_rn(((1.f + TT * inv) * o1 - o2) * inv);
        } else {
          float* rec = a.partials + (bh * a.splits + x.c) * (2 * D + 4);
          if (dim == 0) {
            rec[0] = hm[h];
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
        if (r == 0) sm.last = (atomicAdd(a.counters + x.bkv, 1) == x.nch - 1);
        if (!(ok = rendezvous())) break;
        if (sm.last) {
          __threadfence();
          float Mg[G], om[G], TT[G], p1[G], p2[G];
#pragma unroll
          for (int h = 0; h < G; ++h) {
            Mg[h] = -CUDART_INF_F;
            om[h] = TT[h] = p1[h] = p2[h] = 0.f;
          }
          for (int cc = 0; cc < x.nch; ++cc) {
            float mc[G], oc[G], tcv[G], q1[G], q2[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float* rc = a.partials + ((bh0 + h) * a.splits + cc) * (2 * D + 4);
              mc[h] = __ldcg(rc);
              oc[h] = __ldcg(rc + 1);
              tcv[h] = __ldcg(rc + 2);
              q1[h] = __ldcg(rc + 4 + dim);
              q2[h] = __ldcg(rc + 4 + D + dim);
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float Mn = fmaxf(Mg[h], mc[h]);
              const float so = exp2f(Mg[h] - Mn), sc = exp2f(mc[h] - Mn);
              om[h] = so * om[h] + sc * oc[h];
              TT[h] = so * TT[h] + sc * tcv[h];
              p1[h] = so * p1[h] + sc * q1[h];
              p2[h] = so * p2[h] + sc * q2[h];
              Mg[h] = Mn;
            }
          }
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float inv = 1.f / om[h];
            out[(bh0 + h) * D + dim] = __float2bfloat16_rn(((1.f + TT[h] * inv) * p1[h] - p2[h]) * inv);
          }
          if (r == 0) a.counters[x.bkv] = 0;
        }
      }
      if (!(ok = rendezvous())) break;
      blk += x.nblk;
      ++ou;
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsConv));
    // ---------------- converters: half of key r's V row to the bf16 value tile ----------------
    const int cq = warp & 3, r = 32 * cq + lane;
    const int half = (warp - kFirstCv) >> 2;  // dims 64 half .. 64 half + 63
    uint32_t pos = 0, blk = 0;
    bool ok = true;
    for (int ui = 0; ok; ++ui) {
      long long uu;
      int n;
      if (!(ok = take_unit(ui, uu, n))) break;
      if (uu < 0) break;
      const Unit x = unit_of(uu, n, 1, a);
      if (x.nblk == 0) continue;
      for (int i = 0; i < x.nblk; ++i) {
        const uint32_t p = pos + i, bb = blk + i;
        const int st = p % kStages, vb = bb & 1;
        if (!(ok = warp_wait(&sm.raw_full[st], (p / kStages) & 1, abort, a.status))) break;
        // V: 128 codes -> 128 bf16 in key row r of the value tile (rows past
        // the sequence are zeroed: the cache there may hold anything).
        if (!(ok = warp_wait(&sm.vc_free[vb], ((bb >> 1) & 1) ^ 1, abort, a.status))) break;
        const bool inside = x.kbeg + kKeys * i + r < x.n;
        const uint8_t* vr = sm.raw[st][1];
        // All four 16-code chunks of this half row are loaded before any store:
        // the stores into the bf16 tile could alias the raw stage as far as
        // the compiler knows, and would otherwise serialise the loads.  Code 0
        // converts to +0, so rows past the sequence load zeros.
        uint4 cvv[4];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          cvv[cc] = inside ? *reinterpret_cast<const uint4*>(vr + sw128_chunk(r, 4 * half + cc)) : make_uint4(0u, 0u, 0u, 0u);
        uint8_t* dst = sm.vc[vb][half];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          // dims 64 half + 16 cc .. + 15: chunks 2 cc and 2 cc + 1 of the half's tile
          uint32_t h8[8];
          e4m3x4_to_bf16(cvv[cc].x, h8[0], h8[1]);
          e4m3x4_to_bf16(cvv[cc].y, h8[2], h8[3]);
          e4m3x4_to_bf16(cvv[cc].z, h8[4], h8[5]);
          e4m3x4_to_bf16(cvv[cc].w, h8[6], h8[7]);
          *reinterpret_cast<uint4*>(dst + sw128_chunk(r, 2 * cc)) = make_uint4(h8[0], h8[1], h8[2], h8[3]);
          *reinterpret_cast<uint4*>(dst + sw128_chunk(r, 2 * cc + 1)) = make_uint4(h8[4], h8[5], h8[6], h8[7]);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sm.vc_full[vb]);
          mbar_arrive(&sm.raw_empty[st]);  // the value codes are read
        }
      }
      if (!ok) break;
      pos += x.nblk;
      blk += x.nblk;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&g_f8_cta_done, 1u) == gridDim.x - 1) {
      atomicExch(&g_f8_unit_next, 0ull);
      atomicExch(&g_f8_cta_done, 0u);
    }
  }
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

// 2-D view [rows, 128] of an e4m3 cache, boxes of 128 rows x 128 bytes, 128B swizzle.
bool make_map_e4m3(CUtensorMap* m, const void* base, long long rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D};
  cuuint32_t box[2] = {128, (cuuint32_t)kKeys};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 1-D view of a scale array of `rows` floats, boxes of kScaleBox floats
// (elements past the end read as zero).
bool make_map_scales(CUtensorMap* m, const float* base, long long rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[1] = {(cuuint64_t)rows};
  cuuint64_t strides[1] = {0};
  cuuint32_t box[1] = {(cuuint32_t)kScaleBox};
  cuuint32_t estr[1] = {1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 1, const_cast<float*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int G>
cudaError_t launch_f8(const DecodeArgs& args, cudaStream_t st, int num_sms) {
  DecodeArgs a = args;
  const char* fi = getenv("PLX_FAULT_INJECT");
  a.inject_stall = (fi != nullptr && strcmp(fi, "decode_stall") == 0) ? 1 : 0;
  CUtensorMap mK, mV, mKs, mVs;
  const long long kv_rows = (long long)a.B * a.Hkv * a.L;
  if (!make_map_e4m3(&mK, a.K, kv_rows) || !make_map_e4m3(&mV, a.V, kv_rows) ||
      !make_map_scales(&mKs, a.Kscale, kv_rows) || !make_map_scales(&mVs, a.Vscale, kv_rows))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(SmemF<G>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(decode_fp8kv_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long units = (long long)a.B * a.Hkv * a.splits;
  const long long grid = units < num_sms ? units : num_sms;
  decode_fp8kv_kernel<G><<<(unsigned)grid, kThreads, smem, st>>>(mK, mV, mKs, mVs, a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Quantiser: one warp per cache row of d = 32 * kPer values.
// ---------------------------------------------------------------------------
template <int kPer>
__global__ void __launch_bounds__(256) kv_quantize_fp8_kernel(const __nv_bfloat16* __restrict__ X,
                                                                uint8_t* __restrict__ codes,
                                                                float* __restrict__ scales, long long rows) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  constexpr int d = 32 * kPer;
  float x[kPer];
  const __nv_bfloat16* src = X + row * d + kPer * lane;
#pragma unroll
  for (int k = 0; k < kPer; ++k) x[k] = __bfloat162float(src[k]);
  float m = 0.f;
#pragma unroll
  for (int k = 0; k < kPer; ++k) m = fmaxf(m, fabsf(x[k]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float s = __fdiv_rn(m, 448.f);
  uint8_t c[kPer];
#pragma unroll
  for (int k = 0; k < kPer; k += 2) {
    const float y0 = s > 0.f ? __fdiv_rn(x[k], s) : 0.f;
    const float y1 = s > 0.f ? __fdiv_rn(x[k + 1], s) : 0.f;
    const __nv_fp8x2_storage_t p = __nv_cvt_float2_to_fp8x2(make_float2(y0, y1), __NV_SATFINITE, __NV_E4M3);
    c[k] = (uint8_t)(p & 0xffu);
    c[k + 1] = (uint8_t)(p >> 8);
  }
  uint8_t* dst = codes + row * d + kPer * lane;
#pragma unroll
  for (int k = 0; k < kPer; ++k) dst[k] = c[k];
  if (lane == 0) scales[row] = s;
}

}  // namespace

cudaError_t launch_decode_fp8kv(const DecodeArgs& a, cudaStream_t st, int num_sms) {
  if (a.d != D || a.Hkv < 1 || a.H % a.Hkv != 0 || !a.Kscale || !a.Vscale) return cudaErrorInvalidValue;
  if ((long long)a.B * a.Hkv * a.L + kKeys >= (1ll << 31)) return cudaErrorInvalidValue;
  const int G = a.H / a.Hkv;
  if (G == 1) return launch_f8<1>(a, st, num_sms);
  if (G == 2) return launch_f8<2>(a, st, num_sms);
  if (G == 4) return launch_f8<4>(a, st, num_sms);
  if (G == 8) return launch_f8<8>(a, st, num_sms);
  return cudaErrorInvalidValue;
}

cudaError_t launch_kv_quantize_fp8(const void* X, void* codes, float* scales, long long rows, int d,
                                   cudaStream_t st) {
  if (rows < 1) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (d == 128) {
    kv_quantize_fp8_kernel<4><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(X),
                                                     static_cast<uint8_t*>(codes), scales, rows);
  } else if (d == 64) {
    kv_quantize_fp8_kernel<2><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(X),
                                                     static_cast<uint8_t*>(codes), scales, rows);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace plx
