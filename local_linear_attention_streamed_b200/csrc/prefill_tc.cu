// Causal (or full) Parallax prefill for bf16, d in {64, 128}, on sm_100a tensor cores.
//
// Per CTA, one 128-query tile at a time; persistent CTAs take (b, h, tile)
// work from a global counter in head chunks, longest causal tiles first within
// a chunk (so a few heads' K/V stay in L2).  Warp roles:
//   warp 0      TMA producer: Q and R tiles, then a ring of 64-key K and V tiles
//               (128B-swizzled boxes, one mbarrier per stage and direction).
//   warp 1      TMEM owner and score MMA issuer (one elected thread):
//                 S1 = Q K^T and S2 = R K^T from ONE K tile into TMEM
//                 (rainbus.top summary, "方法步骤详情": S1 and S2 per KV block
//                 from one shared instruction stream);
//   warp 10     value MMA issuer (one elected thread): O1 += P V and
//                 O2 += (w t) V with P and w t read from TMEM and V from shared
//                 memory ("accumulate O1 and O2 in parallel").  Two issuing
//                 threads keep the tensor pipe fed while either one waits on a
//                 barrier (an MMA issue stalls until the pipe takes it).
//   warps 2..9  two softmax warpgroups taking alternate 64-key blocks; each
//               thread owns one query row (= TMEM lane): the whole row of its
//               warpgroup's blocks, and half of the output dims in the epilogue.
//               One running max and one rescale factor shared by both branches
//               (agihunt.info summary, hardware paragraph), omega = sum w,
//               T = sum w t in fp32, P = bf16(w) and bf16(w (t - c)) into a P
//               buffer, and the epilogue out = ((1 + T/omega) O1 - O2) / omega.
// TMEM (512 columns): one S stage (S1 at 0, S2 at 64: 64 fp32 columns each),
// two P buffers at 128 and 192 (bf16 pairs: bf16(w) in columns 0..31 and
// bf16(w (t - c)) in 32..63), O1 at 256 and O2 at 384 (128 fp32 columns each).
// At D = 64, O1 and O2 take 256..383 and a second S stage sits at 384 (one
// stage per softmax warpgroup).
// The scores of block g+1 are computed as soon as the softmax has loaded those
// of block g into registers, and the value MMAs of block g read P buffer g % 2,
// so the tensor pipe runs ahead of the softmax by a block instead of waiting
// for it: the two overlap without either one's latency entering the other's
// period.  Each softmax thread reads the whole row of S1 (its partner's half
// too) to take the block's row max without an exchange; the row sums are
// exchanged once per block.
//
// Centring.  The output is unchanged when every t_ij of a query is shifted by
// the same c_i (the pages' key-query difference z_ij = k_j - q_i is one such
// shift: rho_i . q_i).  The kernel keeps c_i at the running softmax mean of t,
// so that O2 = sum w (t - c) v and the combine ((1 + T/omega) O1 - O2)/omega
// stay well conditioned when one key dominates a row and |t| is large; with
// c = 0 a single bf16 rounding of w t there is amplified by |t| (tens, in
// trained models and in the rescale test).  c is set from the first block and
// moved (O2 -= delta O1 in TMEM) only when the running mean drifts by more than
// kTheta, always before the block's w (t - c) is rounded.
//
// The running max is raised only when a block's max exceeds it by more than
// 2^8 (exact: omega, T, O1 and O2 always share one scale); a raise or a centre
// move on a later block updates that row of O1 and O2 in TMEM after the
// previous value MMAs completed.  Every wait is bounded in time; a wait that
// runs out sets the device status word, stops the CTA's loops and frees its TMEM.
#include "sm100.cuh"

#include <math_constants.h>

#include <cstdlib>
#include <cstring>

namespace plx {
namespace {

constexpr int kBM = 128;                 // queries per tile
constexpr int kBN = 64;                  // keys per block
constexpr int kStages = 4;               // K/V ring depth
constexpr int kTileRing = 4;             // tile indices in flight from producer to consumers
// 12 warps in three warpgroups: {TMA, S MMA, PV MMA, idle} and two softmax
// warpgroups.  The first gives registers to the other two (setmaxnreg):
// 128 x 72 + 256 x 216 = 384 x 168, the registers the block launched with.
constexpr int kThreads = 384;
constexpr int kPVWarp = 2;
constexpr int kFirstSoftmaxWarp = 4;
constexpr int kRegsControl = 72, kRegsSoftmax = 216;
constexpr uint32_t kHalfQ = kBM * 128;       // one 64-dim half of a Q tile (128 B rows)
constexpr uint32_t kHalfKV = kBN * 128;      // one 64-dim half of a K/V block
constexpr float kLazyTau = 8.f;

// TMEM column map: the S stage, two P buffers (bf16(w) then bf16(w (t - c))
// in each), O1 (D columns from 256) and O2 (after O1).
constexpr uint32_t kColS1 = 0, kColS2 = 64, kColP = 128, kColPBuf = 64, kColPT = 32, kColO1 = 256;

// Instruction descriptors (kind::f16): D f32 (bits 4-5 = 1), A and B bf16
// (bits 7-9, 10-12 = 1), A K-major, B K-major (S) or MN-major (bit 16, PV),
// N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((kBN >> 3) << 17) | ((kBM >> 4) << 24);
// Head dimension D in {64, 128}: the tile sizes, the value MMA's N and O2's columns.
template <int D>
struct Dims {
  static constexpr int kHalves = D / 64;                // 64-dim halves (TMA boxes) per row
  static constexpr uint32_t kQBytes = kBM * D * 2;      // Q tile (also R tile)
  static constexpr uint32_t kKVBytes = kBN * D * 2;     // one K or V block
  static constexpr uint32_t kColO2 = kColO1 + D;
  // Re-centre t once its running mean drifts this far (section "Centring"
  // above).  2 at D = 128: 1.7 % on the rescale test, and 8 % faster than 1
  // (fewer O passes).  At D = 64 the rescale test gives 2.7 % (causal) with
  // 2 and 2.2 % (all keys) with 1, 1.8 % and 2.0 % with 0.5.
  static constexpr float kTheta = D == 128 ? 2.f : 0.5f;
  static constexpr uint32_t kIdescPV =
      (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((D >> 3) << 17) | ((kBM >> 4) << 24);
};

template <int D>
struct Smem {
  static constexpr uint32_t kQBytes = Dims<D>::kQBytes, kKVBytes = Dims<D>::kKVBytes;
  // Tiles first (1024-byte aligned for the 128B swizzle).
  uint8_t q[kQBytes];
  uint8_t r[kQBytes];
  uint8_t k[kStages][kKVBytes];
  uint8_t v[kStages][kKVBytes];
  uint64_t q_full, q_empty;
  // One full and one empty barrier per K/V stage: K and V of a block land
  // together, and the stage frees once that block's value MMAs completed.
  uint64_t kv_full[kStages], kv_empty[kStages];
  // Block g's scores complete on s_full[g % 2] (the barrier of the softmax
  // warpgroup that owns the block); its P on p_full[g % 2].  The S stage goes
  // back to the score issuer on s_free[0] (one stage) or s_free[g % 2] (two).
  uint64_t s_full[2], s_free[2], p_full[2];
  uint64_t o_full, o_empty, drain;
  // Row state handed from the owner of block g to the owner of block g + 1:
  // (running max, centre, the poster's own sum w, its own sum w (t - c)) in
  // the state after block g, and the flag holding the last posted g + 1.
  float4 post[2][kBM];        // [poster's warpgroup][row]
  uint32_t post_flag[2][kBM];
  // Tile indices handed from the producer to the MMA and softmax roles.
  int tile_ring[kTileRing];
  uint32_t s_issued;  // blocks whose scores were issued (all ones: no more)
  uint64_t tile_full[kTileRing], tile_empty[kTileRing];
  uint32_t tmem_base;
  int abort;
};

using namespace sm100;

struct TileInfo {
  int bh, m, j0, nblk;  // key blocks j0 .. j0 + nblk - 1 (block-sparse: list entries j0 .. j0 + nblk - 1)
};

// Tile t of the schedule: heads are taken in chunks of `ch`; within a chunk
// the tiles go longest causal rows first across the chunk's heads.  CTAs take
// tiles in this order from a global counter, so the K/V of a few heads stay in
// L2 while every tile that reads them runs, and the causal work balances.
__device__ __forceinline__ TileInfo tile_info(int t, int BH, int N, int causal, int ch, int window,
                                              const int* blk_ptr) {
  const int ntile = (N + kBM - 1) / kBM;
  const int per_chunk = ch * ntile;
  const int chunk = t / per_chunk;
  const int nh = min(ch, BH - chunk * ch);
  const int pos = t - chunk * per_chunk;
  TileInfo ti;
  ti.m = ntile - 1 - pos / nh;
  ti.bh = chunk * ch + pos % nh;
  const int kmax = causal ? min(N, (ti.m + 1) * kBM) : N;
  if (blk_ptr != nullptr) {
    // Block-sparse: the tile's active key blocks are a list (CSR row m).
    ti.j0 = blk_ptr[ti.m];
    ti.nblk = blk_ptr[ti.m + 1] - ti.j0;
    return ti;
  }
  // A sliding window of W keys: the tile's first query sees keys from m kBM - W + 1.
  ti.j0 = window > 0 ? max(0, ti.m * kBM - window + 1) / kBN : 0;
  ti.nblk = (kmax + kBN - 1) / kBN - ti.j0;
  return ti;
}

// Dynamic tile scheduler state: the next tile to hand out, and the number of
// CTAs that finished; the last CTA of a launch resets both for the next one.
__device__ unsigned int g_tile_next;
__device__ unsigned int g_cta_done;

struct Params {
  int B, H, N, causal;
  int Hkv;     // KV heads (H: one per head); query head h reads KV head h / (H / Hkv)
  int window;  // sliding window of keys per query (0: none)
  // Block-sparse (else null): per 128-query tile m, the active 64-key blocks
  // blk_idx[blk_ptr[m] .. blk_ptr[m + 1]), ascending, on or below the diagonal.
  const int* blk_ptr;
  const int* blk_idx;
  int chunk_heads;
  int inject_stall;  // failure-detection test: withhold the first Q/R tile
  __nv_bfloat16* out;
  int* status;
  // Optional outputs a backward pass needs (all null or all set): vbar = the
  // softmax mean of v (fp32), lse = log sum_j exp(s_ij) (natural log, s
  // scaled by 1/sqrt(d)) and tbar = the softmax mean of t_ij = rho_i . k_j.
  float* vbar;
  float* lse;
  float* tbar;
  // Dilation r (1: none).  With r > 1 the kernel runs B*H*r sequences of N/r
  // rows (p.N is N/r): sequence (bh, rho) holds rows rho, rho + r, rho + 2r, ...
  // of head bh, read through 3-D tensor maps [rows/r, r, d] and written back
  // to those rows, so the causal (and window) masks act within a residue
  // class: query i sees keys i, i - r, i - 2r, ...
  int dil;
};

// kMode: 0 causal or full, 1 sliding window, 2 block-sparse; kDil: dilated
// (strided 3-D loads and row mapping; modes 0 and 1).  The causal and full
// prefills compile without any of the other variants' per-row logic (a
// run-time dilation branch alone cost the causal kernel 11 %).
template <int D, int kMode, bool kDil>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmR,
                      const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  constexpr bool kWin = kMode == 1, kSparse = kMode == 2;
  // At D = 64, O1 and O2 end at column 384, so a second S stage fits in TMEM
  // (columns 384..511): each softmax warpgroup then has its own, and the
  // scores of block g + 1 need not wait until the owner of block g has read
  // its scores.  At D = 128 the 512 columns hold one stage.
  constexpr bool kTwoS = D == 64;
  static_assert(!kTwoS || kColO1 + 2 * D <= 384, "second S stage above O1, O2");
  // Rows that may see no key in a block (window or block sparsity) need the
  // guards for an empty running max.
  constexpr bool kRobust = kMode != 0;
  const int window = kWin ? p.window : 0;
  const int* blk_ptr = kSparse ? p.blk_ptr : nullptr;
  // The key block of the tile's j-th iteration.
  auto kblock = [&](const TileInfo& ti, int j) { return kSparse ? p.blk_idx[ti.j0 + j] : ti.j0 + j; };
  constexpr uint32_t kQBytes = Dims<D>::kQBytes, kKVBytes = Dims<D>::kKVBytes;
  constexpr uint32_t kColO2 = Dims<D>::kColO2, kIdescPV = Dims<D>::kIdescPV;
  constexpr int kHalves = Dims<D>::kHalves;
  Smem<D>& sm =
      *reinterpret_cast<Smem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  static_assert(!kDil || kMode != 2, "dilation with the causal or window masks");
  const int dil = kDil ? p.dil : 1;
  const int BH = p.B * p.H * dil;  // sequences (dilation: one per residue class of each head)
  const int ntile = (p.N + kBM - 1) / kBM;
  const int tiles = ntile * BH;
  volatile int* abort = &sm.abort;

  for (int x = threadIdx.x; x < 2 * kBM; x += blockDim.x) (&sm.post_flag[0][0])[x] = 0u;
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], 128);  // the owning warpgroup's threads
    }
    mbar_init(&sm.s_free[0], 4);  // one lane of each warp of the owning warpgroup
    mbar_init(&sm.s_free[1], 4);
    for (int s = 0; s < kTileRing; ++s) {
      mbar_init(&sm.tile_full[s], 1);
      mbar_init(&sm.tile_empty[s], 10);  // both MMA threads and one lane of each softmax warp
    }
    mbar_init(&sm.o_full, 1);
    mbar_init(&sm.o_empty, 256);
    mbar_init(&sm.drain, 2);  // one commit from each MMA thread
    sm.s_issued = 0;
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

  if (warp < kFirstSoftmaxWarp) {
  // The control warpgroup hands registers to the softmax warpgroups.
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t kv = 0;
      int tc = 0;
      long long kv_issued[kStages], q_issued = -1;  // last use index per stage
      for (int s = 0; s < kStages; ++s) kv_issued[s] = -1;
      for (; !*abort; ++tc) {
        const int slot = tc % kTileRing;
        if (!mbar_wait(&sm.tile_empty[slot], ((tc / kTileRing) & 1) ^ 1, abort, p.status)) break;
        const unsigned int nt = atomicAdd(&g_tile_next, 1u);
        const int t = nt < (unsigned int)tiles ? (int)nt : -1;
        sm.tile_ring[slot] = t;
        mbar_arrive(&sm.tile_full[slot]);
        if (t < 0) break;
        const TileInfo ti = tile_info(t, BH, p.N, p.causal, p.chunk_heads, window, blk_ptr);
        // Sequence ti.bh is residue class rho of head hb (rho = 0 without dilation).
        const int hb = kDil ? ti.bh / dil : ti.bh, rho = kDil ? ti.bh - hb * dil : 0;
        const int row0 = hb * p.N;
        // Grouped KV heads: consecutive query heads share one K/V head.
        const int kvrow0 = ((hb / p.H) * p.Hkv + (hb % p.H) / (p.H / p.Hkv)) * p.N;
        // Rows of a 2-D map, or (residue class, row within it) of a 3-D one.
        auto load = [&](void* dst, const CUtensorMap* map, uint64_t* bar, int x, int row) {
          if constexpr (kDil) {
            tma_load_3d(dst, map, bar, x, rho, row);
          } else {
            tma_load_2d(dst, map, bar, x, row);
          }
        };
        if (tc > 0 && !mbar_wait(&sm.q_empty, (tc - 1) & 1, abort, p.status)) break;
        mbar_expect_tx(&sm.q_full, 2 * kQBytes);
        q_issued = tc;
        // The failure-detection test withholds the first Q/R tile: its barrier
        // never completes, the MMA warp's bounded wait runs out and every role
        // unwinds through the abort path.
        if (!(p.inject_stall && tc == 0)) {
          for (int h = 0; h < kHalves; ++h) {
            load(sm.q + h * kHalfQ, &tmQ, &sm.q_full, 64 * h, row0 + ti.m * kBM);
            load(sm.r + h * kHalfQ, &tmR, &sm.q_full, 64 * h, row0 + ti.m * kBM);
          }
        }
        for (int j = 0; j < ti.nblk; ++j, ++kv) {
          const int st = kv % kStages;
          const uint32_t par = ((kv / kStages) & 1) ^ 1;
          if (!mbar_wait(&sm.kv_empty[st], par, abort, p.status)) break;
          mbar_expect_tx(&sm.kv_full[st], 2 * kKVBytes);
          kv_issued[st] = kv / kStages;
          for (int h = 0; h < kHalves; ++h) {
            load(sm.k[st] + h * kHalfKV, &tmK, &sm.kv_full[st], 64 * h, kvrow0 + kblock(ti, j) * kBN);
            load(sm.v[st] + h * kHalfKV, &tmV, &sm.kv_full[st], 64 * h, kvrow0 + kblock(ti, j) * kBN);
          }
        }
      }
      // After an abort, let every copy this thread issued land before the CTA
      // exits (each wait is bounded; consumed stages pass at once).
      if (*abort) {
        if (q_issued >= 0) mbar_drain(&sm.q_full, (uint32_t)(q_issued & 1));
        for (int s = 0; s < kStages; ++s) {
          if (kv_issued[s] >= 0) mbar_drain(&sm.kv_full[s], (uint32_t)(kv_issued[s] & 1));
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- score MMA issuer ----------------
    if (lane == 0) {
      uint32_t g = 0;  // blocks processed by this CTA = K/V ring position = S phase
      int tc = 0;
      const uint64_t dQ = sdesc(smem_u32(sm.q), 16, 1024), dR = sdesc(smem_u32(sm.r), 16, 1024);
      const uint64_t dK0 = sdesc(smem_u32(sm.k[0]), 16, 1024);
      bool ok = true;
      for (; ok; ++tc) {
        const int slot = tc % kTileRing;
        if (!(ok = mbar_wait(&sm.tile_full[slot], (tc / kTileRing) & 1, abort, p.status))) break;
        const int t = *reinterpret_cast<volatile int*>(&sm.tile_ring[slot]);
        mbar_arrive(&sm.tile_empty[slot]);
        if (t < 0) break;
        const TileInfo ti = tile_info(t, BH, p.N, p.causal, p.chunk_heads, window, blk_ptr);
        if (!(ok = mbar_wait(&sm.q_full, tc & 1, abort, p.status))) break;
        for (int j = 0; j < ti.nblk; ++j, ++g) {
          // K of this block (long resident: checked first), then the S stage,
          // free once the softmax has read the previous block's scores: the
          // wait on the critical path comes last, right before the issue.
          const uint32_t st = g % kStages;
          if (!(ok = mbar_wait(&sm.kv_full[st], (g / kStages) & 1, abort, p.status))) break;
          if constexpr (kTwoS) {
            if (g > 1 && !(ok = mbar_wait(&sm.s_free[g & 1], ((g >> 1) & 1) ^ 1, abort, p.status))) break;
          } else {
            if (g > 0 && !(ok = mbar_wait(&sm.s_free[0], (g - 1) & 1, abort, p.status))) break;
          }
          tc_fence_after();
          const uint32_t sst = kTwoS ? (g & 1) * 384u : 0u;  // the S stage of block g
          const uint64_t dk = dK0 + (uint64_t)(st * (kKVBytes >> 4));
          // S1 and S2 k-steps interleaved (one B tile feeds both GEMMs); every
          // MMA comes from the descriptors built once plus a compile-time
          // offset in the start-address field (shared-memory addresses
          // < 256 KB keep that 14-bit field from carrying).
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint64_t off = (uint64_t)((((ks >> 2) * kHalfQ) + (ks & 3) * 32) >> 4);
            const uint64_t koff = (uint64_t)((((ks >> 2) * kHalfKV) + (ks & 3) * 32) >> 4);
            mma_ss(tmem + kColS1 + sst, dQ + off, dk + koff, kIdescS, ks > 0);
            mma_ss(tmem + kColS2 + sst, dR + off, dk + koff, kIdescS, ks > 0);
          }
          mma_commit(&sm.s_full[g & 1]);
          if (j + 1 == ti.nblk) mma_commit(&sm.q_empty);
          *reinterpret_cast<volatile uint32_t*>(&sm.s_issued) = g + 1;
        }
      }
      // No more scores: the value issuer stops waiting for them.
      *reinterpret_cast<volatile uint32_t*>(&sm.s_issued) = 0xFFFFFFFFu;
      mma_commit(&sm.drain);
      mbar_drain(&sm.drain, 0);
    }
  } else if (warp == kPVWarp) {
    // ---------------- value MMA issuer ----------------
    // The scores of the next blocks are the critical path (the single S stage
    // frees only when the softmax has loaded the previous block), so the
    // value MMAs of block k go into the tensor pipe only behind the scores of
    // block k + 2: issuing stalls while the pipe is full, so issue order is
    // the order the pipe works in.  (The scores never wait on these values:
    // the softmax waits for block k's before it overwrites P buffer k % 2.)
    if (lane == 0) {
      uint32_t g = 0;
      int tc = 0;
      const uint64_t dV0 = sdesc(smem_u32(sm.v[0]), kHalfKV, 1024);
      const uint32_t oa1 = tmem + kColO1, oa2 = tmem + kColO2;
      bool ok = true;
      for (; ok; ++tc) {
        const int slot = tc % kTileRing;
        if (!(ok = mbar_wait(&sm.tile_full[slot], (tc / kTileRing) & 1, abort, p.status))) break;
        const int t = *reinterpret_cast<volatile int*>(&sm.tile_ring[slot]);
        mbar_arrive(&sm.tile_empty[slot]);
        if (t < 0) break;
        const TileInfo ti = tile_info(t, BH, p.N, p.causal, p.chunk_heads, window, blk_ptr);
        // The epilogue of the previous tile must have read O before it is overwritten.
        if (tc > 0 && !(ok = mbar_wait(&sm.o_empty, (tc - 1) & 1, abort, p.status))) break;
        for (int j = 0; j < ti.nblk; ++j, ++g) {
          const uint32_t b = g & 1;
          if (!(ok = mbar_wait(&sm.p_full[b], (g >> 1) & 1, abort, p.status))) break;
          // Behind the scores of block g + 2 (bounded in time like every wait).
          if ((int)(*reinterpret_cast<volatile uint32_t*>(&sm.s_issued) - (g + 3)) < 0) {
            const unsigned long long t0 = now_ns();
            while ((int)(*reinterpret_cast<volatile uint32_t*>(&sm.s_issued) - (g + 3)) < 0 &&
                   *reinterpret_cast<volatile uint32_t*>(&sm.s_issued) != 0xFFFFFFFFu) {
              if (*abort) {
                ok = false;
                break;
              }
              if (now_ns() - t0 > kWaitNs) {
                *abort = 1;
                atomicOr(p.status, kStatusTimeout);
                ok = false;
                break;
              }
              __nanosleep(32);
            }
            if (!ok) break;
          }
          tc_fence_after();
          const uint32_t st = g % kStages;
          const uint64_t dv = dV0 + (uint64_t)(st * (kKVBytes >> 4));
          const uint32_t pbase = tmem + kColP + b * kColPBuf;
          const uint32_t first = (j == 0) ? 0u : 1u;
#pragma unroll
          for (int ks = 0; ks < kBN / 16; ++ks) {
            const uint64_t bv = dv + (uint64_t)((ks * 2048) >> 4);
            const uint32_t acc = ks > 0 ? 1u : first;
            mma_ts(oa1, pbase + ks * 8, bv, kIdescPV, acc);
            mma_ts(oa2, pbase + kColPT + ks * 8, bv, kIdescPV, acc);
          }
          // Frees the K/V stage and P buffer b.
          mma_commit(&sm.kv_empty[st]);
        }
        if (!ok) break;
        mma_commit(&sm.o_full);
      }
      // Drain: all MMAs this thread issued complete before TMEM is freed.
      mma_commit(&sm.drain);
      mbar_drain(&sm.drain, 0);
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ---------------- softmax / epilogue: two warpgroups ----------------
    // Warpgroup wg owns the blocks g with g % 2 == wg: each thread takes the
    // whole 64-key row of its query (TMEM lane) for those blocks, while the
    // other warpgroup works on the neighbouring blocks.  The row state passes
    // from block to block through a post per block: the lazy max m and the
    // centre c are the same for both warpgroups, and each keeps its own sums
    // (omega, T) in that state.  The epilogue writes output dims 64wg..64wg+63.
    const int wg = (warp - kFirstSoftmaxWarp) >> 2;
    const int row = 32 * (warp & 3) + lane;  // TMEM lane == query row within the tile
    const uint32_t sb = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    const float scale = 1.4426950408889634f * rsqrtf((float)D);
    uint32_t gb = 0;  // the CTA's block counter at the current tile's first block
    int tc = 0;
    bool ok = true;
    // The epilogue out = ((1 + T/omega) O1 - O2) / omega for dims 64wg.. of one
    // row of tile etc: inv = 1/omega, c1 = (1 + T/omega)/omega.
    auto epilogue = [&](int etc, __nv_bfloat16* orow, float* vrow, float inv, float c1) -> bool {
      if (!mbar_wait(&sm.o_full, etc & 1, abort, p.status)) return false;
      tc_fence_after();
#pragma unroll 1
      for (int c0 = (D / 2) * wg; c0 < (D / 2) * wg + D / 2; c0 += 32) {
        uint32_t o1[32], o2[32];
        tmem_ld32(sb + kColO1 + c0, o1);
        tmem_ld32(sb + kColO2 + c0, o2);
        tc_wait_ld();
        if (orow != nullptr) {
          uint32_t packed[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float v0 = c1 * __uint_as_float(o1[2 * c]) - inv * __uint_as_float(o2[2 * c]);
            const float v1 = c1 * __uint_as_float(o1[2 * c + 1]) - inv * __uint_as_float(o2[2 * c + 1]);
            packed[c] = pack_bf16(v0, v1);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            dst[c] = make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
        }
        if (vrow != nullptr) {
          float4* dst = reinterpret_cast<float4*>(vrow + c0);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            dst[c] = make_float4(inv * __uint_as_float(o1[4 * c]), inv * __uint_as_float(o1[4 * c + 1]),
                                 inv * __uint_as_float(o1[4 * c + 2]), inv * __uint_as_float(o1[4 * c + 3]));
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.o_empty);
      return true;
    };
    // The warpgroup that did not own a tile's last block defers that tile's
    // epilogue until it has handled its first block of the next tile (its own
    // by parity), so the scores keep flowing across the tile boundary.
    bool epi_pending = false;
    int epi_tc = 0;
    __nv_bfloat16* epi_row = nullptr;
    float* epi_vrow = nullptr;
    float epi_inv = 0.f, epi_c1 = 0.f;
    for (; ok; ++tc) {
      const int slot = tc % kTileRing;
      if (!(ok = mbar_wait(&sm.tile_full[slot], (tc / kTileRing) & 1, abort, p.status))) break;
      const int t = *reinterpret_cast<volatile int*>(&sm.tile_ring[slot]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.tile_empty[slot]);
      if (t < 0) {
        if (epi_pending) ok = epilogue(epi_tc, epi_row, epi_vrow, epi_inv, epi_c1);
        break;
      }
      const TileInfo ti = tile_info(t, BH, p.N, p.causal, p.chunk_heads, window, blk_ptr);
      const int i = ti.m * kBM + row;                      // query position
      const int kend = p.causal ? min(i + 1, p.N) : p.N;  // keys < kend are visible
      const int kbeg = i - window + 1;                    // and, with a window, keys >= kbeg
      // Row state: running max (log2 units) and centre c (shared), this
      // warpgroup's omega = sum w and T = sum w (t - c), and the other
      // warpgroup's sums as last posted (brought to the current state).
      float m_run = -CUDART_INF_F, cen = 0.f, omega = 0.f, T = 0.f, om_o = 0.f, T_o = 0.f;
      // Brings this warpgroup's sums from its copy of the state to a posted one
      // (the max only rises; a raise rescales, then the centre moves).
      auto adopt = [&](const float4 ps) {
        if (ps.x > m_run) {
          const float a = ex2(m_run - ps.x);  // 0 while m_run = -inf
          omega *= a;
          T *= a;
          m_run = ps.x;
        }
        T -= (ps.y - cen) * omega;
        cen = ps.y;
      };
      for (int j = ((gb & 1u) == (uint32_t)wg) ? 0 : 1; j < ti.nblk; j += 2) {
        const uint32_t g = gb + j;
        if (!(ok = mbar_wait(&sm.s_full[wg], (g >> 1) & 1, abort, p.status))) break;
        tc_fence_after();
        const int kb = kblock(ti, j) * kBN;
        uint32_t x[64], y[64];
        const uint32_t ss = sb + (kTwoS ? (uint32_t)wg * 384u : 0u);  // this block's S stage
        tmem_ld32(ss + kColS1, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
        tmem_ld32(ss + kColS1 + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
        tmem_ld32(ss + kColS2, *reinterpret_cast<uint32_t(*)[32]>(&y[0]));
        tmem_ld32(ss + kColS2 + 32, *reinterpret_cast<uint32_t(*)[32]>(&y[32]));
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_free[kTwoS ? wg : 0]);  // the S stage goes back to the MMA
        if ((p.causal && kb + kBN - 1 > ti.m * kBM) || kb + kBN > p.N ||
            (kWin && kb < ti.m * kBM + kBM - window)) {
          // Block-uniform: only blocks that cross the diagonal, the end or the
          // window's start.
          if constexpr (kWin) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (kb + c >= kend || kb + c < kbeg) x[c] = __float_as_uint(-CUDART_INF_F);
          } else {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (kb + c >= kend) x[c] = __float_as_uint(-CUDART_INF_F);
          }
        }
        float rmax;
        {
          float m4[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              m4[q] = max3(m4[q], __uint_as_float(x[c + 2 * q]), __uint_as_float(x[c + 2 * q + 1]));
          }
          rmax = fmaxf(max3(m4[0], m4[1], m4[2]), m4[3]);
        }
        // The state after block g - 1 (the other warpgroup's), except on the
        // tile's first block.
        if (j > 0) {
          if (!(ok = flag_await(&sm.post_flag[wg ^ 1][row], g, abort, p.status))) break;
          const float4 ps = sm.post[wg ^ 1][row];
          adopt(ps);
          om_o = ps.z;
          T_o = ps.w;
        }
        // Raise the max by more than 2^8 only (always on a tile's first block).
        const float mx = rmax * scale;
        float alpha = 1.f;
        if (mx > m_run + kLazyTau) {
          alpha = ex2(m_run - mx);  // 0 on the first block
          m_run = mx;
          omega *= alpha;
          T *= alpha;
          om_o *= alpha;
          T_o *= alpha;
        }
        // w = 2^(s*scale - m_run), a = w (t - c).  x <- w, y <- a.
        float wb, tb;
        {
          // A row that has seen no key yet (only with a window) keeps m_run =
          // -inf and gets w = 2^(-inf) = 0 from the reference 0.
          const float mref = (kRobust && m_run == -CUDART_INF_F) ? 0.f : m_run;
          const uint64_t sc2 = f2(scale, scale), nm2 = f2(-mref, -mref), nc2 = f2(-cen, -cen);
          uint64_t ws2a = f2(0.f, 0.f), ts2a = f2(0.f, 0.f), ws2b = ws2a, ts2b = ts2a;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            float s0, s1;
            uf2(fma2(f2(__uint_as_float(x[2 * c]), __uint_as_float(x[2 * c + 1])), sc2, nm2), s0, s1);
            const float w0 = ex2(s0), w1 = ex2(s1);
            const uint64_t w2 = f2(w0, w1);
            const uint64_t a2 = mul2(w2, add2(f2(__uint_as_float(y[2 * c]), __uint_as_float(y[2 * c + 1])), nc2));
            if (c & 1) {
              ws2b = add2(ws2b, w2);
              ts2b = add2(ts2b, a2);
            } else {
              ws2a = add2(ws2a, w2);
              ts2a = add2(ts2a, a2);
            }
            float a0, a1;
            uf2(a2, a0, a1);
            x[2 * c] = __float_as_uint(w0);
            x[2 * c + 1] = __float_as_uint(w1);
            y[2 * c] = __float_as_uint(a0);
            y[2 * c + 1] = __float_as_uint(a1);
          }
          float lo, hi;
          uf2(add2(ws2a, ws2b), lo, hi);
          wb = lo + hi;
          uf2(add2(ts2a, ts2b), lo, hi);
          tb = lo + hi;
        }
        // Re-centre before this block's w (t - c) is rounded to bf16, on the
        // first block and whenever the running mean of t - c (both warpgroups'
        // sums through this block) has drifted by more than kTheta.
        float delta = 0.f;
        {
          // The centre is set by the row's first block with weight (the tile's
          // first block unless a window hides it) and moved on drift.  A window
          // that starts inside the previous block left that first estimate
          // from a few keys: the row's second block re-centres unconditionally.
          // Rows of short windows see few keys, so they track the mean more
          // closely (drift 0.5 below 256 keys: 1.6 % on a 37-key window where
          // the causal kernel's threshold gives 3.7 %); from 256 keys on the
          // causal threshold holds (1.5-1.9 % at 256..1024) and moves O less.
          const float Wp = omega + om_o;
          const float Tn = (T + T_o) + tb, Wn = Wp + wb;
          bool recentre;
          if constexpr (kWin) {
            const bool second = kbeg > kb - kBN && kbeg < kb;
            const float theta = window >= 256 ? Dims<D>::kTheta : 0.5f;
            recentre = Wn > 0.f && (Wp == 0.f || second || fabsf(Tn) > theta * Wn);
          } else if constexpr (kSparse) {
            // Rows of a sparse tile may start from a partial (diagonal) block.
            recentre = Wn > 0.f && (Wp == 0.f || fabsf(Tn) > 0.5f * Wn);
          } else {
            recentre = j == 0 || fabsf(Tn) > Dims<D>::kTheta * Wn;  // key 0 is visible: Wn > 0
          }
          if (recentre) {
            const float cn = cen + Tn / Wn;
            delta = cn - cen;  // the shift as represented
            cen = cn;
            T -= delta * omega;
            T_o -= delta * om_o;
            tb -= delta * wb;
          }
        }
        omega += wb;
        T += tb;
        // Hand the state after this block to the owner of block g + 1.
        sm.post[wg][row] = make_float4(m_run, cen, omega, T);
        flag_post(&sm.post_flag[wg][row], g + 1);
        // Rows whose max rose or whose centre moved update O1 and O2 (all 128
        // dims: O1 <- alpha O1, O2 <- alpha (O2 - delta O1)) once the value MMAs
        // of block g - 1 are complete.
        if (__any_sync(0xffffffffu, j > 0 && (alpha != 1.f || delta != 0.f))) {
          // The value MMAs of block g - 1 completed when its K/V stage was freed
          // (the block counter equals the K/V ring position).
          const uint32_t gp = g - 1;
          if (!(ok = mbar_wait(&sm.kv_empty[gp % kStages], (gp / kStages) & 1, abort, p.status))) break;
          tc_fence_after();
          const float ad = alpha * delta;
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 16) {
            uint32_t o1[16], o2[16];
            const uint32_t a1 = sb + kColO1 + c0, a2 = sb + kColO2 + c0;
            tmem_ld16(a1, o1);
            tmem_ld16(a2, o2);
            tc_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float v1 = __uint_as_float(o1[c]);
              o2[c] = __float_as_uint(alpha * __uint_as_float(o2[c]) - ad * v1);
              o1[c] = __float_as_uint(alpha * v1);
            }
            tmem_st16(a1, o1);
            tmem_st16(a2, o2);
            tc_wait_st();
          }
        }
        // P buffer wg (= g % 2) is free once the value MMAs of block g - 2, its
        // last reader, completed (the MMA issuer runs them after the scores).
        if (g >= 2) {
          const uint32_t gq = g - 2;
          if (!(ok = mbar_wait(&sm.kv_empty[gq % kStages], (gq / kStages) & 1, abort, p.status))) break;
          tc_fence_after();
        }
        const uint32_t pb = sb + kColP + (uint32_t)wg * kColPBuf;
        // bf16(w (t - c)) is a - delta w with the centre settled above.
        const bool moved = __any_sync(0xffffffffu, delta != 0.f);
        const uint64_t nd2 = f2(-delta, -delta);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t P[16], PT[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int e = 32 * h + 2 * c;
            P[c] = pack_bf16(__uint_as_float(x[e]), __uint_as_float(x[e + 1]));
            float a0 = __uint_as_float(y[e]), a1 = __uint_as_float(y[e + 1]);
            if (moved) uf2(fma2(f2(__uint_as_float(x[e]), __uint_as_float(x[e + 1])), nd2, f2(a0, a1)), a0, a1);
            PT[c] = pack_bf16(a0, a1);
          }
          tmem_st16(pb + 16 * h, P);
          tmem_st16(pb + kColPT + 16 * h, PT);
        }
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(&sm.p_full[wg]);
        if (epi_pending) {
          if (!(ok = epilogue(epi_tc, epi_row, epi_vrow, epi_inv, epi_c1))) break;
          epi_pending = false;
        }
      }
      if (!ok) break;
      if (epi_pending) {  // not reached: a pending epilogue's next tile starts with this warpgroup
        if (!(ok = epilogue(epi_tc, epi_row, epi_vrow, epi_inv, epi_c1))) break;
        epi_pending = false;
      }
      // ---- epilogue: out = ((1 + T/omega) O1 - O2) / omega, dims 64wg.. of this row,
      // with omega and T the sums of both warpgroups in the final state.
      const int jl = ti.nblk - 1;
      if (((gb + jl) & 1u) == (uint32_t)wg) {
        omega += om_o;  // this warpgroup owned the last block
        T += T_o;
      } else {
        if (!(ok = flag_await(&sm.post_flag[wg ^ 1][row], gb + jl + 1, abort, p.status))) break;
        const float4 ps = sm.post[wg ^ 1][row];
        adopt(ps);
        omega += ps.z;
        T += ps.w;
      }
      const bool owner_last = ((gb + ti.nblk - 1) & 1u) == (uint32_t)wg;
      gb += ti.nblk;
      const float inv = 1.f / omega;
      const float c1 = (1.f + T * inv) * inv;
      // The output row: row i of the sequence, or of its residue class.
      long long grow = (long long)ti.bh * p.N + i;
      if constexpr (kDil) {
        const int ohb = ti.bh / dil, orho = ti.bh - ohb * dil;
        grow = (long long)ohb * p.N * dil + orho + (long long)dil * i;
      }
      __nv_bfloat16* orow = i < p.N ? p.out + grow * D : nullptr;
      float* vrow = (i < p.N && p.vbar != nullptr) ? p.vbar + grow * D : nullptr;
      if (vrow != nullptr && wg == 0) {
        // lse in natural-log units of the 1/sqrt(d)-scaled scores (m_run and
        // the exponents are in log2 units), tbar = c + T/omega.
        p.lse[grow] = (m_run + log2f(omega)) * 0.6931471805599453f;
        p.tbar[grow] = cen + T * inv;
      }
      if (owner_last) {
        if (!(ok = epilogue(tc, orow, vrow, inv, c1))) break;
      } else {
        epi_pending = true;
        epi_tc = tc;
        epi_row = orow;
        epi_vrow = vrow;
        epi_inv = inv;
        epi_c1 = c1;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) {
    // Every CTA fetched its last tile before this point; the last CTA to get
    // here leaves the scheduler at zero for the next launch.
    __threadfence();
    if (atomicAdd(&g_cta_done, 1u) == gridDim.x - 1) {
      atomicExch(&g_tile_next, 0u);
      atomicExch(&g_cta_done, 0u);
    }
  }
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

}  // namespace

namespace {

template <int D>
cudaError_t launch_d(const PrefillArgs& a, cudaStream_t st, int num_sms) {
  const long long rows = (long long)a.B * a.H * a.N;
  const long long kv_rows = (long long)a.B * (a.Hkv > 0 ? a.Hkv : a.H) * a.N;
  if (rows >= (1ll << 31)) return cudaErrorInvalidValue;
  const int dil = a.dilation > 1 ? a.dilation : 1;
  if (a.N % dil != 0 || (dil > 1 && (a.blk_ptr != nullptr || a.vbar != nullptr))) return cudaErrorInvalidValue;
  const int n = a.N / dil;  // rows per sequence the kernel runs
  CUtensorMap mQ, mR, mK, mV;
  if (dil == 1) {
    if (!make_map(&mQ, a.Q, rows, kBM, D) || !make_map(&mR, a.R, rows, kBM, D) ||
        !make_map(&mK, a.K, kv_rows, kBN, D) || !make_map(&mV, a.V, kv_rows, kBN, D))
      return cudaErrorInvalidValue;
  } else {
    if (!make_map_strided(&mQ, a.Q, rows, dil, kBM, D) || !make_map_strided(&mR, a.R, rows, dil, kBM, D) ||
        !make_map_strided(&mK, a.K, kv_rows, dil, kBN, D) || !make_map_strided(&mV, a.V, kv_rows, dil, kBN, D))
      return cudaErrorInvalidValue;
  }
  const int ntile = (n + kBM - 1) / kBM;
  const int seqs = a.B * a.H * dil;
  int ch = (2 * num_sms + ntile - 1) / ntile;  // about two waves of tiles per chunk
  ch = ch < 1 ? 1 : (ch > seqs ? seqs : ch);
  // PLX_FAULT_INJECT=prefill_stall makes the kernel's bounded waits run out
  // (tests of the timeout status only).
  const char* fi = getenv("PLX_FAULT_INJECT");
  const int inject = (fi != nullptr && strcmp(fi, "prefill_stall") == 0) ? 1 : 0;
  Params p{a.B,      a.H,    n, a.causal, a.Hkv > 0 ? a.Hkv : a.H, a.window, a.blk_ptr, a.blk_idx, ch, inject,
           reinterpret_cast<__nv_bfloat16*>(a.out), a.status,
           reinterpret_cast<float*>(a.vbar), a.lse, a.tbar, dil};
  const size_t smem = sizeof(Smem<D>) + 1024;
  auto kernel = a.blk_ptr != nullptr ? prefill_tc_kernel<D, 2, false>
                : dil > 1 ? (a.window > 0 ? prefill_tc_kernel<D, 1, true> : prefill_tc_kernel<D, 0, true>)
                          : (a.window > 0 ? prefill_tc_kernel<D, 1, false> : prefill_tc_kernel<D, 0, false>);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long tiles = (long long)ntile * seqs;
  const int grid = (int)(tiles < num_sms ? tiles : num_sms);
  kernel<<<grid, kThreads, smem, st>>>(mQ, mR, mK, mV, p);
  return cudaGetLastError();
}

}  // namespace

bool prefill_tc_supported(int d) { return d == 64 || d == 128; }

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t st, int num_sms) {
  if (a.d == 128) return launch_d<128>(a, st, num_sms);
  if (a.d == 64) return launch_d<64>(a, st, num_sms);
  return cudaErrorInvalidValue;
}

}  // namespace plx
