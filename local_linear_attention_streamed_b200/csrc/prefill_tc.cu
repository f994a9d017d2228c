// Causal (or full) Parallax prefill for bf16, d = 128, on sm_100a tensor cores.
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
//   warps 2..9  two softmax warpgroups, each thread = one half (32 keys of every
//               block, 64 output dims) of one query row (= TMEM lane): one running
//               max and one rescale factor shared by both branches (agihunt.info
//               summary, hardware paragraph), omega = sum w, T = sum w t in fp32,
//               P = bf16(w) and bf16(w (t - c)) into a P buffer, and the
//               epilogue out = ((1 + T/omega) O1 - O2) / omega.
// TMEM (512 columns): one S stage (S1 at 0, S2 at 64: 64 fp32 columns each),
// two P buffers at 128 and 192 (bf16 pairs: bf16(w) in columns 0..31 and
// bf16(w (t - c)) in 32..63), O1 at 256 and O2 at 384 (128 fp32 columns each).
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
#include "plx_internal.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <math_constants.h>

#include <cstdlib>
#include <cstring>

namespace plx {
namespace {

constexpr int kD = 128;
constexpr int kBM = 128;                 // queries per tile
constexpr int kBN = 64;                  // keys per block
constexpr int kStages = 4;               // K/V ring depth
constexpr int kTileRing = 4;             // tile indices in flight from producer to consumers
constexpr int kThreads = 352;            // 11 warps: TMA, S MMA, 2 softmax warpgroups, PV MMA
constexpr int kPVWarp = 10;
constexpr uint32_t kQBytes = kBM * kD * 2;   // 32 KiB (Q tile, also R tile)
constexpr uint32_t kKVBytes = kBN * kD * 2;  // 16 KiB (one K or V block)
constexpr uint32_t kHalfQ = kBM * 128;       // one 64-dim half of a Q tile (128 B rows)
constexpr uint32_t kHalfKV = kBN * 128;      // one 64-dim half of a K/V block
constexpr float kLazyTau = 8.f;
constexpr float kTheta = 2.f;  // re-centre t once its running mean drifts this far
constexpr unsigned long long kWaitNs = 2000000000ull;  // 2 s bound on every wait

// TMEM column map: the S stage, two P buffers (bf16(w) then bf16(w (t - c))
// in each), O1 and O2.
constexpr uint32_t kColS1 = 0, kColS2 = 64, kColP = 128, kColPBuf = 64, kColPT = 32, kColO1 = 256,
                   kColO2 = 384;

// Instruction descriptors (kind::f16): D f32 (bits 4-5 = 1), A and B bf16
// (bits 7-9, 10-12 = 1), A K-major, B K-major (S) or MN-major (bit 16, PV),
// N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((kBN >> 3) << 17) | ((kBM >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((kD >> 3) << 17) |
                              ((kBM >> 4) << 24);

struct Smem {
  // Tiles first (1024-byte aligned for the 128B swizzle).
  uint8_t q[kQBytes];
  uint8_t r[kQBytes];
  uint8_t k[kStages][kKVBytes];
  uint8_t v[kStages][kKVBytes];
  uint64_t q_full, q_empty;
  // One full and one empty barrier per K/V stage: K and V of a block land
  // together, and the stage frees once that block's value MMAs completed.
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full, s_free, p_full[2];
  uint64_t o_full, o_empty, drain;
  // Row-sum exchange between the two softmax warpgroups, double-buffered by
  // epoch parity: one 64-bit word per slot holds (sum w, sum w (t - c)), with
  // the sign bit of sum w (never negative) carrying the epoch tag.
  unsigned long long xch[2][2][kBM];  // [epoch & 1][warpgroup][row]
  // Tile indices handed from the producer to the MMA and softmax roles.
  int tile_ring[kTileRing];
  uint64_t tile_full[kTileRing], tile_empty[kTileRing];
  uint32_t tmem_base;
  int abort;
};

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

// Slow path of mbar_wait (kept out of line so that the common, already
// complete case costs one try_wait and no call).
__device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, volatile int* abort,
                                            int* status) {
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

// Bounded wait for the phase of `parity` to complete.  Returns false (and
// raises the CTA's abort flag and the device timeout status) if it ran out,
// or false at once if another role already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int* status) {
  if (mbar_test(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, abort, status);
}

// Pairwise exchange between the two threads that share a query row: each
// posts one 64-bit word (a single-copy-atomic shared-memory access, so the
// values and their tag arrive together) and polls the partner's word until
// its tag matches the epoch (bounded in time).
__device__ __forceinline__ void xch_post(unsigned long long* slot, unsigned long long v) {
  asm volatile("st.volatile.shared::cta.u64 [%0], %1;" ::"r"(smem_u32(slot)), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long xch_peek(const unsigned long long* slot) {
  unsigned long long v;
  asm volatile("ld.volatile.shared::cta.u64 %0, [%1];" : "=l"(v) : "r"(smem_u32(slot)) : "memory");
  return v;
}
__device__ __noinline__ bool xch_await_slow(const unsigned long long* slot, uint32_t tag, unsigned long long* out,
                                            volatile int* abort, int* status) {
  const unsigned long long t0 = now_ns();
  for (uint32_t it = 1;; ++it) {
    const unsigned long long v = xch_peek(slot);
    if ((uint32_t)(v >> 31 & 1u) == tag) {
      *out = v;
      return true;
    }
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
__device__ __forceinline__ bool xch_await(const unsigned long long* slot, uint32_t tag, unsigned long long* out,
                                          volatile int* abort, int* status) {
  const unsigned long long v = xch_peek(slot);
  if ((uint32_t)(v >> 31 & 1u) == tag) {
    *out = v;
    return true;
  }
  return xch_await_slow(slot, tag, out, abort, status);
}

// Bounded wait used only on the way out (ignores the abort flag).
__device__ __noinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
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

// Shared-memory matrix descriptor, 128B swizzle, sm100 version bits.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // version
  d |= (uint64_t)2 << 61;  // SWIZZLE_128B
  return d;
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accum));
}

__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                       uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accum));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 consecutive TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]),
        "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]),
        "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
      "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]),
      "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]),
      "r"(v[30]), "r"(v[31]));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (two lanes of one 64-bit register): Blackwell's f32x2 ALU.
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void uf2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

struct TileInfo {
  int bh, m, nblk;
};

// Tile t of the schedule: heads are taken in chunks of `ch`; within a chunk
// the tiles go longest causal rows first across the chunk's heads.  CTAs take
// tiles in this order from a global counter, so the K/V of a few heads stay in
// L2 while every tile that reads them runs, and the causal work balances.
__device__ __forceinline__ TileInfo tile_info(int t, int BH, int N, int causal, int ch) {
  const int ntile = (N + kBM - 1) / kBM;
  const int per_chunk = ch * ntile;
  const int chunk = t / per_chunk;
  const int nh = min(ch, BH - chunk * ch);
  const int pos = t - chunk * per_chunk;
  TileInfo ti;
  ti.m = ntile - 1 - pos / nh;
  ti.bh = chunk * ch + pos % nh;
  const int kmax = causal ? min(N, (ti.m + 1) * kBM) : N;
  ti.nblk = (kmax + kBN - 1) / kBN;
  return ti;
}

// Dynamic tile scheduler state: the next tile to hand out, and the number of
// CTAs that finished; the last CTA of a launch resets both for the next one.
__device__ unsigned int g_tile_next;
__device__ unsigned int g_cta_done;

struct Params {
  int B, H, N, causal;
  int chunk_heads;
  int inject_stall;  // failure-detection test: withhold the first Q/R tile
  __nv_bfloat16* out;
  int* status;
};

__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmR,
                      const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = p.B * p.H;
  const int ntile = (p.N + kBM - 1) / kBM;
  const int tiles = ntile * BH;
  volatile int* abort = &sm.abort;

  // Slot 1 is first used by epoch 1 (tag 0) and slot 0 by epoch 2 (tag 1):
  // start each with the other tag.
  for (int x = threadIdx.x; x < 2 * 2 * kBM; x += blockDim.x)
    (&sm.xch[0][0][0])[x] = x < 2 * kBM ? 0ull : 0x80000000ull;
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.s_free, 8);  // one lane of each softmax warp
    for (int s = 0; s < 2; ++s) mbar_init(&sm.p_full[s], 256);
    for (int s = 0; s < kTileRing; ++s) {
      mbar_init(&sm.tile_full[s], 1);
      mbar_init(&sm.tile_empty[s], 10);  // the two MMA threads and one lane of each softmax warp
    }
    mbar_init(&sm.o_full, 1);
    mbar_init(&sm.o_empty, 256);
    mbar_init(&sm.drain, 2);  // one commit from each MMA thread
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
        const TileInfo ti = tile_info(t, BH, p.N, p.causal, p.chunk_heads);
        const int row0 = ti.bh * p.N;
        if (tc > 0 && !mbar_wait(&sm.q_empty, (tc - 1) & 1, abort, p.status)) break;
        mbar_expect_tx(&sm.q_full, 2 * kQBytes);
        q_issued = tc;
        // The failure-detection test withholds the first Q/R tile: its barrier
        // never completes, the MMA warp's bounded wait runs out and every role
        // unwinds through the abort path.
        if (!(p.inject_stall && tc == 0)) {
          for (int h = 0; h < 2; ++h) {
            tma_load_2d(sm.q + h * kHalfQ, &tmQ, &sm.q_full, 64 * h, row0 + ti.m * kBM);
            tma_load_2d(sm.r + h * kHalfQ, &tmR, &sm.q_full, 64 * h, row0 + ti.m * kBM);
          }
        }
        for (int j = 0; j < ti.nblk; ++j, ++kv) {
          const int st = kv % kStages;
          const uint32_t par = ((kv / kStages) & 1) ^ 1;
          if (!mbar_wait(&sm.kv_empty[st], par, abort, p.status)) break;
          mbar_expect_tx(&sm.kv_full[st], 2 * kKVBytes);
          kv_issued[st] = kv / kStages;
          for (int h = 0; h < 2; ++h) {
            tma_load_2d(sm.k[st] + h * kHalfKV, &tmK, &sm.kv_full[st], 64 * h, row0 + j * kBN);
            tma_load_2d(sm.v[st] + h * kHalfKV, &tmV, &sm.kv_full[st], 64 * h, row0 + j * kBN);
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
      // Each issuing thread shares its scheduler with two softmax warps, so
      // every MMA is issued from descriptors built once: a k-step or a stage
      // only adds a compile-time offset to the start-address field (smem
      // addresses < 256 KB keep that 14-bit field from carrying).
      bool ok = true;
      for (; ok; ++tc) {
        const int slot = tc % kTileRing;
        if (!(ok = mbar_wait(&sm.tile_full[slot], (tc / kTileRing) & 1, abort, p.status))) break;
        const int t = *reinterpret_cast<volatile int*>(&sm.tile_ring[slot]);
        mbar_arrive(&sm.tile_empty[slot]);
        if (t < 0) break;
        const TileInfo ti = tile_info(t, BH, p.N, p.causal, p.chunk_heads);
        if (!(ok = mbar_wait(&sm.q_full, tc & 1, abort, p.status))) break;
        for (int j = 0; j < ti.nblk; ++j, ++g) {
          // The S stage is free once the softmax has read the previous block's
          // scores; P buffer g % 2, which the softmax fills once these scores
          // land, is free once the value MMAs of block g - 2 completed.
          if (g > 0 && !(ok = mbar_wait(&sm.s_free, (g - 1) & 1, abort, p.status))) break;
          if (g > 1) {
            const uint32_t gq = g - 2;
            if (!(ok = mbar_wait(&sm.kv_empty[gq % kStages], (gq / kStages) & 1, abort, p.status))) break;
          }
          const uint32_t st = g % kStages;
          if (!(ok = mbar_wait(&sm.kv_full[st], (g / kStages) & 1, abort, p.status))) break;
          tc_fence_after();
          const uint64_t dk = dK0 + (uint64_t)(st * (kKVBytes >> 4));
          // S1 and S2 k-steps interleaved: on this per-block sequence that keeps
          // the tensor pipe at the sum of the two GEMMs (issuing all of S1 and
          // then all of S2 measured about a quarter slower).
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const uint64_t off = (uint64_t)((((ks >> 2) * kHalfQ) + (ks & 3) * 32) >> 4);
            const uint64_t koff = (uint64_t)((((ks >> 2) * kHalfKV) + (ks & 3) * 32) >> 4);
            mma_ss(tmem + kColS1, dQ + off, dk + koff, kIdescS, ks > 0);
            mma_ss(tmem + kColS2, dR + off, dk + koff, kIdescS, ks > 0);
          }
          mma_commit(&sm.s_full);
          if (j + 1 == ti.nblk) mma_commit(&sm.q_empty);
        }
      }
      // Drain: all MMAs this thread issued complete before TMEM is freed.
      mma_commit(&sm.drain);
      mbar_drain(&sm.drain, 0);
    }
  } else if (warp == kPVWarp) {
    // ---------------- value MMA issuer ----------------
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
        const TileInfo ti = tile_info(t, BH, p.N, p.causal, p.chunk_heads);
        // The epilogue of the previous tile must have read O before it is overwritten.
        if (tc > 0 && !(ok = mbar_wait(&sm.o_empty, (tc - 1) & 1, abort, p.status))) break;
        for (int j = 0; j < ti.nblk; ++j, ++g) {
          const uint32_t b = g & 1;
          // P of this block is in TMEM; its scores (so its K) were consumed
          // before, and V arrived with K.
          if (!(ok = mbar_wait(&sm.p_full[b], (g >> 1) & 1, abort, p.status))) break;
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
      mma_commit(&sm.drain);
      mbar_drain(&sm.drain, 0);
    }
  } else {
    // ---------------- softmax / epilogue: two warpgroups ----------------
    // Warpgroup hf (warps 2..5 -> 0, 6..9 -> 1) owns keys 32hf..32hf+31 of every
    // block and output dims 64hf..64hf+63; both threads of a row take the max
    // over all 64 scores of a block and exchange their partial sums through
    // shared memory, so both keep identical copies of the row state
    // (m, omega, T, c).
    const int hf = (warp - 2) >> 2;
    const int row = 32 * (warp & 3) + lane;  // TMEM lane == query row within the tile
    const uint32_t lane_addr = (uint32_t)(32 * (warp & 3)) << 16;
    const float scale = 1.4426950408889634f * rsqrtf((float)kD);
    uint32_t g = 0;  // blocks processed by this CTA (also the exchange epoch)
    int tc = 0;
    bool ok = true;
    for (; ok; ++tc) {
      const int slot = tc % kTileRing;
      if (!(ok = mbar_wait(&sm.tile_full[slot], (tc / kTileRing) & 1, abort, p.status))) break;
      const int t = *reinterpret_cast<volatile int*>(&sm.tile_ring[slot]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.tile_empty[slot]);
      if (t < 0) break;
      const TileInfo ti = tile_info(t, BH, p.N, p.causal, p.chunk_heads);
      const int i = ti.m * kBM + row;  // query position
      // Row state: running max (log2 units), omega = sum w, T = sum w (t - c)
      // around the row's centre c (see the file comment), all in fp32.
      float m_run = -CUDART_INF_F, omega = 0.f, T = 0.f, cen = 0.f;
      for (int j = 0; j < ti.nblk; ++j, ++g) {
        if (!(ok = mbar_wait(&sm.s_full, g & 1, abort, p.status))) break;
        tc_fence_after();
        const uint32_t sb = tmem + lane_addr;
        const int kb = j * kBN;
        const bool edge = (p.causal && kb + kBN - 1 > ti.m * kBM) || (kb + kBN > p.N);
        const int kend = p.causal ? min(i + 1, p.N) : p.N;  // keys < kend are visible
        uint32_t x[32], y[32];
        float rmax;
        {
          // This thread's 32 scores and t values, and the partner half of the
          // scores for the row max; then the S stage is handed back to the MMA.
          uint32_t z[32];
          tmem_ld32(sb + kColS1 + 32 * hf, x);
          tmem_ld32(sb + kColS1 + 32 * (hf ^ 1), z);
          tmem_ld32(sb + kColS2 + 32 * hf, y);
          tc_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.s_free);
          if (edge) {  // block-uniform: only blocks that cross the diagonal or the end
            const int k0 = kb + 32 * hf, kz = kb + 32 * (hf ^ 1);
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              if (k0 + c >= kend) x[c] = __float_as_uint(-CUDART_INF_F);
              if (kz + c >= kend) z[c] = __float_as_uint(-CUDART_INF_F);
            }
          }
          // Four independent chains over the 64 scores, then their max.
          float m4[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            m4[0] = max3(m4[0], __uint_as_float(x[c]), __uint_as_float(x[c + 1]));
            m4[1] = max3(m4[1], __uint_as_float(x[c + 2]), __uint_as_float(x[c + 3]));
            m4[2] = max3(m4[2], __uint_as_float(z[c]), __uint_as_float(z[c + 1]));
            m4[3] = max3(m4[3], __uint_as_float(z[c + 2]), __uint_as_float(z[c + 3]));
          }
          rmax = fmaxf(max3(m4[0], m4[1], m4[2]), m4[3]);
        }
        // Both halves of the row took the max of the same 64 scores, so the
        // raise decision below is the same on both sides.
        const float mx = rmax * scale;
        float alpha = 1.f;
        if (mx > m_run + kLazyTau) {  // always on a tile's first block (m_run = -inf)
          alpha = ex2(m_run - mx);    // 0 on the first block
          m_run = mx;
          omega *= alpha;
          T *= alpha;
        }
        // w = 2^(s*scale - m_run); a = w (t - c) is kept for bf16(w (t - c))
        // once the centre is settled.  x <- w, y <- a.
        uint32_t P[16];
        float wpart, tpart;
        {
          const uint64_t sc2 = f2(scale, scale), nm2 = f2(-m_run, -m_run), nc2 = f2(-cen, -cen);
          uint64_t ws2a = f2(0.f, 0.f), ts2a = f2(0.f, 0.f), ws2b = ws2a, ts2b = ts2a;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
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
            P[c] = pack_bf16(w0, w1);
            float a0, a1;
            uf2(a2, a0, a1);
            x[2 * c] = __float_as_uint(w0);
            x[2 * c + 1] = __float_as_uint(w1);
            y[2 * c] = __float_as_uint(a0);
            y[2 * c + 1] = __float_as_uint(a1);
          }
          float lo, hi;
          uf2(add2(ws2a, ws2b), lo, hi);
          wpart = lo + hi;
          uf2(add2(ts2a, ts2b), lo, hi);
          tpart = lo + hi;
        }
        // Exchange (sum w, sum w (t - c)) with the partner thread of this row.
        const uint32_t e0 = g + 1, tag = (e0 >> 1) & 1u;
        xch_post(&sm.xch[e0 & 1][hf][row],
                 (unsigned long long)__float_as_uint(tpart) << 32 | __float_as_uint(wpart) | tag << 31);
        unsigned long long theirs;
        if (!(ok = xch_await(&sm.xch[e0 & 1][hf ^ 1][row], tag, &theirs, abort, p.status))) break;
        // Both threads of the row form the same sums (a + b == b + a exactly).
        const float wsum = wpart + __uint_as_float((uint32_t)theirs & 0x7FFFFFFFu);
        float Tb = tpart + __uint_as_float((uint32_t)(theirs >> 32));
        // Re-centre before this block's w (t - c) is rounded to bf16, on the
        // first block and whenever the running mean of t has drifted by more
        // than kTheta from the centre.
        float delta = 0.f;
        const float Tn = T + Tb, Wn = omega + wsum;  // Wn > 0: key 0 is visible to every row
        if (j == 0 || fabsf(Tn) > kTheta * Wn) {
          delta = Tn / Wn;
          cen += delta;
          T -= delta * omega;
          Tb -= delta * wsum;
        }
        omega += wsum;
        T += Tb;
        // Rows whose max rose or whose centre moved update their part of O1 and
        // O2 (O1 <- alpha O1, O2 <- alpha (O2 - delta O1)) once the value MMAs
        // of the previous block are complete; each warpgroup updates its 64 dims.
        const bool need = (j > 0) && (alpha != 1.f || delta != 0.f);
        if (__any_sync(0xffffffffu, need)) {
          // The previous block's value MMAs completed when its K/V stage was freed
          // (block counter g equals the K/V ring position).
          const uint32_t gp = g - 1;
          if (!(ok = mbar_wait(&sm.kv_empty[gp % kStages], (gp / kStages) & 1, abort, p.status))) break;
          tc_fence_after();
          const float ad = alpha * delta;
#pragma unroll 1
          for (int c0 = 64 * hf; c0 < 64 * hf + 64; c0 += 32) {
            uint32_t o1[32], o2[32];
            const uint32_t a1 = sb + kColO1 + c0, a2 = sb + kColO2 + c0;
            tmem_ld32(a1, o1);
            tmem_ld32(a2, o2);
            tc_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const float v1 = __uint_as_float(o1[c]);
              o2[c] = __float_as_uint(alpha * __uint_as_float(o2[c]) - ad * v1);
              o1[c] = __float_as_uint(alpha * v1);
            }
            tmem_st32(a1, o1);
            tmem_st32(a2, o2);
          }
        }
        // P buffer g % 2 is free: the scores of this block were issued only
        // after the value MMAs of block g - 2 (its last reader) completed.
        const uint32_t pb = sb + kColP + (g & 1) * kColPBuf;
        tmem_st16(pb + 16 * hf, P);
        uint32_t PT[16];
        if (__any_sync(0xffffffffu, delta != 0.f)) {
          const uint64_t nd2 = f2(-delta, -delta);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            float a0, a1;
            uf2(fma2(f2(__uint_as_float(x[2 * c]), __uint_as_float(x[2 * c + 1])), nd2,
                     f2(__uint_as_float(y[2 * c]), __uint_as_float(y[2 * c + 1]))),
                a0, a1);
            PT[c] = pack_bf16(a0, a1);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) PT[c] = pack_bf16(__uint_as_float(y[2 * c]), __uint_as_float(y[2 * c + 1]));
        }
        tmem_st16(pb + kColPT + 16 * hf, PT);
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(&sm.p_full[g & 1]);
      }
      if (!ok) break;
      // ---- epilogue: out = ((1 + T/omega) O1 - O2) / omega, dims 64hf.. of this row.
      if (!(ok = mbar_wait(&sm.o_full, tc & 1, abort, p.status))) break;
      tc_fence_after();
      const float inv = 1.f / omega;
      const float c1 = (1.f + T * inv) * inv;
      __nv_bfloat16* orow = p.out + ((long long)ti.bh * p.N + i) * kD;
#pragma unroll 1
      for (int c0 = 64 * hf; c0 < 64 * hf + 64; c0 += 32) {
        uint32_t o1[32], o2[32];
        tmem_ld32(tmem + lane_addr + kColO1 + c0, o1);
        tmem_ld32(tmem + lane_addr + kColO2 + c0, o2);
        tc_wait_ld();
        if (i < p.N) {
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
      }
      tc_fence_before();
      mbar_arrive(&sm.o_empty);
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

// 2-D view [rows, 128] of a bf16 [B, H, N, 128] tensor, boxes of 64 dims x box_rows rows.
bool make_map(CUtensorMap* m, const void* base, long long rows, int box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bool prefill_tc_supported(int d) { return d == kD; }

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t st, int num_sms) {
  const long long rows = (long long)a.B * a.H * a.N;
  if (rows >= (1ll << 31)) return cudaErrorInvalidValue;
  CUtensorMap mQ, mR, mK, mV;
  if (!make_map(&mQ, a.Q, rows, kBM) || !make_map(&mR, a.R, rows, kBM) || !make_map(&mK, a.K, rows, kBN) ||
      !make_map(&mV, a.V, rows, kBN))
    return cudaErrorInvalidValue;
  const int ntile = (a.N + kBM - 1) / kBM;
  int ch = (2 * num_sms + ntile - 1) / ntile;  // about two waves of tiles per chunk
  ch = ch < 1 ? 1 : (ch > a.B * a.H ? a.B * a.H : ch);
  // PLX_FAULT_INJECT=prefill_stall makes the kernel's bounded waits run out
  // (tests of the timeout status only).
  const char* fi = getenv("PLX_FAULT_INJECT");
  const int inject = (fi != nullptr && strcmp(fi, "prefill_stall") == 0) ? 1 : 0;
  Params p{a.B, a.H, a.N, a.causal, ch, inject, reinterpret_cast<__nv_bfloat16*>(a.out), a.status};
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long tiles = (long long)((a.N + kBM - 1) / kBM) * a.B * a.H;
  const int grid = (int)(tiles < num_sms ? tiles : num_sms);
  prefill_tc_kernel<<<grid, kThreads, smem, st>>>(mQ, mR, mK, mV, p);
  return cudaGetLastError();
}

}  // namespace plx
