// Internal declarations shared by the translation units of libplx.so.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

namespace plx {

// Bits of the per-device status word that kernels set (atomicOr); the host
// maps the lowest set bit to a status code.
enum : int {
  kStatusBadSeqlen = 1,
  kStatusTimeout = 2,
};

// Iteration cap of every bounded wait in the kernels (mbarrier try_wait loops).
// A wait that reaches it sets kStatusTimeout and abandons the tile.
constexpr long long kWaitCap = 1ll << 26;

struct PrefillArgs {
  const void* Q;
  const void* K;
  const void* V;
  const void* R;
  void* out;
  int B, H, N, d;
  int causal;
  int* status;
  // Optional (tensor-core path only): softmax mean of v [rows, d] and the
  // per-row lse and tbar [rows], all fp32, for the backward pass.
  void* vbar = nullptr;
  float* lse = nullptr;
  float* tbar = nullptr;
  int window = 0;  // sliding window: query i sees keys i - window + 1 .. i (0: none; implies causal)
  // Block-sparse causal prefill (tensor-core path; device CSR over 128-query
  // tiles of ascending 64-key block indices), or null.
  const int* blk_ptr = nullptr;
  const int* blk_idx = nullptr;
  // Grouped KV heads (tensor-core path): K and V are [B, Hkv, N, d] and query
  // head h reads KV head h / (H / Hkv); 0 means Hkv = H.
  int Hkv = 0;
  // Dilation r (tensor-core path; 1 or 0: none): query i sees keys i, i - r,
  // i - 2r, ... (the causal and window masks within its residue class mod r).
  // N must be a multiple of r.
  int dilation = 1;
};

struct DecodeArgs {
  const void* q;
  const void* r;
  const void* K;
  const void* V;
  const int32_t* seqlens;
  void* out;
  int B, H, L, d;
  int splits;       // key chunks per (b, h)
  int chunk;        // keys per chunk (multiple of 64)
  float* partials;  // [B*H, splits, 2*d + 4] fp32: (m, omega, T, pad, O1[d], O2[d])
  int* counters;    // [B*H] arrival counters, zero between calls ([B*Hkv] for grouped KV)
  int* status;
  int Hkv;          // KV heads (grouped-KV decode only; H is a multiple of it)
  int window;       // sliding window: the last `window` keys of each sequence (0: all)
  int inject_stall = 0;  // failure-detection test (tensor-core decode): CTA 0 never loads its K/V
  // e4m3 caches (decode_fp8kv): K and V hold one byte per element, and these
  // fp32 [B*Hkv*L] arrays the scale of every cached row.
  const float* Kscale = nullptr;
  const float* Vscale = nullptr;
};

// SIMT kernels: any d that is a multiple of 32 up to 128, f32 or bf16 storage.
cudaError_t launch_prefill_simt(const PrefillArgs& a, bool bf16, cudaStream_t st);
cudaError_t launch_decode_simt(const DecodeArgs& a, bool bf16, cudaStream_t st);

// bf16 split-KV decode on tensor-core MMAs, d in {64, 128}.
cudaError_t launch_decode_bf16(const DecodeArgs& a, cudaStream_t st, int num_sms);
// bf16 split-KV decode with grouped KV heads (H = G * Hkv, G in {2, 4, 8}),
// d in {64, 128}: K/V blocks staged by TMA, the q and rho rows of the heads of
// a group in one MMA tile.
cudaError_t launch_decode_gqa(const DecodeArgs& a, cudaStream_t st, int num_sms);
// Decode on tcgen05 (d = 128; G = H / Hkv in {1, 2, 4, 8}); called by
// launch_decode_gqa and, with Hkv = H, by launch_decode_bf16.
cudaError_t launch_decode_gqa_tc(const DecodeArgs& a, cudaStream_t st, int num_sms);
// Decode over an e4m3 cache with per-row scales (d = 128, G = H / Hkv in {1, 2, 4, 8}).
cudaError_t launch_decode_fp8kv(const DecodeArgs& a, cudaStream_t st, int num_sms);
// Per-row dynamic e4m3 quantisation of bf16 cache rows [rows, d] (d in {64, 128}).
cudaError_t launch_kv_quantize_fp8(const void* X, void* codes, float* scales, long long rows, int d,
                                   cudaStream_t st);
// Split heuristic shared by the launcher and the workspace-size query;
// ctas_per_sm is how many CTAs of the decode kernel an SM holds.
void decode_split_plan(int B, int H, int L, int num_sms, int* splits, int* chunk, int ctas_per_sm = 2);
// The grouped-KV decode runs on the tensor-core kernel at d = 128, and at
// d = 64 with groups of 2, 4 or 8 when Hkv is even (two KV heads per unit);
// otherwise on the warp-MMA kernel.  KV heads per unit and CTAs per SM of the
// kernel that runs (the split plan's inputs).
inline bool decode_gqa_tc(int Hkv, int d) { return d == 128 || (d == 64 && Hkv % 2 == 0); }
inline int decode_gqa_kv_per_unit(int Hkv, int d) { return (d == 64 && Hkv % 2 == 0) ? 2 : 1; }
inline int decode_gqa_ctas_per_sm(int G, int Hkv, int d) { return (decode_gqa_tc(Hkv, d) || G == 8) ? 1 : 2; }
// Which kernel serves the ungrouped bf16 decode of bh (b, h) pairs with
// `keys` visible keys per query (L, or the window) and head dim d: the
// tensor-core kernel (one CTA per SM) once units carry enough keys to hide its
// per-unit start-up and merge, else the warp-MMA kernel (two CTAs per SM),
// which wins on short sequences and on few of them (the decode sweep, H = 16,
// lengths uniform on [L/2, L]).  A pure function of the sizes, so that the
// split plan, the workspace size and the launch agree.
inline bool decode_bf16_tc(long long bh, int keys, int d) {
  if (d != 128) return false;
  if (keys >= 16384) return true;
  if (keys >= 2048) return bh >= 256;
  if (keys >= 1024) return bh >= 512 && bh <= 2048;
  return false;
}
// CTAs per SM of that kernel (the split plan's input).
inline int decode_bf16_ctas_per_sm(long long bh, int keys, int d) { return decode_bf16_tc(bh, keys, d) ? 1 : 2; }
// The ungrouped bf16 decode's kernel: at d = 128 the size rule above; at d = 64
// with H even the tcgen05 kernel takes two heads a unit (their 64-dim halves
// side by side, as for grouped KV heads) for long contexts over few heads
// (>= 16384 keys, B*H < 128: 1.16x at B=1, H=32, L=32768), else the warp-MMA
// kernel, which measured equal or faster elsewhere (0.95 of the copy peak at
// B=64, H=32, L=4096; 1.5x at L=128).
inline bool decode_bf16_tc_h(int B, int H, int keys, int d) {
  if (d == 64) return H % 2 == 0 && keys >= 16384 && (long long)B * H < 128;
  return decode_bf16_tc((long long)B * H, keys, d);
}
// The split plan of the ungrouped bf16 decode (units (b, h), or (b, head pair)
// on the d = 64 tensor-core kernel), shared by the launch, the workspace size
// and the diagnostics so that they agree.
inline void decode_bf16_plan(int B, int H, int keys, int d, int num_sms, int* splits, int* chunk) {
  const bool tc = decode_bf16_tc_h(B, H, keys, d);
  decode_split_plan(B, (tc && d == 64) ? H / 2 : H, keys, num_sms, splits, chunk, tc ? 1 : 2);
}

// Sizes every decode entry point accepts: at most 2^24 query (b, h) pairs, and
// cache rows (B * KV heads * L) that stay below 2^31 even after the largest
// staged key block (128 keys) is added to the last row a unit can start at, so
// that whichever decode kernel the sizes select can address them.
inline bool decode_sizes_supported(int B, int H, int Hkv, int L) {
  return (long long)B * H <= (1ll << 24) && (long long)B * Hkv * L + 128 < (1ll << 31);
}

// bf16 causal/full prefill on tcgen05 + TMA + TMEM, d == 128.
bool prefill_tc_supported(int d);
cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t st, int num_sms);

// Backward pass of the bf16 tensor-core prefill (d in {64, 128}): gradients of
// Q, K, V, R from the output gradient dO and the forward's out, vbar, lse and
// tbar.  `stats` is a workspace of B * H * bwd_padded_rows(N) float4.
struct BwdArgs {
  const void* Q;
  const void* K;
  const void* V;
  const void* R;
  const void* out;
  const void* vbar;
  const void* dO;
  const float* lse;
  const float* tbar;
  void* dQ;
  void* dK;
  void* dV;
  void* dR;
  int B, H, N, d, causal;
  void* stats;
  int* status;
  int window = 0;  // sliding window of the forward (0: none; implies causal)
  int Hkv = 0;     // KV heads of K, V, dK, dV (0: H); H a multiple of it
};
size_t bwd_padded_rows(int N);
// The step of this thread's last failed backward launch ("" if none).
const char* bwd_last_failure();
cudaError_t launch_prefill_bwd(const BwdArgs& a, cudaStream_t st, int num_sms);

// Dynamic per-tensor fp8 (e4m3) linears: |max| reductions of `count` (<= 5)
// tensors of n values each into amax_bits[0..count) (zeroed first),
// quantisation (s = max/448, written to *scale), quantisation with a
// transpose of `count` [rows, cols] weights into Wt + i * wt_stride (scales to
// scale[i]), and the e4m3 GEMM Y[M, Dout] = X8[M, Din] Wt8[Dout, Din]^T sX sW
// in bf16 through cuBLASLt (returns 0 on success).  Sizes are multiples of 64;
// pointers 16-byte aligned.
cudaError_t launch_amax(const void* const* x, int count, size_t n, unsigned* amax_bits, cudaStream_t st);
cudaError_t launch_quant(const void* x, size_t n, const unsigned* amax_bits, void* out, float* scale,
                         cudaStream_t st);
cudaError_t launch_quant_t(const void* const* W, int count, int rows, int cols, const unsigned* amax_bits,
                           void* Wt, size_t wt_stride, float* scale, cudaStream_t st);
int fp8_gemm(void* lt_handle, const void* Wt8, const void* X8, void* Y, int Dout, int Din, long long M,
             const float* sW, const float* sX, void* ws, size_t ws_bytes, cudaStream_t st);

// Per-head RMSNorm + RoPE with the head split folded in.
cudaError_t launch_qkr_norm_rope(const void* x, void* y, int B, int N, int H, int d, float eps,
                                 float base, cudaStream_t st);
// bf16 [B, A1, A2, d] -> [B, A2, A1, d] (head split and merge of a layer).
cudaError_t launch_swap_axes(const void* src, void* dst, int B, int A1, int A2, int d,
                             cudaStream_t st);

}  // namespace plx

namespace plx {
// Device address of this device's kernel status word (nullptr if CUDA fails).
int* status_word_address();
}  // namespace plx
