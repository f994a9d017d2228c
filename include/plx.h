/*
 * plx.h — C ABI of libplx.so: Parallax attention forward on NVIDIA B200 (sm_100a).
 *
 * Method: "Parallax: Parameterized Local Linear Attention for Language Modeling"
 * (arXiv 2605.29157).  Per query i over its visible keys J_i:
 *
 *   p_ij  = softmax_j(q_i . k_j / sqrt(d))                (rainbus.top summary, "Softmax Attention")
 *   out_i = o^SA_i - Sigma_KV^(i) rho_i                    (gist.science summary, "Mecanismo central")
 *         = sum_j p_ij (1 - t_ij + tbar_i) v_j,  t_ij = rho_i . k_j,  tbar_i = sum_j p_ij t_ij
 *
 * computed in the streamed form with one running max and one rescale factor
 * shared by the softmax branch and the covariance branch (rainbus.top summary,
 * "方法步骤详情": per KV block S1 = QK^T and S2 = RK^T, then O1 = sum w v and
 * O2 = sum w t v accumulated together; agihunt.info summary, hardware paragraph).
 * The boundary amplification factor eta is zero (gist.science, "Eliminación de la
 * Amplificación de Frontera").  rho_i (R) is an input: the probe W_R x after its
 * RMSNorm and RoPE.
 *
 * Conventions (the pages give no layout):
 *   - Prefill tensors Q, K, V, R, out are [B, H, N, d], row-major, d fastest.
 *   - Decode: q, r, out are [B, H, d]; Kcache, Vcache are [B, H, L, d] with each
 *     sequence padded to stride L; seqlens is int32 [B] with 1 <= seqlens[b] <= L.
 *     The query of sequence b sits at position seqlens[b]-1 and sees keys
 *     0 .. seqlens[b]-1.
 *   - Scores are scaled by 1/sqrt(d); the probe term t = rho . k is not scaled.
 *   - causal != 0: query row i sees keys 0..i (diagonal included).  causal == 0:
 *     every row sees all N keys.
 *   - Every head has its own K and V, except in the entry points that take Hkv
 *     (grouped KV heads: query head h reads KV head h / (H / Hkv)).
 *   - out has the dtype of the inputs; arithmetic is fp32.
 *
 * Memory and ownership: every tensor pointer is a DEVICE pointer owned by the
 * caller; the library keeps no reference after the call returns.  Calls are
 * asynchronous on the given CUDA stream (void* stands for cudaStream_t; NULL is
 * the legacy default stream).  All tensor pointers must be 16-byte aligned.
 *
 * Errors: every entry point returns PLX_OK (0) or a negative code.  Argument
 * errors are detected on the host before anything is launched.  Errors found by
 * a kernel (a seqlen outside 1..L, a bounded wait that ran out) are recorded in a
 * per-device status word that plx_get_device_status() reads and clears; such a
 * kernel writes zeros for the affected outputs and never traps.
 */
#ifndef PLX_H
#define PLX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PLX_ABI_VERSION 1

/* Element type of all tensors of one call. */
typedef enum { PLX_F32 = 0, PLX_BF16 = 1 } plx_dtype;

/* Status codes. */
#define PLX_OK 0
#define PLX_ERR_INVALID_ARG (-1)  /* null pointer, non-positive size, bad enum      */
#define PLX_ERR_UNSUPPORTED (-2)  /* head dim or dtype combination not implemented */
#define PLX_ERR_MISALIGNED (-3)   /* a tensor pointer is not 16-byte aligned       */
#define PLX_ERR_CUDA (-4)         /* a CUDA runtime/driver call or launch failed   */
#define PLX_ERR_WORKSPACE (-5)    /* caller workspace smaller than required        */
#define PLX_ERR_BAD_SEQLEN (-6)   /* device-reported: a seqlens[b] outside 1..L    */
#define PLX_ERR_TIMEOUT (-7)      /* device-reported: a bounded wait gave up (tests force it
                                     with the environment PLX_FAULT_INJECT=prefill_stall,
                                     bwd_stall or decode_stall) */

/* Name of the CUDA error behind this thread's last PLX_ERR_CUDA from a kernel
 * launch ("no error" if there was none).  Static string. */
const char* plx_last_cuda_error(void);

/* Supported shapes: bf16 with d in {64, 128}; f32 with d a multiple of 32 and
 * d <= 128.  B, H, N, L >= 1. */

/*
 * Causal (or full) prefill forward.  bf16 on the legacy default stream.
 * Q, K, V, R, out: [B, H, N, d].
 */
int plx_prefill(const void* Q, const void* K, const void* V, const void* R, void* out,
                int B, int H, int N, int d, int causal);

/* As plx_prefill with an explicit element type and stream. */
int plx_prefill_ex(const void* Q, const void* K, const void* V, const void* R, void* out,
                   int B, int H, int N, int d, int causal, int dtype, void* stream);

/*
 * Sliding-window causal prefill: query i sees keys max(0, i - window + 1)..i
 * (the pages list kernels combining Parallax with sliding-window sparsity as
 * future work: rainbus.top "未来方向"; the rule is this build's reading).
 * Layout, dtypes, head dims and errors as plx_prefill_ex; window >= 1 (a window
 * of N or more keys is the causal prefill), else PLX_ERR_INVALID_ARG.
 */
int plx_prefill_window(const void* Q, const void* K, const void* V, const void* R, void* out,
                       int B, int H, int N, int d, int window, int dtype, void* stream);

/*
 * Causal (or full) bf16 prefill with grouped KV heads: Q, R, out [B, H, N, d];
 * K, V [B, Hkv, N, d] with H a multiple of Hkv; query head h reads KV head
 * h / (H / Hkv) (consecutive query heads share one).  The pages place Parallax
 * in a Qwen-3 architecture (rainbus.top reproduction notes), whose attention
 * groups KV heads.  d in {64, 128}, else PLX_ERR_UNSUPPORTED; H not a multiple
 * of Hkv gives PLX_ERR_INVALID_ARG.  Other arguments as plx_prefill_ex.
 */
int plx_prefill_gqa(const void* Q, const void* K, const void* V, const void* R, void* out, int B, int H,
                    int Hkv, int N, int d, int causal, void* stream);

/* plx_prefill_gqa with a sliding window of `window` keys (query i sees keys
 * i - window + 1 .. i, as plx_prefill_window).  window >= 1, else
 * PLX_ERR_INVALID_ARG. */
int plx_prefill_gqa_window(const void* Q, const void* K, const void* V, const void* R, void* out, int B, int H,
                           int Hkv, int N, int d, int window, void* stream);

/*
 * Block-sparse causal prefill, bf16, d in {64, 128}: query i sees key j when
 * j <= i and block_mask[i / 128][j / 64] is non-zero (the pages list
 * block-sparse kernels as future work: rainbus.top "未来方向"; the rule is
 * this build's reading).  block_mask: HOST array of ceil(N/128) x ceil(N/64)
 * bytes, row-major, shared by all heads; copied during the call.  Each tile's
 * own diagonal blocks (2m and 2m+1 where they exist) must be active, else
 * PLX_ERR_INVALID_ARG; blocks above the diagonal are ignored.  The block lists
 * live in a library-owned device buffer: calls on one device must be ordered.
 * Other arguments and errors as plx_prefill_ex.
 */
int plx_prefill_block_sparse(const void* Q, const void* K, const void* V, const void* R, void* out,
                             int B, int H, int N, int d, const uint8_t* block_mask, void* stream);

/*
 * Sliding-window decode step: the query of sequence b sees its last `window`
 * keys, max(0, seqlens[b] - window)..seqlens[b]-1.  Hkv == H is the decode of
 * plx_decode_ex (bf16 or fp32); Hkv < H is the grouped-KV decode of
 * plx_decode_gqa (bf16 only, else PLX_ERR_UNSUPPORTED).  Workspace: at least
 * plx_decode_window_workspace_bytes(B, H, Hkv, L, d, window) bytes, or NULL;
 * other arguments and errors as those two calls; window >= 1 (window >= L is
 * the full decode), else PLX_ERR_INVALID_ARG.
 */
int plx_decode_window(const void* q, const void* r, const void* Kcache, const void* Vcache,
                      const int32_t* seqlens, void* out, int B, int H, int Hkv, int L, int d,
                      int window, int dtype, void* workspace, size_t workspace_bytes, void* stream);
size_t plx_decode_window_workspace_bytes(int B, int H, int Hkv, int L, int d, int window);

/*
 * Training forward: the causal (or full) bf16 prefill of plx_prefill_ex that
 * also saves what plx_prefill_bwd needs, per query row i of head (b, h):
 *   vbar[b,h,i,:] = sum_j p_ij v_j                 (fp32 [B, H, N, d]),
 *   lse[b,h,i]    = log sum_j exp(q_i . k_j / sqrt(d))  (fp32 [B, H, N], natural log),
 *   tbar[b,h,i]   = sum_j p_ij (rho_i . k_j)       (fp32 [B, H, N]),
 * with p_ij the softmax weights over the visible keys ("Parallax: Parameterized
 * Local Linear Attention for Language Modeling": the softmax weights and the
 * probe scores of the rainbus.top summary's forward steps; vbar and tbar are
 * the weighted means that centre the covariance of the gist.science summary's
 * "Mecanismo central").  out as plx_prefill_ex.  d in {64, 128}, else
 * PLX_ERR_UNSUPPORTED.  All pointers device memory, caller-owned; Q, K, V, R,
 * out and vbar 16-byte aligned, lse and tbar 4-byte aligned, else
 * PLX_ERR_MISALIGNED.
 * Asynchronous on `stream`.
 */
int plx_prefill_train(const void* Q, const void* K, const void* V, const void* R, void* out,
                      void* vbar, float* lse, float* tbar, int B, int H, int N, int d, int causal,
                      void* stream);

/* plx_prefill_train for the sliding-window prefill of plx_prefill_window
 * (query i sees keys i - window + 1 .. i): the statistics are those of the
 * windowed softmax.  window >= 1, else PLX_ERR_INVALID_ARG. */
int plx_prefill_train_window(const void* Q, const void* K, const void* V, const void* R, void* out,
                             void* vbar, float* lse, float* tbar, int B, int H, int N, int d, int window,
                             void* stream);

/* plx_prefill_train with grouped KV heads, as plx_prefill_gqa: K and V are
 * [B, Hkv, N, d] and query head h reads KV head h / (H / Hkv); Q, R, out, vbar,
 * lse and tbar keep H heads.  Hkv >= 1 dividing H, else PLX_ERR_INVALID_ARG;
 * Hkv = H is plx_prefill_train.  Causal or full. */
int plx_prefill_train_gqa(const void* Q, const void* K, const void* V, const void* R, void* out, void* vbar,
                          float* lse, float* tbar, int B, int H, int Hkv, int N, int d, int causal,
                          void* stream);

/* The training forward in its general form: Hkv KV heads (as
 * plx_prefill_train_gqa; Hkv = H for one KV head per query head) and a
 * sliding window of `window` keys (0: none; a window implies the causal
 * mask, and `causal` is then ignored).  Hkv >= 1 dividing H and window >= 0,
 * else PLX_ERR_INVALID_ARG.  Every other plx_prefill_train* call is this one
 * with some arguments fixed. */
int plx_prefill_train_ex(const void* Q, const void* K, const void* V, const void* R, void* out, void* vbar,
                         float* lse, float* tbar, int B, int H, int Hkv, int N, int d, int causal, int window,
                         void* stream);

/* Bytes of the statistics workspace plx_prefill_bwd needs:
 * 16 * B * H * (N rounded up to a multiple of 128); 0 for invalid sizes. */
size_t plx_prefill_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * Backward pass of the prefill: the gradients dQ, dK, dV, dR (bf16, each
 * [B, H, N, d], overwritten) of sum(out * dO) for one causal (or full) bf16
 * prefill, given its inputs Q, K, V, R, the output gradient dO and the tensors
 * plx_prefill_train saved (out, vbar, lse, tbar).  The pages train the layer
 * but print no backward pass: these are the exact gradients of the forward
 * definition (per query i, out_i = sum_j p_ij (1 - t_ij + tbar_i) v_j with
 * t_ij = rho_i . k_j), computed on tensor cores with fp32 accumulation and
 * bf16 rounding of the per-pair weights before each gradient MMA.
 * workspace: device memory of plx_prefill_bwd_workspace_bytes(B, H, N, d)
 * bytes, 16-byte aligned, no initial contents, or NULL for a library-owned
 * one (grown on demand, per device; calls on one device must then be ordered).
 * d in {64, 128}, else PLX_ERR_UNSUPPORTED; tensors 16-byte aligned, lse and
 * tbar 4-byte aligned, else PLX_ERR_MISALIGNED; a short workspace gives
 * PLX_ERR_WORKSPACE.  Three kernel launches, asynchronous on `stream`.
 */
int plx_prefill_bwd(const void* Q, const void* K, const void* V, const void* R, const void* out,
                    const void* vbar, const float* lse, const float* tbar, const void* dO, void* dQ,
                    void* dK, void* dV, void* dR, int B, int H, int N, int d, int causal,
                    void* workspace, size_t workspace_bytes, void* stream);

/* plx_prefill_bwd for a sliding-window prefill (the tensors plx_prefill_train_window
 * saved): key j takes gradient only from queries j .. j + window - 1.
 * window >= 1, else PLX_ERR_INVALID_ARG; workspace as plx_prefill_bwd. */
int plx_prefill_bwd_window(const void* Q, const void* K, const void* V, const void* R, const void* out,
                           const void* vbar, const float* lse, const float* tbar, const void* dO, void* dQ,
                           void* dK, void* dV, void* dR, int B, int H, int N, int d, int window,
                           void* workspace, size_t workspace_bytes, void* stream);

/* plx_prefill_bwd for the grouped-KV prefill of plx_prefill_train_gqa: K, V,
 * dK and dV are [B, Hkv, N, d]; Q, R, dQ, dR, out, vbar, dO, lse and tbar have
 * H heads.  KV head g is shared by query heads g G .. g G + G - 1 of its batch
 * (G = H / Hkv), so dK and dV of a KV head sum the contributions of those G
 * query heads (one CTA per 128-key block of a KV head accumulates all of them
 * in TMEM; no atomics, no second pass).  Hkv >= 1 dividing H, else
 * PLX_ERR_INVALID_ARG; workspace as plx_prefill_bwd (sized by H). */
int plx_prefill_bwd_gqa(const void* Q, const void* K, const void* V, const void* R, const void* out,
                        const void* vbar, const float* lse, const float* tbar, const void* dO, void* dQ, void* dK,
                        void* dV, void* dR, int B, int H, int Hkv, int N, int d, int causal, void* workspace,
                        size_t workspace_bytes, void* stream);

/* The backward pass in its general form, for the tensors plx_prefill_train_ex
 * saved with the same Hkv, causal and window (dK, dV [B, Hkv, N, d]).
 * Hkv >= 1 dividing H and window >= 0, else PLX_ERR_INVALID_ARG; workspace
 * as plx_prefill_bwd. */
int plx_prefill_bwd_ex(const void* Q, const void* K, const void* V, const void* R, const void* out,
                       const void* vbar, const float* lse, const float* tbar, const void* dO, void* dQ, void* dK,
                       void* dV, void* dR, int B, int H, int Hkv, int N, int d, int causal, int window,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * One decode step with split-KV: every (b, h) streams its cache rows
 * 0..seqlens[b]-1; partial results (running max m, omega = sum w, T = sum w t,
 * O1, O2) of the key chunks are merged inside the kernel by the last chunk to
 * finish.  bf16 on the legacy default stream with a library-owned workspace.
 */
int plx_decode(const void* q, const void* r, const void* Kcache, const void* Vcache,
               const int32_t* seqlens, void* out, int B, int H, int L, int d);

/*
 * As plx_decode with an explicit element type, workspace and stream.
 * workspace: device memory of at least plx_decode_workspace_bytes(B, H, L, d)
 * bytes, 256-byte aligned, for the fp32 partial records of the key chunks (no
 * initial contents needed), or NULL for a library-owned workspace, grown on
 * demand, one per device.  The last chunk of each (b, h) to finish is found
 * with an arrival counter; the counters live in a small library-owned array per
 * device (allocated and zeroed on first use, left at zero by every call).
 * Because of that array and of the library-owned workspace, decode calls on one
 * device must be ordered (one stream, or synchronised), not run concurrently.
 */
int plx_decode_ex(const void* q, const void* r, const void* Kcache, const void* Vcache,
                  const int32_t* seqlens, void* out, int B, int H, int L, int d, int dtype,
                  void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace plx_decode_ex needs for these sizes (0 if none is needed). */
size_t plx_decode_workspace_bytes(int B, int H, int L, int d);

/*
 * Number of key chunks each (b, h) is split into for these sizes (the partial
 * records per (b, h) the workspace holds).  For tests and diagnostics.
 */
int plx_decode_num_splits(int B, int H, int L, int d);

/*
 * 1 if plx_decode_ex (bf16) runs these sizes on the tcgen05 decode kernel, 0 if
 * on the warp-MMA kernel (the choice is a pure function of the sizes, made so
 * that the split plan, the workspace size and the launch agree); negative for
 * invalid sizes.  For tests and diagnostics.
 */
int plx_decode_uses_tc(int B, int H, int L, int d);

/*
 * One bf16 decode step with grouped KV heads: H query heads share Hkv KV heads,
 * query head h reading KV head h / (H / Hkv) (consecutive query heads form a
 * group).  The pages' decode packs the q and rho rows into one tensor-core tile
 * so that one stream of K serves both score products (agihunt.info summary,
 * decode paragraph); here that tile carries the rows of every head of a group,
 * so each KV head's cache is read once per step.
 *
 * q, r, out: [B, H, d] bf16; Kcache, Vcache: [B, Hkv, L, d] bf16; seqlens:
 * int32 [B] as for plx_decode (the query of sequence b sees keys
 * 0..seqlens[b]-1; an entry outside 1..L writes zeros for that sequence and
 * reports PLX_ERR_BAD_SEQLEN through plx_get_device_status).  d in {64, 128};
 * H / Hkv in {1, 2, 4, 8} (1 is plx_decode_ex itself), else
 * PLX_ERR_UNSUPPORTED; H not a multiple of Hkv gives PLX_ERR_INVALID_ARG.
 * workspace: NULL (library-owned) or at least
 * plx_decode_gqa_workspace_bytes(B, H, Hkv, L, d) bytes, 256-byte aligned; the
 * arrival counters are the same library-owned per-device array as
 * plx_decode_ex's, so decode calls on one device must be ordered.  Pointers
 * 16-byte aligned (seqlens 4-byte), else PLX_ERR_MISALIGNED.
 */
int plx_decode_gqa(const void* q, const void* r, const void* Kcache, const void* Vcache,
                   const int32_t* seqlens, void* out, int B, int H, int Hkv, int L, int d,
                   void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace plx_decode_gqa needs for these sizes (0 if none is needed). */
size_t plx_decode_gqa_workspace_bytes(int B, int H, int Hkv, int L, int d);

/*
 * Dilated causal prefill: query i sees keys i, i - r, i - 2r, ... (r =
 * dilation), the last `window` of them, or every one back to the start when
 * window is 0.  The pages list kernels that combine Parallax with dilated
 * sparsity next to sliding-window and block-sparse ones as future work
 * (rainbus.top summary, 未来方向) and fix no rule; this is the dilated sliding
 * window.  Every key a query sees lies in its residue class mod r, so each
 * class runs as the causal (windowed) prefill of its own subsequence, read and
 * written through strided views: no masked MMA work.  bf16, d in {64, 128};
 * Q, R, out [B, H, N, d]; K, V [B, Hkv, N, d] (query head h reads KV head
 * h / (H/Hkv)); N must be a multiple of r (else PLX_ERR_UNSUPPORTED).  r = 1
 * is plx_prefill_gqa (window 0) or plx_prefill_gqa_window.
 */
int plx_prefill_dilated(const void* Q, const void* K, const void* V, const void* R, void* out, int B, int H,
                        int Hkv, int N, int d, int dilation, int window, void* stream);

/*
 * Writes an fp8 (e4m3) KV cache: every row of X (bf16 [rows, d], d in {64, 128})
 * gets its own fp32 scale s = max|x| / 448 (scales[row]) and d codes
 * e4m3(x / s) (codes [rows, d], one byte each; round to nearest even, both
 * divisions in IEEE fp32); an all-zero row gets s = 0 and zero codes.  The row
 * then stands for code * s.  This is the reading of the pages' dynamic fp8
 * (rainbus.top summary, reproduction notes: dynamic fp8 precision) for a cache
 * that grows a token at a time: each appended key or value row is quantised on
 * its own, so rows = B*Hkv*L for a whole cache or the new rows of one step.
 * X and codes 16-byte aligned, scales 4-byte aligned; device memory, caller-owned.
 */
int plx_kv_quantize_fp8(const void* X, void* codes, float* scales, long long rows, int d, void* stream);

/* Workspace plx_decode_fp8kv needs for its partial records (0 if keys are not split). */
size_t plx_decode_fp8kv_workspace_bytes(int B, int H, int Hkv, int L, int d);

/*
 * One decode step over an e4m3 KV cache written by plx_kv_quantize_fp8: the
 * result of plx_decode_gqa over the cache values code * scale (rainbus.top
 * summary, 方法步骤详情: the streamed S1/S2, O1/O2 form; out = ((1 + T/omega) O1
 * - O2) / omega).  q, r, out: bf16 [B, H, d]; Kcodes, Vcodes: e4m3 [B, Hkv, L, d];
 * Kscales, Vscales: fp32 [B, Hkv, L]; seqlens: int32 [B] in 1..L (others write
 * zeros and report PLX_ERR_BAD_SEQLEN).  Query head h reads KV head h / (H/Hkv),
 * groups of 1, 2, 4 or 8; d = 128, else PLX_ERR_UNSUPPORTED.  It reads
 * 2 * (d + 4) bytes per cached row instead of the bf16 decode's 4 d.
 * workspace: plx_decode_fp8kv_workspace_bytes() bytes, 256-byte aligned, or NULL
 * for a library-owned one.  Pointers 16-byte aligned (seqlens 4).
 */
int plx_decode_fp8kv(const void* q, const void* r, const void* Kcodes, const float* Kscales,
                     const void* Vcodes, const float* Vscales, const int32_t* seqlens, void* out, int B,
                     int H, int Hkv, int L, int d, void* workspace, size_t workspace_bytes, void* stream);

/*
 * plx_decode_noalloc — one bf16 decode step that allocates nothing.
 * (The paper has no counterpart: this is a deployment variant of plx_decode_ex.)
 *
 * For callers that cannot allocate device memory where they decode: a runtime
 * that reserves all device memory up front and passes kernels only buffers it
 * owns, or a latency-critical loop that must not risk the device-wide
 * synchronisation a cudaMalloc or cudaFree can cause.  Same arguments and
 * result as plx_decode_ex with dtype PLX_BF16, d in {64, 128}; the caller still
 * passes every input and output.  The split-KV scratch (arrival counters and
 * partial records) is a fixed 8 MiB array compiled into the library, which every
 * GPU that loads the library holds until the process exits.  Limits: when the
 * keys are split, B*H <= 32768 and B*H*splits*(2d+4)*4 bytes <= 8 MiB - 128 KiB
 * (splits = plx_decode_num_splits); larger sizes return PLX_ERR_WORKSPACE before
 * anything is launched; sizes plx_decode_ex rejects (B*H > 2^24, B*H*L + 128 >=
 * 2^31) return PLX_ERR_UNSUPPORTED here too.  No cudaMalloc, cudaFree or
 * allocating library routine is called.  The first call on a device looks up the
 * array's device address; under CUDA's lazy module loading (the default) that
 * lookup is also what makes the driver load the array's module and reserve its
 * 8 MiB on that device.  So make the first call on each device before the caller
 * reserves the rest of device memory, and before any stream capture; later calls
 * reserve nothing.  Every call clears the counters with an asynchronous memset on
 * `stream`.  All calls share the one array, so calls that overlap on the GPU
 * (other streams, other threads) race: order them.
 */
int plx_decode_noalloc(const void* q, const void* r, const void* Kcache, const void* Vcache,
                       const int32_t* seqlens, void* out, int B, int H, int L, int d,
                       void* stream);

/*
 * Per-head RMSNorm (unit weight, eps) followed by rotate-half RoPE (frequencies
 * base^(-2k/d), position = token index) of a projected activation, with the
 * head split folded in: x is bf16 [B, N, H*d] (token-major, as a GEMM writes it),
 * y is bf16 [B, H, N, d].  The agihunt.info summary states that rho gets its own
 * RMSNorm and RoPE; q and k take the same treatment (Qwen-3 style).
 */
int plx_qkr_norm_rope(const void* x, void* y, int B, int N, int H, int d, float eps,
                      float rope_base, void* stream);

/* The library-owned scratch a full layer forward needs, in bytes. */
size_t plx_layer_workspace_bytes(int B, int N, int H, int d);

/*
 * Full Parallax attention layer, bf16 (projections with fp32 accumulation):
 *   q,k,v,rho = x W_Q, x W_K, x W_V, x W_R     (W stored [in, out] = [H*d, H*d])
 *   q,k,rho  <- RoPE(RMSNorm(.)) per head     (plx_qkr_norm_rope, eps 1e-6, base 10000)
 *   o         = causal Parallax prefill over [B, H, N, d]
 *   y         = o W_O                          (o merged back to [B, N, H*d])
 * x, y: bf16 [B, N, H*d].  workspace: device memory of plx_layer_workspace_bytes()
 * bytes, 256-byte aligned, or NULL for a library-owned one.  A caller workspace
 * is nine slots of round_up(B*N*H*d*2, 256) bytes; on return slots 4..7 hold the
 * attention inputs q, k, v, rho and slot 8 the attention output, all bf16
 * [B, H, N, d] (slots 0..3 hold the projections, slot 0 then the merged
 * attention output), so a caller can inspect exactly what the prefill consumed.
 */
int plx_layer_forward(const void* x, const void* WQ, const void* WK, const void* WV,
                      const void* WR, const void* WO, void* y, int B, int N, int H, int d,
                      void* workspace, size_t workspace_bytes, void* stream);

/* The scratch plx_layer_forward_fp8 needs, in bytes (includes a 32 MB GEMM workspace). */
size_t plx_layer_fp8_workspace_bytes(int B, int N, int H, int d);

/*
 * The layer of plx_layer_forward with its five linears in dynamic fp8, as the
 * pages pretrain it (rainbus.top reproduction notes: dynamic fp8 for the
 * linear layers): per call and per tensor, s = max|a| / 448 for the input x,
 * each weight and the merged attention output; each operand rounded to e4m3
 * (nearest, ties to even) after division by its scale; e4m3 GEMMs with fp32
 * accumulation, scaled by s_a s_w, written as bf16.  Norms, RoPE and attention
 * as plx_layer_forward (bf16 tensor-core prefill, so d in {64, 128}).
 * B*N must be a multiple of 16 and H*d of 64, else PLX_ERR_UNSUPPORTED.
 * workspace: plx_layer_fp8_workspace_bytes() bytes, 256-byte aligned, or NULL.
 */
int plx_layer_forward_fp8(const void* x, const void* WQ, const void* WK, const void* WV,
                          const void* WR, const void* WO, void* y, int B, int N, int H, int d,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * Waits for `stream`, then reads and clears this device's kernel status word.
 * Returns PLX_OK, or the first device-reported error since the last read
 * (PLX_ERR_BAD_SEQLEN, PLX_ERR_TIMEOUT), or PLX_ERR_CUDA if the wait failed.
 * On PLX_ERR_TIMEOUT it also zeroes the library's decode arrival counters,
 * which a decode whose waits ran out may have left above zero.
 */
int plx_get_device_status(void* stream);

/* Static description of a status code (never NULL). */
const char* plx_status_string(int code);

/* PLX_ABI_VERSION of the loaded library. */
int plx_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PLX_H */
