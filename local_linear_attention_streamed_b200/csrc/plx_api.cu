// C ABI of libplx.so (declared in include/plx.h): host-side validation,
// kernel selection, library-owned workspaces and the per-device status word.
#include "plx_internal.cuh"

#include <cublasLt.h>
#include <cublas_v2.h>

#include <algorithm>
#include <cstdio>
#include <mutex>
#include <vector>

#include "../../include/plx.h"

namespace plx {
namespace {

constexpr int kMaxDevices = 64;

// Per-device kernel status word (bits of kStatus*); kernels atomicOr into it.
__device__ int g_status;

struct DeviceCache {
  bool init = false;
  int num_sms = 0;
  int* status = nullptr;  // device address of g_status on this device
  void* decode_ws = nullptr;  // partial records (library-owned workspace)
  size_t decode_ws_bytes = 0;
  void* counters = nullptr;   // arrival counters, one per (b, h); zero between calls
  size_t counters_bytes = 0;
  void* layer_ws = nullptr;
  size_t layer_ws_bytes = 0;
  void* bwd_ws = nullptr;  // per-row statistics of the prefill backward pass
  size_t bwd_ws_bytes = 0;
  void* sparse_ws = nullptr;  // block lists of the block-sparse prefill
  size_t sparse_ws_bytes = 0;
  cublasHandle_t cublas = nullptr;
  cublasLtHandle_t cublas_lt = nullptr;  // fp8 GEMMs of the fp8 layer
};

std::mutex g_mu;
DeviceCache g_dev[kMaxDevices];

int current_device(DeviceCache** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PLX_ERR_CUDA;
  // Binds the device's primary context to this thread: the tensor-map encoder
  // (a driver call) fails in a thread whose context is not yet current, e.g.
  // an autograd worker that has made no runtime call of its own.
  if (cudaSetDevice(dev) != cudaSuccess) return PLX_ERR_CUDA;
  // Launch failures are read back with cudaGetLastError, which also returns a
  // non-sticky error that an earlier runtime call of this thread left unread
  // (another library's, e.g. on an autograd worker thread).  Drop it here so
  // that only this call's own launches are judged; a sticky error (a faulted
  // context) comes back from the launch itself.
  (void)cudaGetLastError();
  DeviceCache& c = g_dev[dev];
  if (!c.init) {
    if (cudaDeviceGetAttribute(&c.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return PLX_ERR_CUDA;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&c.status), g_status) != cudaSuccess)
      return PLX_ERR_CUDA;
    c.init = true;
  }
  *out = &c;
  return PLX_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The CUDA error behind this thread's last PLX_ERR_CUDA from a launch
// (plx_last_cuda_error reports it).
thread_local cudaError_t t_last_cuda = cudaSuccess;

int cuda_rc(cudaError_t e) {
  if (e == cudaSuccess) return PLX_OK;
  t_last_cuda = e;
  return PLX_ERR_CUDA;
}


// Shapes each kernel family supports.
int check_head_dim(int d, int dtype) {
  if (dtype == PLX_BF16) return (d == 64 || d == 128) ? PLX_OK : PLX_ERR_UNSUPPORTED;
  if (dtype == PLX_F32) return (d >= 32 && d <= 128 && d % 32 == 0) ? PLX_OK : PLX_ERR_UNSUPPORTED;
  return PLX_ERR_INVALID_ARG;
}

// Grows a library-owned buffer; new memory is zeroed (decode counters start at 0).
int grow(void** ptr, size_t* bytes, size_t need, cudaStream_t st) {
  if (*bytes >= need) return PLX_OK;
  if (*ptr) {
    if (cudaFree(*ptr) != cudaSuccess) return PLX_ERR_CUDA;
    *ptr = nullptr;
    *bytes = 0;
  }
  if (cudaMalloc(ptr, need) != cudaSuccess) {
    *ptr = nullptr;
    return PLX_ERR_CUDA;
  }
  if (cudaMemsetAsync(*ptr, 0, need, st) != cudaSuccess) return PLX_ERR_CUDA;
  *bytes = need;
  return PLX_OK;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr size_t kLtWorkspace = 32u << 20;  // cuBLASLt workspace of the fp8 GEMMs

// Bytes of partial records a split decode needs (0 when keys are not split).
size_t decode_ws_layout(int B, int H, int L, int d, int num_sms, int* splits, int* chunk) {
  decode_bf16_plan(B, H, L, d, num_sms, splits, chunk);
  if (*splits <= 1) return 0;
  return sizeof(float) * (size_t)B * H * (size_t)(*splits) * (size_t)(2 * d + 4);
}

int num_sms_or_default() {
  DeviceCache* c = nullptr;
  if (current_device(&c) == PLX_OK) return c->num_sms;
  return 148;
}

}  // namespace

int* status_word_address() {
  DeviceCache* c = nullptr;
  return current_device(&c) == PLX_OK ? c->status : nullptr;
}

}  // namespace plx

using namespace plx;

extern "C" {

int plx_abi_version(void) { return PLX_ABI_VERSION; }

const char* plx_last_cuda_error(void) {
  thread_local char buf[160];
  const char* where = bwd_last_failure();
  snprintf(buf, sizeof buf, "%s%s%s", cudaGetErrorString(t_last_cuda), where[0] ? " at " : "", where);
  return buf;
}

const char* plx_status_string(int code) {
  switch (code) {
    case PLX_OK: return "ok";
    case PLX_ERR_INVALID_ARG: return "invalid argument (null pointer, non-positive size or bad enum)";
    case PLX_ERR_UNSUPPORTED: return "unsupported head dimension / dtype combination";
    case PLX_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
    case PLX_ERR_CUDA: return "CUDA runtime or launch failure";
    case PLX_ERR_WORKSPACE: return "workspace too small";
    case PLX_ERR_BAD_SEQLEN: return "device reported a seqlens entry outside 1..L";
    case PLX_ERR_TIMEOUT: return "device reported a bounded wait that ran out";
    default: return "unknown status code";
  }
}

static int prefill_impl(const void* Q, const void* K, const void* V, const void* R, void* out, int B, int H,
                        int N, int d, int causal, int window, int dtype, void* stream) {
  if (!Q || !K || !V || !R || !out) return PLX_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || d < 1) return PLX_ERR_INVALID_ARG;
  if (dtype != PLX_F32 && dtype != PLX_BF16) return PLX_ERR_INVALID_ARG;
  int rc = check_head_dim(d, dtype);
  if (rc != PLX_OK) return rc;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(R) || !aligned16(out))
    return PLX_ERR_MISALIGNED;
  if ((long long)B * H > (1ll << 24)) return PLX_ERR_UNSUPPORTED;
  DeviceCache* dc = nullptr;
  if ((rc = current_device(&dc)) != PLX_OK) return rc;
  PrefillArgs a{Q, K, V, R, out, B, H, N, d, causal ? 1 : 0, dc->status};
  a.window = window < N ? window : 0;  // a window of N or more keys is the causal prefill
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (dtype == PLX_BF16 && prefill_tc_supported(d)) {
    e = launch_prefill_tc(a, st, dc->num_sms);
  } else {
    e = launch_prefill_simt(a, dtype == PLX_BF16, st);
  }
  return cuda_rc(e);
}

int plx_prefill_ex(const void* Q, const void* K, const void* V, const void* R, void* out, int B,
                   int H, int N, int d, int causal, int dtype, void* stream) {
  return prefill_impl(Q, K, V, R, out, B, H, N, d, causal, 0, dtype, stream);
}

int plx_prefill_window(const void* Q, const void* K, const void* V, const void* R, void* out, int B,
                       int H, int N, int d, int window, int dtype, void* stream) {
  if (window < 1) return PLX_ERR_INVALID_ARG;
  return prefill_impl(Q, K, V, R, out, B, H, N, d, 1, window, dtype, stream);
}

static int prefill_gqa_impl(const void* Q, const void* K, const void* V, const void* R, void* out, int B, int H,
                            int Hkv, int N, int d, int causal, int window, void* stream) {
  if (!Q || !K || !V || !R || !out) return PLX_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Hkv < 1 || N < 1 || d < 1 || H % Hkv != 0) return PLX_ERR_INVALID_ARG;
  if (!prefill_tc_supported(d)) return PLX_ERR_UNSUPPORTED;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(R) || !aligned16(out))
    return PLX_ERR_MISALIGNED;
  if ((long long)B * H > (1ll << 24)) return PLX_ERR_UNSUPPORTED;
  int rc;
  DeviceCache* dc = nullptr;
  if ((rc = current_device(&dc)) != PLX_OK) return rc;
  PrefillArgs a{Q, K, V, R, out, B, H, N, d, causal ? 1 : 0, dc->status};
  a.Hkv = Hkv;
  a.window = window < N ? window : 0;
  return cuda_rc(launch_prefill_tc(a, reinterpret_cast<cudaStream_t>(stream), dc->num_sms));
}

int plx_prefill_gqa(const void* Q, const void* K, const void* V, const void* R, void* out, int B, int H,
                    int Hkv, int N, int d, int causal, void* stream) {
  return prefill_gqa_impl(Q, K, V, R, out, B, H, Hkv, N, d, causal, 0, stream);
}

int plx_prefill_gqa_window(const void* Q, const void* K, const void* V, const void* R, void* out, int B, int H,
                           int Hkv, int N, int d, int window, void* stream) {
  if (window < 1) return PLX_ERR_INVALID_ARG;
  return prefill_gqa_impl(Q, K, V, R, out, B, H, Hkv, N, d, 1, window, stream);
}

int plx_prefill_dilated(const void* Q, const void* K, const void* V, const void* R, void* out, int B, int H,
                        int Hkv, int N, int d, int dilation, int window, void* stream) {
  if (!Q || !K || !V || !R || !out) return PLX_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Hkv < 1 || N < 1 || d < 1 || H % Hkv != 0 || dilation < 1 || window < 0)
    return PLX_ERR_INVALID_ARG;
  if (!prefill_tc_supported(d) || N % dilation != 0) return PLX_ERR_UNSUPPORTED;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(R) || !aligned16(out))
    return PLX_ERR_MISALIGNED;
  if ((long long)B * H * dilation > (1ll << 24)) return PLX_ERR_UNSUPPORTED;
  int rc;
  DeviceCache* dc = nullptr;
  if ((rc = current_device(&dc)) != PLX_OK) return rc;
  PrefillArgs a{Q, K, V, R, out, B, H, N, d, 1, dc->status};
  a.Hkv = Hkv;
  a.dilation = dilation;
  // The window counts keys of the query's residue class; one covering the
  // whole class (N / dilation keys) is the causal mask within the class.
  a.window = window < N / dilation ? window : 0;
  return cuda_rc(launch_prefill_tc(a, reinterpret_cast<cudaStream_t>(stream), dc->num_sms));
}

int plx_prefill_block_sparse(const void* Q, const void* K, const void* V, const void* R, void* out, int B,
                             int H, int N, int d, const uint8_t* block_mask, void* stream) {
  if (!Q || !K || !V || !R || !out || !block_mask) return PLX_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || d < 1) return PLX_ERR_INVALID_ARG;
  if (!prefill_tc_supported(d)) return PLX_ERR_UNSUPPORTED;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(R) || !aligned16(out))
    return PLX_ERR_MISALIGNED;
  if ((long long)B * H > (1ll << 24)) return PLX_ERR_UNSUPPORTED;
  // The mask as lists of active key blocks per tile (blocks above a tile's
  // diagonal hold no visible key and are dropped); every row must see its
  // own key, so each tile's diagonal blocks must be active.
  const int ntile = (N + 127) / 128, nkb = (N + 63) / 64;
  std::vector<int> list;
  list.reserve((size_t)ntile + 1 + (size_t)ntile * 2);
  list.resize((size_t)ntile + 1);
  for (int m = 0; m < ntile; ++m) {
    list[m] = (int)(list.size() - (ntile + 1));
    const int last = std::min(nkb - 1, 2 * m + 1);
    for (int kb = 0; kb <= last; ++kb) {
      const bool on = block_mask[(size_t)m * nkb + kb] != 0;
      if (kb >= 2 * m && !on) return PLX_ERR_INVALID_ARG;  // a diagonal block is off
      if (on) list.push_back(kb);
    }
  }
  list[ntile] = (int)(list.size() - (ntile + 1));
  int rc;
  DeviceCache* dc = nullptr;
  if ((rc = current_device(&dc)) != PLX_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t bytes = list.size() * sizeof(int);
  std::lock_guard<std::mutex> lk(g_mu);
  if ((rc = grow(&dc->sparse_ws, &dc->sparse_ws_bytes, bytes, st)) != PLX_OK) return rc;
  if (cudaMemcpyAsync(dc->sparse_ws, list.data(), bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return PLX_ERR_CUDA;
  PrefillArgs a{Q, K, V, R, out, B, H, N, d, 1, dc->status};
  a.blk_ptr = static_cast<const int*>(dc->sparse_ws);
  a.blk_idx = a.blk_ptr + ntile + 1;
  return cuda_rc(launch_prefill_tc(a, st, dc->num_sms));
}

int plx_prefill(const void* Q, const void* K, const void* V, const void* R, void* out, int B,
                int H, int N, int d, int causal) {
  return plx_prefill_ex(Q, K, V, R, out, B, H, N, d, causal, PLX_BF16, nullptr);
}

static int prefill_train_impl(const void* Q, const void* K, const void* V, const void* R, void* out,
                              void* vbar, float* lse, float* tbar, int B, int H, int N, int d, int causal,
                              int window, void* stream, int Hkv = 0) {
  if (!Q || !K || !V || !R || !out || !vbar || !lse || !tbar) return PLX_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || d < 1) return PLX_ERR_INVALID_ARG;
  if (Hkv != 0 && (Hkv < 1 || H % Hkv != 0)) return PLX_ERR_INVALID_ARG;
  if (!prefill_tc_supported(d)) return PLX_ERR_UNSUPPORTED;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(R) || !aligned16(out) ||
      !aligned16(vbar) || (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(tbar) & 3u))
    return PLX_ERR_MISALIGNED;
  if ((long long)B * H > (1ll << 24)) return PLX_ERR_UNSUPPORTED;
  int rc;
  DeviceCache* dc = nullptr;
  if ((rc = current_device(&dc)) != PLX_OK) return rc;
  PrefillArgs a{Q, K, V, R, out, B, H, N, d, causal ? 1 : 0, dc->status};
  a.vbar = vbar;
  a.lse = lse;
  a.tbar = tbar;
  a.window = window < N ? window : 0;
  a.Hkv = Hkv > 0 ? Hkv : H;
  return cuda_rc(launch_prefill_tc(a, reinterpret_cast<cudaStream_t>(stream), dc->num_sms));
}

int plx_prefill_train(const void* Q, const void* K, const void* V, const void* R, void* out,
                      void* vbar, float* lse, float* tbar, int B, int H, int N, int d, int causal,
                      void* stream) {
  return prefill_train_impl(Q, K, V, R, out, vbar, lse, tbar, B, H, N, d, causal, 0, stream);
}

int plx_prefill_train_window(const void* Q, const void* K, const void* V, const void* R, void* out,
                             void* vbar, float* lse, float* tbar, int B, int H, int N, int d, int window,
                             void* stream) {
  if (window < 1) return PLX_ERR_INVALID_ARG;
  return prefill_train_impl(Q, K, V, R, out, vbar, lse, tbar, B, H, N, d, 1, window, stream);
}

int plx_prefill_train_ex(const void* Q, const void* K, const void* V, const void* R, void* out, void* vbar,
                         float* lse, float* tbar, int B, int H, int Hkv, int N, int d, int causal, int window,
                         void* stream) {
  if (Hkv < 1 || window < 0) return PLX_ERR_INVALID_ARG;
  return prefill_train_impl(Q, K, V, R, out, vbar, lse, tbar, B, H, N, d, window > 0 ? 1 : causal, window, stream,
                            Hkv);
}

int plx_prefill_train_gqa(const void* Q, const void* K, const void* V, const void* R, void* out, void* vbar,
                          float* lse, float* tbar, int B, int H, int Hkv, int N, int d, int causal,
                          void* stream) {
  if (Hkv < 1) return PLX_ERR_INVALID_ARG;
  return prefill_train_impl(Q, K, V, R, out, vbar, lse, tbar, B, H, N, d, causal, 0, stream, Hkv);
}

size_t plx_prefill_bwd_workspace_bytes(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || d < 1) return 0;
  return 16 * (size_t)B * H * bwd_padded_rows(N);
}

static int prefill_bwd_impl(const void* Q, const void* K, const void* V, const void* R, const void* out,
                            const void* vbar, const float* lse, const float* tbar, const void* dO, void* dQ,
                            void* dK, void* dV, void* dR, int B, int H, int N, int d, int causal, int window,
                            void* workspace, size_t workspace_bytes, void* stream, int Hkv = 0) {
  if (!Q || !K || !V || !R || !out || !vbar || !lse || !tbar || !dO || !dQ || !dK || !dV || !dR)
    return PLX_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || d < 1) return PLX_ERR_INVALID_ARG;
  if (Hkv != 0 && (Hkv < 1 || H % Hkv != 0)) return PLX_ERR_INVALID_ARG;
  if (!prefill_tc_supported(d)) return PLX_ERR_UNSUPPORTED;
  const void* t16[] = {Q, K, V, R, out, vbar, dO, dQ, dK, dV, dR};
  for (const void* t : t16)
    if (!aligned16(t)) return PLX_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(tbar) & 3u))
    return PLX_ERR_MISALIGNED;
  if ((long long)B * H * (long long)bwd_padded_rows(N) >= (1ll << 31)) return PLX_ERR_UNSUPPORTED;
  const size_t need = plx_prefill_bwd_workspace_bytes(B, H, N, d);
  if (workspace && workspace_bytes < need) return PLX_ERR_WORKSPACE;
  if (workspace && !aligned16(workspace)) return PLX_ERR_MISALIGNED;
  int rc;
  DeviceCache* dc = nullptr;
  if ((rc = current_device(&dc)) != PLX_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  BwdArgs a{Q, K, V, R, out, vbar, dO, lse, tbar, dQ, dK, dV, dR, B, H, N, d, causal ? 1 : 0, workspace,
            dc->status};
  a.window = window < N ? window : 0;
  a.Hkv = Hkv > 0 ? Hkv : H;
  if (!workspace) {
    std::lock_guard<std::mutex> lk(g_mu);
    if ((rc = grow(&dc->bwd_ws, &dc->bwd_ws_bytes, need, st)) != PLX_OK) return rc;
    a.stats = dc->bwd_ws;
    return cuda_rc(launch_prefill_bwd(a, st, dc->num_sms));
  }
  return cuda_rc(launch_prefill_bwd(a, st, dc->num_sms));
}

int plx_prefill_bwd(const void* Q, const void* K, const void* V, const void* R, const void* out,
                    const void* vbar, const float* lse, const float* tbar, const void* dO, void* dQ,
                    void* dK, void* dV, void* dR, int B, int H, int N, int d, int causal,
                    void* workspace, size_t workspace_bytes, void* stream) {
  return prefill_bwd_impl(Q, K, V, R, out, vbar, lse, tbar, dO, dQ, dK, dV, dR, B, H, N, d, causal, 0, workspace,
                          workspace_bytes, stream);
}

int plx_prefill_bwd_window(const void* Q, const void* K, const void* V, const void* R, const void* out,
                           const void* vbar, const float* lse, const float* tbar, const void* dO, void* dQ,
                           void* dK, void* dV, void* dR, int B, int H, int N, int d, int window,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (window < 1) return PLX_ERR_INVALID_ARG;
  return prefill_bwd_impl(Q, K, V, R, out, vbar, lse, tbar, dO, dQ, dK, dV, dR, B, H, N, d, 1, window, workspace,
                          workspace_bytes, stream);
}

int plx_prefill_bwd_ex(const void* Q, const void* K, const void* V, const void* R, const void* out,
                       const void* vbar, const float* lse, const float* tbar, const void* dO, void* dQ, void* dK,
                       void* dV, void* dR, int B, int H, int Hkv, int N, int d, int causal, int window,
                       void* workspace, size_t workspace_bytes, void* stream) {
  if (Hkv < 1 || window < 0) return PLX_ERR_INVALID_ARG;
  return prefill_bwd_impl(Q, K, V, R, out, vbar, lse, tbar, dO, dQ, dK, dV, dR, B, H, N, d, window > 0 ? 1 : causal,
                          window, workspace, workspace_bytes, stream, Hkv);
}

int plx_prefill_bwd_gqa(const void* Q, const void* K, const void* V, const void* R, const void* out,
                        const void* vbar, const float* lse, const float* tbar, const void* dO, void* dQ, void* dK,
                        void* dV, void* dR, int B, int H, int Hkv, int N, int d, int causal, void* workspace,
                        size_t workspace_bytes, void* stream) {
  if (Hkv < 1) return PLX_ERR_INVALID_ARG;
  return prefill_bwd_impl(Q, K, V, R, out, vbar, lse, tbar, dO, dQ, dK, dV, dR, B, H, N, d, causal, 0, workspace,
                          workspace_bytes, stream, Hkv);
}

int plx_decode_num_splits(int B, int H, int L, int d) {
  (void)d;
  if (B < 1 || H < 1 || L < 1) return 0;
  int splits = 1, chunk = 0;
  decode_bf16_plan(B, H, L, d, num_sms_or_default(), &splits, &chunk);
  return splits;
}

int plx_decode_uses_tc(int B, int H, int L, int d) {
  if (B < 1 || H < 1 || L < 1 || (d != 64 && d != 128)) return PLX_ERR_INVALID_ARG;
  return decode_bf16_tc_h(B, H, L, d) ? 1 : 0;
}

size_t plx_decode_workspace_bytes(int B, int H, int L, int d) {
  if (B < 1 || H < 1 || L < 1 || d < 1) return 0;
  int splits = 1, chunk = 0;
  return decode_ws_layout(B, H, L, d, num_sms_or_default(), &splits, &chunk);
}

static int decode_impl(const void* q, const void* r, const void* Kcache, const void* Vcache,
                       const int32_t* seqlens, void* out, int B, int H, int L, int d, int window, int dtype,
                       void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !r || !Kcache || !Vcache || !seqlens || !out) return PLX_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || L < 1 || d < 1) return PLX_ERR_INVALID_ARG;
  if (dtype != PLX_F32 && dtype != PLX_BF16) return PLX_ERR_INVALID_ARG;
  int rc = check_head_dim(d, dtype);
  if (rc != PLX_OK) return rc;
  if (!aligned16(q) || !aligned16(r) || !aligned16(Kcache) || !aligned16(Vcache) ||
      !aligned16(out) || (reinterpret_cast<uintptr_t>(seqlens) & 3u))
    return PLX_ERR_MISALIGNED;
  if (!decode_sizes_supported(B, H, H, L)) return PLX_ERR_UNSUPPORTED;
  DeviceCache* dc = nullptr;
  if ((rc = current_device(&dc)) != PLX_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DecodeArgs a{};
  a.q = q;
  a.r = r;
  a.K = Kcache;
  a.V = Vcache;
  a.seqlens = seqlens;
  a.out = out;
  a.B = B;
  a.H = H;
  a.L = L;
  a.d = d;
  a.status = dc->status;
  a.window = window < L ? window : 0;
  if (dtype == PLX_F32) {
    return cuda_rc(launch_decode_simt(a, false, st));
  }
  // The split plan covers the keys one query can see (the window, when set).
  size_t need = decode_ws_layout(B, H, a.window > 0 ? a.window : L, d, dc->num_sms, &a.splits, &a.chunk);
  if (need > 0) {
    if (workspace && workspace_bytes < need) return PLX_ERR_WORKSPACE;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return PLX_ERR_MISALIGNED;
    std::lock_guard<std::mutex> lk(g_mu);
    // The counters live apart from the partial records so that no call's
    // records can ever land where a later call (other B*H) keeps counters.
    if ((rc = grow(&dc->counters, &dc->counters_bytes, sizeof(int) * (size_t)B * H, st)) != PLX_OK)
      return rc;
    a.counters = static_cast<int*>(dc->counters);
    if (workspace) {
      a.partials = static_cast<float*>(workspace);
    } else {
      if ((rc = grow(&dc->decode_ws, &dc->decode_ws_bytes, need, st)) != PLX_OK) return rc;
      a.partials = static_cast<float*>(dc->decode_ws);
    }
  }
  return cuda_rc(launch_decode_bf16(a, st, dc->num_sms));
}

int plx_decode_ex(const void* q, const void* r, const void* Kcache, const void* Vcache,
                  const int32_t* seqlens, void* out, int B, int H, int L, int d, int dtype,
                  void* workspace, size_t workspace_bytes, void* stream) {
  return decode_impl(q, r, Kcache, Vcache, seqlens, out, B, H, L, d, 0, dtype, workspace, workspace_bytes,
                     stream);
}

size_t plx_decode_gqa_workspace_bytes(int B, int H, int Hkv, int L, int d) {
  if (B < 1 || H < 1 || Hkv < 1 || L < 1 || d < 1 || H % Hkv != 0) return 0;
  if (H == Hkv) return plx_decode_workspace_bytes(B, H, L, d);
  int splits = 1, chunk = 0;
  decode_split_plan(B, Hkv / decode_gqa_kv_per_unit(Hkv, d), L, num_sms_or_default(), &splits, &chunk,
                    decode_gqa_ctas_per_sm(H / Hkv, Hkv, d));
  if (splits <= 1) return 0;
  return sizeof(float) * (size_t)B * H * (size_t)splits * (size_t)(2 * d + 4);
}

static int decode_gqa_impl(const void* q, const void* r, const void* Kcache, const void* Vcache,
                           const int32_t* seqlens, void* out, int B, int H, int Hkv, int L, int d, int window,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !r || !Kcache || !Vcache || !seqlens || !out) return PLX_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Hkv < 1 || L < 1 || d < 1 || H % Hkv != 0) return PLX_ERR_INVALID_ARG;
  const int G = H / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PLX_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return PLX_ERR_UNSUPPORTED;
  if (G == 1)
    return decode_impl(q, r, Kcache, Vcache, seqlens, out, B, H, L, d, window, PLX_BF16, workspace,
                       workspace_bytes, stream);
  if (!aligned16(q) || !aligned16(r) || !aligned16(Kcache) || !aligned16(Vcache) ||
      !aligned16(out) || (reinterpret_cast<uintptr_t>(seqlens) & 3u))
    return PLX_ERR_MISALIGNED;
  if (!decode_sizes_supported(B, H, Hkv, L)) return PLX_ERR_UNSUPPORTED;
  int rc;
  DeviceCache* dc = nullptr;
  if ((rc = current_device(&dc)) != PLX_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DecodeArgs a{};
  a.q = q;
  a.r = r;
  a.K = Kcache;
  a.V = Vcache;
  a.seqlens = seqlens;
  a.out = out;
  a.B = B;
  a.H = H;
  a.Hkv = Hkv;
  a.L = L;
  a.d = d;
  a.status = dc->status;
  a.window = window < L ? window : 0;
  decode_split_plan(B, Hkv / decode_gqa_kv_per_unit(Hkv, d), a.window > 0 ? a.window : L, dc->num_sms, &a.splits,
                    &a.chunk, decode_gqa_ctas_per_sm(G, Hkv, d));
  if (a.splits > 1) {
    const size_t need = sizeof(float) * (size_t)B * H * (size_t)a.splits * (size_t)(2 * d + 4);
    if (workspace && workspace_bytes < need) return PLX_ERR_WORKSPACE;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return PLX_ERR_MISALIGNED;
    std::lock_guard<std::mutex> lk(g_mu);
    // One arrival counter per (b, KV head), in the same library-owned array
    // (always left at zero) as the ungrouped decode's.
    if ((rc = grow(&dc->counters, &dc->counters_bytes, sizeof(int) * (size_t)B * Hkv, st)) != PLX_OK)
      return rc;
    a.counters = static_cast<int*>(dc->counters);
    if (workspace) {
      a.partials = static_cast<float*>(workspace);
    } else {
      if ((rc = grow(&dc->decode_ws, &dc->decode_ws_bytes, need, st)) != PLX_OK) return rc;
      a.partials = static_cast<float*>(dc->decode_ws);
    }
  }
  return cuda_rc(launch_decode_gqa(a, st, dc->num_sms));
}

int plx_decode_gqa(const void* q, const void* r, const void* Kcache, const void* Vcache,
                   const int32_t* seqlens, void* out, int B, int H, int Hkv, int L, int d,
                   void* workspace, size_t workspace_bytes, void* stream) {
  return decode_gqa_impl(q, r, Kcache, Vcache, seqlens, out, B, H, Hkv, L, d, 0, workspace, workspace_bytes,
                         stream);
}

int plx_kv_quantize_fp8(const void* X, void* codes, float* scales, long long rows, int d, void* stream) {
  if (!X || !codes || !scales || rows < 1) return PLX_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return PLX_ERR_UNSUPPORTED;
  if (!aligned16(X) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u)) return PLX_ERR_MISALIGNED;
  DeviceCache* dc = nullptr;
  int rc = current_device(&dc);
  if (rc != PLX_OK) return rc;
  return cuda_rc(launch_kv_quantize_fp8(X, codes, scales, rows, d, reinterpret_cast<cudaStream_t>(stream)));
}

size_t plx_decode_fp8kv_workspace_bytes(int B, int H, int Hkv, int L, int d) {
  if (B < 1 || H < 1 || Hkv < 1 || L < 1 || d < 1 || H % Hkv != 0) return 0;
  int splits = 1, chunk = 0;
  decode_split_plan(B, Hkv, L, num_sms_or_default(), &splits, &chunk, 1);
  if (splits <= 1) return 0;
  return sizeof(float) * (size_t)B * H * (size_t)splits * (size_t)(2 * d + 4);
}

int plx_decode_fp8kv(const void* q, const void* r, const void* Kcodes, const float* Kscales, const void* Vcodes,
                     const float* Vscales, const int32_t* seqlens, void* out, int B, int H, int Hkv, int L, int d,
                     void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !r || !Kcodes || !Kscales || !Vcodes || !Vscales || !seqlens || !out) return PLX_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Hkv < 1 || L < 1 || d < 1 || H % Hkv != 0) return PLX_ERR_INVALID_ARG;
  const int G = H / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PLX_ERR_UNSUPPORTED;
  if (d != 128) return PLX_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(r) || !aligned16(Kcodes) || !aligned16(Vcodes) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(seqlens) & 3u) || !aligned16(Kscales) || !aligned16(Vscales))
    return PLX_ERR_MISALIGNED;
  if (!decode_sizes_supported(B, H, Hkv, L)) return PLX_ERR_UNSUPPORTED;
  int rc;
  DeviceCache* dc = nullptr;
  if ((rc = current_device(&dc)) != PLX_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DecodeArgs a{};
  a.q = q;
  a.r = r;
  a.K = Kcodes;
  a.V = Vcodes;
  a.Kscale = Kscales;
  a.Vscale = Vscales;
  a.seqlens = seqlens;
  a.out = out;
  a.B = B;
  a.H = H;
  a.Hkv = Hkv;
  a.L = L;
  a.d = d;
  a.status = dc->status;
  decode_split_plan(B, Hkv, L, dc->num_sms, &a.splits, &a.chunk, 1);
  if (a.splits > 1) {
    const size_t need = sizeof(float) * (size_t)B * H * (size_t)a.splits * (size_t)(2 * d + 4);
    if (workspace && workspace_bytes < need) return PLX_ERR_WORKSPACE;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return PLX_ERR_MISALIGNED;
    std::lock_guard<std::mutex> lk(g_mu);
    if ((rc = grow(&dc->counters, &dc->counters_bytes, sizeof(int) * (size_t)B * Hkv, st)) != PLX_OK) return rc;
    a.counters = static_cast<int*>(dc->counters);
    if (workspace) {
      a.partials = static_cast<float*>(workspace);
    } else {
      if ((rc = grow(&dc->decode_ws, &dc->decode_ws_bytes, need, st)) != PLX_OK) return rc;
      a.partials = static_cast<float*>(dc->decode_ws);
    }
  }
  return cuda_rc(launch_decode_fp8kv(a, st, dc->num_sms));
}

size_t plx_decode_window_workspace_bytes(int B, int H, int Hkv, int L, int d, int window) {
  if (window < 1) return 0;
  const int Leff = window < L ? window : L;
  return Hkv == H ? plx_decode_workspace_bytes(B, H, Leff, d) : plx_decode_gqa_workspace_bytes(B, H, Hkv, Leff, d);
}

int plx_decode_window(const void* q, const void* r, const void* Kcache, const void* Vcache,
                      const int32_t* seqlens, void* out, int B, int H, int Hkv, int L, int d, int window,
                      int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  if (window < 1 || Hkv < 1) return PLX_ERR_INVALID_ARG;
  if (Hkv == H)
    return decode_impl(q, r, Kcache, Vcache, seqlens, out, B, H, L, d, window, dtype, workspace, workspace_bytes,
                       stream);
  if (dtype != PLX_BF16) return PLX_ERR_UNSUPPORTED;
  return decode_gqa_impl(q, r, Kcache, Vcache, seqlens, out, B, H, Hkv, L, d, window, workspace, workspace_bytes,
                         stream);
}

int plx_decode(const void* q, const void* r, const void* Kcache, const void* Vcache,
               const int32_t* seqlens, void* out, int B, int H, int L, int d) {
  return plx_decode_ex(q, r, Kcache, Vcache, seqlens, out, B, H, L, d, PLX_BF16, nullptr, 0,
                       nullptr);
}

int plx_qkr_norm_rope(const void* x, void* y, int B, int N, int H, int d, float eps,
                      float rope_base, void* stream) {
  if (!x || !y) return PLX_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || H < 1 || !(eps >= 0.f) || !(rope_base > 0.f)) return PLX_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return PLX_ERR_UNSUPPORTED;
  if ((long long)B * N * H * d >= (1ll << 31)) return PLX_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(y)) return PLX_ERR_MISALIGNED;
  return cuda_rc(launch_qkr_norm_rope(x, y, B, N, H, d, eps, rope_base,
                              reinterpret_cast<cudaStream_t>(stream)));
}

size_t plx_layer_workspace_bytes(int B, int N, int H, int d) {
  if (B < 1 || N < 1 || H < 1 || d < 1) return 0;
  size_t t = round_up((size_t)B * N * H * d * 2, 256);
  return 9 * t;  // 4 projections, 4 head-split tensors, attention output
}

int plx_layer_forward(const void* x, const void* WQ, const void* WK, const void* WV, const void* WR,
                      const void* WO, void* y, int B, int N, int H, int d, void* workspace,
                      size_t workspace_bytes, void* stream) {
  if (!x || !WQ || !WK || !WV || !WR || !WO || !y) return PLX_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || H < 1) return PLX_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return PLX_ERR_UNSUPPORTED;
  if ((long long)B * N * H * d >= (1ll << 31)) return PLX_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(WQ) || !aligned16(WK) || !aligned16(WV) || !aligned16(WR) ||
      !aligned16(WO) || !aligned16(y))
    return PLX_ERR_MISALIGNED;
  DeviceCache* dc = nullptr;
  int rc = current_device(&dc);
  if (rc != PLX_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  size_t need = plx_layer_workspace_bytes(B, N, H, d);
  char* ws = nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (workspace) {
    if (workspace_bytes < need) return PLX_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return PLX_ERR_MISALIGNED;
    ws = static_cast<char*>(workspace);
  } else {
    if ((rc = grow(&dc->layer_ws, &dc->layer_ws_bytes, need, st)) != PLX_OK) return rc;
    ws = static_cast<char*>(dc->layer_ws);
  }
  if (!dc->cublas) {
    if (cublasCreate(&dc->cublas) != CUBLAS_STATUS_SUCCESS) {
      dc->cublas = nullptr;
      return PLX_ERR_CUDA;
    }
  }
  if (cublasSetStream(dc->cublas, st) != CUBLAS_STATUS_SUCCESS) return PLX_ERR_CUDA;
  const size_t t = round_up((size_t)B * N * H * d * 2, 256);
  void* proj[4] = {ws, ws + t, ws + 2 * t, ws + 3 * t};          // q, k, v, rho: [B, N, H*d]
  void* head[4] = {ws + 4 * t, ws + 5 * t, ws + 6 * t, ws + 7 * t};  // [B, H, N, d]
  void* attn = ws + 8 * t;                                       // [B, H, N, d]
  const void* W[4] = {WQ, WK, WV, WR};
  const int D = H * d;
  const long long M = (long long)B * N;
  const float one = 1.f, zero = 0.f;
  // Row-major Y[M, D] = X[M, D] W[D, D] is column-major Y^T = W^T X^T.
  for (int i = 0; i < 4; ++i) {
    if (cublasGemmEx(dc->cublas, CUBLAS_OP_N, CUBLAS_OP_N, D, (int)M, D, &one, W[i], CUDA_R_16BF, D,
                     x, CUDA_R_16BF, D, &zero, proj[i], CUDA_R_16BF, D, CUBLAS_COMPUTE_32F,
                     CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
      return PLX_ERR_CUDA;
  }
  const float eps = 1e-6f, base = 10000.f;
  if (launch_qkr_norm_rope(proj[0], head[0], B, N, H, d, eps, base, st) != cudaSuccess ||
      launch_qkr_norm_rope(proj[1], head[1], B, N, H, d, eps, base, st) != cudaSuccess ||
      launch_swap_axes(proj[2], head[2], B, N, H, d, st) != cudaSuccess ||
      launch_qkr_norm_rope(proj[3], head[3], B, N, H, d, eps, base, st) != cudaSuccess)
    return PLX_ERR_CUDA;
  PrefillArgs a{head[0], head[1], head[2], head[3], attn, B, H, N, d, 1, dc->status};
  cudaError_t e = prefill_tc_supported(d) ? launch_prefill_tc(a, st, dc->num_sms)
                                          : launch_prefill_simt(a, true, st);
  if (e != cudaSuccess) return PLX_ERR_CUDA;
  // Merge heads back to [B, N, H*d] (reusing the q projection buffer), then W_O.
  if (launch_swap_axes(attn, proj[0], B, H, N, d, st) != cudaSuccess) return PLX_ERR_CUDA;
  if (cublasGemmEx(dc->cublas, CUBLAS_OP_N, CUBLAS_OP_N, D, (int)M, D, &one, WO, CUDA_R_16BF, D,
                   proj[0], CUDA_R_16BF, D, &zero, y, CUDA_R_16BF, D, CUBLAS_COMPUTE_32F,
                   CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
    return PLX_ERR_CUDA;
  return PLX_OK;
}

size_t plx_layer_fp8_workspace_bytes(int B, int N, int H, int d) {
  if (B < 1 || N < 1 || H < 1 || d < 1) return 0;
  const size_t M = (size_t)B * N, D = (size_t)H * d;
  // bf16 buffers of the bf16 layer, two e4m3 activations, five e4m3 weights,
  // the scales, and the GEMM's workspace.
  return plx_layer_workspace_bytes(B, N, H, d) + 2 * round_up(M * D, 256) + 5 * round_up(D * D, 256) + 256 +
         kLtWorkspace;
}

int plx_layer_forward_fp8(const void* x, const void* WQ, const void* WK, const void* WV, const void* WR,
                          const void* WO, void* y, int B, int N, int H, int d, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (!x || !WQ || !WK || !WV || !WR || !WO || !y) return PLX_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || H < 1) return PLX_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return PLX_ERR_UNSUPPORTED;
  if ((long long)B * N * H * d >= (1ll << 31)) return PLX_ERR_UNSUPPORTED;
  if (((long long)B * N) % 16 != 0 || (H * d) % 64 != 0) return PLX_ERR_UNSUPPORTED;  // fp8 operand tiles
  if (!aligned16(x) || !aligned16(WQ) || !aligned16(WK) || !aligned16(WV) || !aligned16(WR) ||
      !aligned16(WO) || !aligned16(y))
    return PLX_ERR_MISALIGNED;
  DeviceCache* dc = nullptr;
  int rc = current_device(&dc);
  if (rc != PLX_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t need = plx_layer_fp8_workspace_bytes(B, N, H, d);
  char* ws = nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (workspace) {
    if (workspace_bytes < need) return PLX_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return PLX_ERR_MISALIGNED;
    ws = static_cast<char*>(workspace);
  } else {
    if ((rc = grow(&dc->layer_ws, &dc->layer_ws_bytes, need, st)) != PLX_OK) return rc;
    ws = static_cast<char*>(dc->layer_ws);
  }
  if (!dc->cublas_lt) {
    if (cublasLtCreate(&dc->cublas_lt) != CUBLAS_STATUS_SUCCESS) {
      dc->cublas_lt = nullptr;
      return PLX_ERR_CUDA;
    }
  }
  const int D = H * d;
  const long long M = (long long)B * N;
  const size_t t = round_up((size_t)M * D * 2, 256);
  void* proj[4] = {ws, ws + t, ws + 2 * t, ws + 3 * t};
  void* head[4] = {ws + 4 * t, ws + 5 * t, ws + 6 * t, ws + 7 * t};
  void* attn = ws + 8 * t;
  char* p8 = ws + 9 * t;
  void* x8 = p8;
  void* a8 = p8 + round_up((size_t)M * D, 256);
  char* w8 = p8 + 2 * round_up((size_t)M * D, 256);
  const size_t wsz = round_up((size_t)D * D, 256);
  unsigned* amax = reinterpret_cast<unsigned*>(w8 + 5 * wsz);  // 7 words: x, W_Q..W_R, W_O, attention
  float* scale = reinterpret_cast<float*>(amax + 8);           // 7 scales
  void* lt_ws = w8 + 5 * wsz + 256;
  const void* W[5] = {WQ, WK, WV, WR, WO};
  if (cudaMemsetAsync(amax, 0, 8 * sizeof(unsigned), st) != cudaSuccess) return PLX_ERR_CUDA;
  cudaError_t e = launch_amax(&x, 1, (size_t)M * D, amax, st);
  if (e == cudaSuccess) e = launch_amax(W, 5, (size_t)D * D, amax + 1, st);
  if (e == cudaSuccess) e = launch_quant(x, (size_t)M * D, amax, x8, scale, st);
  if (e == cudaSuccess) e = launch_quant_t(W, 5, D, D, amax + 1, w8, wsz, scale + 1, st);
  if (e != cudaSuccess) return cuda_rc(e);
  for (int i = 0; i < 4; ++i)
    if (fp8_gemm(dc->cublas_lt, w8 + i * wsz, x8, proj[i], D, D, M, scale + 1 + i, scale, lt_ws, kLtWorkspace,
                 st) != 0)
      return PLX_ERR_CUDA;
  const float eps = 1e-6f, base = 10000.f;
  if (launch_qkr_norm_rope(proj[0], head[0], B, N, H, d, eps, base, st) != cudaSuccess ||
      launch_qkr_norm_rope(proj[1], head[1], B, N, H, d, eps, base, st) != cudaSuccess ||
      launch_swap_axes(proj[2], head[2], B, N, H, d, st) != cudaSuccess ||
      launch_qkr_norm_rope(proj[3], head[3], B, N, H, d, eps, base, st) != cudaSuccess)
    return PLX_ERR_CUDA;
  PrefillArgs a{head[0], head[1], head[2], head[3], attn, B, H, N, d, 1, dc->status};
  if ((e = launch_prefill_tc(a, st, dc->num_sms)) != cudaSuccess) return cuda_rc(e);
  if (launch_swap_axes(attn, proj[0], B, H, N, d, st) != cudaSuccess) return PLX_ERR_CUDA;
  const void* merged = proj[0];
  if ((e = launch_amax(&merged, 1, (size_t)M * D, amax + 6, st)) != cudaSuccess ||
      (e = launch_quant(proj[0], (size_t)M * D, amax + 6, a8, scale + 6, st)) != cudaSuccess)
    return cuda_rc(e);
  if (fp8_gemm(dc->cublas_lt, w8 + 4 * wsz, a8, y, D, D, M, scale + 5, scale + 6, lt_ws, kLtWorkspace, st) != 0)
    return PLX_ERR_CUDA;
  return PLX_OK;
}

int plx_get_device_status(void* stream) {
  DeviceCache* dc = nullptr;
  int rc = current_device(&dc);
  if (rc != PLX_OK) return rc;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PLX_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, dc->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return PLX_ERR_CUDA;
  if (word != 0) {
    int zero = 0;
    if (cudaMemcpy(dc->status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return PLX_ERR_CUDA;
  }
  if (word & kStatusTimeout) {
    // A decode whose waits ran out may have left arrival counters of
    // unfinished (b, KV head) pairs above zero: clear them for the next call.
    std::lock_guard<std::mutex> lk(g_mu);
    if (dc->counters && cudaMemset(dc->counters, 0, dc->counters_bytes) != cudaSuccess) return PLX_ERR_CUDA;
  }
  if (word & kStatusBadSeqlen) return PLX_ERR_BAD_SEQLEN;
  if (word & kStatusTimeout) return PLX_ERR_TIMEOUT;
  return PLX_OK;
}

}  // extern "C"
