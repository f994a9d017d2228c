// plx_decode_noalloc: the bf16 split-KV decode for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they decode: a
// serving runtime that reserves all device memory up front and hands kernels
// only the buffers it owns, or a latency-critical loop that must not risk the
// device-wide synchronisation a cudaMalloc or cudaFree can cause.
// plx_decode_ex needs scratch for its partial records and arrival counters and
// would allocate it (or needs the caller to); this entry point instead uses one
// fixed scratch array compiled into the library as a file-scope __device__
// variable, so it allocates nothing.  Every GPU that loads the library holds
// the array (8 MiB) until the process exits.
#include "plx_internal.cuh"

#include <mutex>

#include "../../include/plx.h"

namespace plx {
namespace {

constexpr size_t kScratchBytes = 8u << 20;          // the whole array
constexpr size_t kCounterBytes = 128u << 10;        // arrival counters: up to 32768 (b, h)
constexpr size_t kPartialBytes = kScratchBytes - kCounterBytes;
constexpr int kMaxDevices = 64;

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, not a device address: kernels get the address that
// cudaGetSymbolAddress returns for the current device.
__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
unsigned char* g_scratch_addr[kMaxDevices];  // per device, filled on first use

}  // namespace
}  // namespace plx

using namespace plx;

extern "C" int plx_decode_noalloc(const void* q, const void* r, const void* Kcache,
                                  const void* Vcache, const int32_t* seqlens, void* out, int B,
                                  int H, int L, int d, void* stream) {
  if (!q || !r || !Kcache || !Vcache || !seqlens || !out) return PLX_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || L < 1) return PLX_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return PLX_ERR_UNSUPPORTED;
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!a16(q) || !a16(r) || !a16(Kcache) || !a16(Vcache) || !a16(out) ||
      (reinterpret_cast<uintptr_t>(seqlens) & 3u))
    return PLX_ERR_MISALIGNED;
  if (!decode_sizes_supported(B, H, H, L)) return PLX_ERR_UNSUPPORTED;  // as plx_decode_ex
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PLX_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return PLX_ERR_CUDA;

  DecodeArgs a{};
  decode_bf16_plan(B, H, L, d, sms, &a.splits, &a.chunk);
  const size_t bh = (size_t)B * H;
  const size_t partial_bytes = a.splits > 1 ? sizeof(float) * bh * a.splits * (2 * d + 4) : 0;
  if (a.splits > 1 && (bh * sizeof(int) > kCounterBytes || partial_bytes > kPartialBytes))
    return PLX_ERR_WORKSPACE;  // these sizes need more than the fixed scratch holds

  unsigned char* base = nullptr;
  {
    // Set-up, once per device, with that device current.
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_addr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return PLX_ERR_CUDA;
      g_scratch_addr[dev] = static_cast<unsigned char*>(p);
    }
    base = g_scratch_addr[dev];
  }
  int* status = status_word_address();
  if (!status) return PLX_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
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
  a.status = status;
  if (a.splits > 1) {
    // The array keeps the previous call's contents; the counters must start at zero.
    if (cudaMemsetAsync(base, 0, bh * sizeof(int), st) != cudaSuccess) return PLX_ERR_CUDA;
    a.counters = reinterpret_cast<int*>(base);
    a.partials = reinterpret_cast<float*>(base + kCounterBytes);
  }
  return launch_decode_bf16(a, st, sms) == cudaSuccess ? PLX_OK : PLX_ERR_CUDA;
}
