// bf16 Parallax prefill on tcgen05 tensor cores (TMA-staged tiles, TMEM
// accumulators).  Not built yet: bf16 prefill runs on the SIMT kernel.
#include "plx_internal.cuh"

namespace plx {

bool prefill_tc_supported(int d) {
  (void)d;
  return false;
}

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t st, int num_sms) {
  (void)a;
  (void)st;
  (void)num_sms;
  return cudaErrorNotSupported;
}

}  // namespace plx
