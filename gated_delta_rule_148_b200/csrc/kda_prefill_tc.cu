// KDA chunkwise prefill on the sm_100a tensor cores (tcgen05 / TMEM / TMA).
#include "kda_internal.cuh"

namespace kda {

bool prefill_tc_supported(const PrefillParams &, bool) { return false; }

cudaError_t launch_prefill_tc(const PrefillParams &, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace kda
