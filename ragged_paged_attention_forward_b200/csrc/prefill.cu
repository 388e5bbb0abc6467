// Tensor-core (tcgen05/TMEM) paged prefill kernel.
#include "rpa_internal.h"

namespace rpa {

cudaError_t launch_prefill(const PrefillLaunch& p, cudaStream_t stream) {
  (void)stream;
  if (p.num_tiles <= 0) return cudaSuccess;
  set_last_error("prefill kernel not built yet");
  return cudaErrorNotSupported;
}

}  // namespace rpa
