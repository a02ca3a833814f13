// Tensor-core (tcgen05 + TMA + TMEM) windowed softmax.  Placeholder until the
// kernel lands: reports itself unsupported so the SIMT kernel runs.
#include "vdn_internal.h"

namespace vdn {
bool softmax_tc_supported(const Dims&) { return false; }
cudaError_t launch_softmax_tc(const Dims&, const Inputs&, const Work&, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace vdn
