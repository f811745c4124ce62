// Tensor-core (tcgen05) attention path: not built yet; every shape takes the CUDA-core path.
#include "ckv_internal.h"

namespace ckv {

bool attention_tc_supported(const LayerParams&) { return false; }
int attention_tc_keys_per_split() { return 128; }
cudaError_t launch_attention_tc(const LayerParams&, int, const int32_t*, int, const float*,
                                const int32_t*, const int32_t*, int, const AttnWs&, uint32_t*,
                                cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace ckv
