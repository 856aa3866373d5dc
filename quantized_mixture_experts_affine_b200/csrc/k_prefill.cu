// Prefill path: placeholder until the tensor-core gather-QMM lands.
#include "prefill.h"

namespace moeq {

size_t prefill_workspace_bytes(const moeq_layer*, int) { return 0; }

moeq_status prefill_forward(const moeq_layer*, const uint16_t*, int, const int32_t*, const float*,
                            const float*, float*, int32_t*, float*, void*, size_t, int*,
                            cudaStream_t) {
  return MOEQ_ERR_UNSUPPORTED;
}

}  // namespace moeq
