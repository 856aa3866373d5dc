// Prefill path (many tokens): sort by expert, tcgen05 gather-QMM, combine.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moeq.h"

namespace moeq {

size_t prefill_workspace_bytes(const moeq_layer* L, int M);

moeq_status prefill_forward(const moeq_layer* L, const uint16_t* x, int M, const int32_t* idx_in,
                            const float* w_in, const float* residual, float* y, int32_t* idx_out,
                            float* w_out, void* ws, size_t ws_bytes, int* status,
                            cudaStream_t st);

}  // namespace moeq
