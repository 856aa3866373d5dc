// Prefill path (many tokens): sort by expert, tcgen05 gather-QMM, combine.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moeq.h"

namespace moeq {

size_t prefill_workspace_bytes(const moeq_layer* L, int M);

// Optional RMS norm of the output rows: y_norm[t][j] =
// bf16(y[t][j] / sqrt(mean(y[t]^2) + eps) * gamma[j]); gamma bf16 [H].
struct NormOut {
  const uint16_t* gamma;
  float eps;
  uint16_t* y_norm;
};

// y_norm for M rows of y (one CTA per row), after y is complete.
cudaError_t launch_rmsnorm_rows(const float* y, int M, int H, const NormOut& n, cudaStream_t st);

moeq_status prefill_forward(const moeq_layer* L, const uint16_t* x, int M, const int32_t* idx_in,
                            const float* w_in, const float* residual, float* y, int32_t* idx_out,
                            float* w_out, void* ws, size_t ws_bytes, int* status,
                            cudaStream_t st, const NormOut* norm = nullptr);

}  // namespace moeq
