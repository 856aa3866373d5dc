// Unpack / dequantise one matrix (bit-exact reference form of the format).
#include "common.cuh"
#include "kernels.h"

namespace moeq {

// One thread per packed word: 32/BITS codes; w = fmaf(q, scale, bias), one
// correctly rounded fp32 operation ("flash-moe-inference": nibble*scale + bias).
template <int BITS>
__global__ void __launch_bounds__(256) k_dequant(const uint32_t* __restrict__ w,
                                                 const uint16_t* __restrict__ sc,
                                                 const uint16_t* __restrict__ bi, int out_dim,
                                                 int in_dim, int G, uint8_t* __restrict__ q_out,
                                                 float* __restrict__ w_out) {
  constexpr int PER = 32 / BITS;
  const int64_t wpr = (int64_t)in_dim / PER;
  const int64_t total = (int64_t)out_dim * wpr;
  const int gpr = in_dim / G;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / wpr;
    const int64_t c0 = (i % wpr) * PER;
    const uint32_t word = w[i];
    const int g = (int)(c0 / G);
    const float s = bf16_bits_to_float(sc[r * gpr + g]);
    const float b = bf16_bits_to_float(bi[r * gpr + g]);
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const uint32_t q = (word >> (BITS * j)) & ((1u << BITS) - 1u);
      if (q_out) q_out[r * in_dim + c0 + j] = (uint8_t)q;
      if (w_out) w_out[r * in_dim + c0 + j] = __fmaf_rn((float)q, s, b);
    }
  }
}

cudaError_t launch_dequant(const moeq_qtensor& t, int expert, uint8_t* q_out, float* w_out,
                           cudaStream_t st) {
  const uint32_t* w = t.w + (int64_t)expert * t.expert_stride_w;
  const uint16_t* s = t.scales + (int64_t)expert * t.expert_stride_sb;
  const uint16_t* b = t.biases + (int64_t)expert * t.expert_stride_sb;
  const int64_t total = (int64_t)t.out_dim * t.in_dim * t.bits / 32;
  int64_t grid = (total + 255) / 256;
  if (grid > 148 * 32) grid = 148 * 32;
  if (grid == 0) return cudaSuccess;
  switch (t.bits) {
    case 2: k_dequant<2><<<(int)grid, 256, 0, st>>>(w, s, b, t.out_dim, t.in_dim, t.group_size, q_out, w_out); break;
    case 4: k_dequant<4><<<(int)grid, 256, 0, st>>>(w, s, b, t.out_dim, t.in_dim, t.group_size, q_out, w_out); break;
    default: k_dequant<8><<<(int)grid, 256, 0, st>>>(w, s, b, t.out_dim, t.in_dim, t.group_size, q_out, w_out); break;
  }
  return cudaGetLastError();
}

}  // namespace moeq
