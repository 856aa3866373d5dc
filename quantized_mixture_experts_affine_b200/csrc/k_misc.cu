// Unpack / dequantise one matrix (bit-exact reference form of the format);
// RMS norm of output rows.
#include "common.cuh"
#include "kernels.h"
#include "prefill.h"

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

// 3-, 5- and 6-bit codes (a row is one little-endian bit stream): one thread
// per 32-value chunk of 12, 20 or 24 bytes, spread to bytes as the decode
// GEMV does.
template <int BITS>
__global__ void __launch_bounds__(256) k_dequant_stream(const uint32_t* __restrict__ w,
                                                        const uint16_t* __restrict__ sc,
                                                        const uint16_t* __restrict__ bi,
                                                        int out_dim, int in_dim, int G,
                                                        uint8_t* __restrict__ q_out,
                                                        float* __restrict__ w_out) {
  constexpr int CW = Chunk<BITS>::BYTES / 4;  // words per 32-value chunk
  const int64_t cpr = in_dim / 32;
  const int64_t total = (int64_t)out_dim * cpr;
  const int gpr = in_dim / G;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / cpr;
    const int64_t c0 = (i % cpr) * 32;
    uint32_t ws[CW];
#pragma unroll
    for (int k = 0; k < CW; ++k) ws[k] = w[i * CW + k];
    uint32_t c[8];
    Chunk<BITS>::split_stream(ws, c);
    const int g = (int)(c0 / G);  // G >= 32: one group per chunk
    const float s = bf16_bits_to_float(sc[r * gpr + g]);
    const float b = bf16_bits_to_float(bi[r * gpr + g]);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const uint32_t q = (c[j / 4] >> (8 * (j % 4))) & 255u;
      if (q_out) q_out[r * in_dim + c0 + j] = (uint8_t)q;
      if (w_out) w_out[r * in_dim + c0 + j] = __fmaf_rn((float)q, s, b);
    }
  }
}

// MX FP4: w = e2m1(q) * 2^(e - 127), exact in fp32 (q' * 2^(e - 128) with
// q' = 2 e2m1(q) + 12, minus 12 * 2^(e - 128)).
__global__ void __launch_bounds__(256) k_dequant_mx(const uint32_t* __restrict__ w,
                                                    const uint8_t* __restrict__ ex, int out_dim,
                                                    int in_dim, uint8_t* __restrict__ q_out,
                                                    float* __restrict__ w_out) {
  const int64_t wpr = (int64_t)in_dim / 8;
  const int64_t total = (int64_t)out_dim * wpr;
  const int gpr = in_dim / 32;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / wpr;
    const int64_t c0 = (i % wpr) * 8;
    const uint32_t word = w[i];
    const float sc = mx_scale(ex[r * gpr + (int)(c0 / 32)]);
    const uint32_t lo = mx_q8(word & 0x0F0F0F0Fu), hi = mx_q8((word >> 4) & 0x0F0F0F0Fu);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t q = (word >> (4 * j)) & 15u;
      const int qq = (int)(((j & 1) ? hi : lo) >> (8 * (j >> 1)) & 255u);  // q' = 2 e2m1 + 12
      if (q_out) q_out[r * in_dim + c0 + j] = (uint8_t)q;
      const float mag = (float)abs(qq - 12) * 0.5f * sc;  // |e2m1| * 2^(e-127), exact
      if (w_out) w_out[r * in_dim + c0 + j] = (q & 8u) ? -mag : mag;  // code 8 is -0
    }
  }
}

cudaError_t launch_dequant(const moeq_qtensor& t, int expert, uint8_t* q_out, float* w_out,
                           cudaStream_t st) {
  if (t.format == MOEQ_FMT_MXFP4) {
    const uint32_t* w = t.w + (int64_t)expert * t.expert_stride_w;
    const uint8_t* e = reinterpret_cast<const uint8_t*>(t.scales) + (int64_t)expert * t.expert_stride_sb;
    const int64_t total = (int64_t)t.out_dim * t.in_dim / 8;
    int64_t grid = (total + 255) / 256;
    if (grid > 148 * 32) grid = 148 * 32;
    if (grid == 0) return cudaSuccess;
    k_dequant_mx<<<(int)grid, 256, 0, st>>>(w, e, t.out_dim, t.in_dim, q_out, w_out);
    return cudaGetLastError();
  }
  const uint32_t* w = t.w + (int64_t)expert * t.expert_stride_w;
  const uint16_t* s = t.scales + (int64_t)expert * t.expert_stride_sb;
  const uint16_t* b = t.biases + (int64_t)expert * t.expert_stride_sb;
  const int64_t total = (int64_t)t.out_dim * t.in_dim * t.bits / 32;
  int64_t grid = (total + 255) / 256;
  if (grid > 148 * 32) grid = 148 * 32;
  if (grid == 0) return cudaSuccess;
  if (stream_bits(t.bits)) {
    const int64_t chunks = (int64_t)t.out_dim * t.in_dim / 32;
    int64_t g2 = (chunks + 255) / 256;
    if (g2 > 148 * 32) g2 = 148 * 32;
    if (t.bits == 3)
      k_dequant_stream<3><<<(int)g2, 256, 0, st>>>(w, s, b, t.out_dim, t.in_dim, t.group_size, q_out, w_out);
    else if (t.bits == 5)
      k_dequant_stream<5><<<(int)g2, 256, 0, st>>>(w, s, b, t.out_dim, t.in_dim, t.group_size, q_out, w_out);
    else
      k_dequant_stream<6><<<(int)g2, 256, 0, st>>>(w, s, b, t.out_dim, t.in_dim, t.group_size, q_out, w_out);
    return cudaGetLastError();
  }
  switch (t.bits) {
    case 2: k_dequant<2><<<(int)grid, 256, 0, st>>>(w, s, b, t.out_dim, t.in_dim, t.group_size, q_out, w_out); break;
    case 4: k_dequant<4><<<(int)grid, 256, 0, st>>>(w, s, b, t.out_dim, t.in_dim, t.group_size, q_out, w_out); break;
    default: k_dequant<8><<<(int)grid, 256, 0, st>>>(w, s, b, t.out_dim, t.in_dim, t.group_size, q_out, w_out); break;
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------------ RMS norm of output rows
// y_norm[t][j] = bf16(y[t][j] / sqrt((1/H) sum_i y[t][i]^2 + eps) * g[j]),
// one CTA of 256 threads per row ("flash-moe-inference", rms_norm_pass1/2:
// the sum of squares, then the scaling).  H a multiple of 8.
__global__ void __launch_bounds__(256) k_rmsnorm_rows(const float* __restrict__ y, int M, int H,
                                                      const uint16_t* __restrict__ gamma,
                                                      float eps, uint16_t* __restrict__ y_norm) {
  __shared__ float red[8];
  const int H8 = H >> 3;
  for (int t = blockIdx.x; t < M; t += gridDim.x) {
    const float4* r = reinterpret_cast<const float4*>(y + (int64_t)t * H);
    float ss = 0.0f;
    for (int i = threadIdx.x; i < 2 * H8; i += 256) {
      const float4 v = r[i];
      ss = fmaf(v.x, v.x, ss);
      ss = fmaf(v.y, v.y, ss);
      ss = fmaf(v.z, v.z, ss);
      ss = fmaf(v.w, v.w, ss);
    }
    const float inv = 1.0f / sqrtf(row_sum_256(ss, red) / (float)H + eps);
    uint4* o = reinterpret_cast<uint4*>(y_norm + (int64_t)t * H);
    const uint4* g = reinterpret_cast<const uint4*>(gamma);
    for (int i = threadIdx.x; i < H8; i += 256) {
      const float4 a = r[2 * i], b = r[2 * i + 1];
      const uint4 gw = g[i];
      const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      const uint32_t gg[4] = {gw.x, gw.y, gw.z, gw.w};
      uint32_t out[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float lo = v[2 * j] * inv * __uint_as_float(gg[j] << 16);
        const float hi = v[2 * j + 1] * inv * __uint_as_float(gg[j] & 0xFFFF0000u);
        out[j] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
                 ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
      }
      o[i] = make_uint4(out[0], out[1], out[2], out[3]);
    }
  }
}

cudaError_t launch_rmsnorm_rows(const float* y, int M, int H, const NormOut& n, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  const int grid = M < 148 * 8 ? M : 148 * 8;
  k_rmsnorm_rows<<<grid, 256, 0, st>>>(y, M, H, n.gamma, n.eps, n.y_norm);
  return cudaGetLastError();
}

}  // namespace moeq
