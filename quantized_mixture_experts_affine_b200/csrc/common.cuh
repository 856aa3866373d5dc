// Device helpers shared by the layer kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <stdint.h>

#include "moeq.h"

namespace moeq {

// ------------------------------------------------------------------ limits
constexpr int kMaxDecodeM = 64;      // tokens per decode call
constexpr int kMaxK = 32;            // top-K
constexpr int kMaxE = 4096;          // experts
constexpr int kXBlock = 32;          // values per fixed-point block of an input vector
constexpr int kWaitSpins = 1 << 22;  // bounded device-side waits

// ------------------------------------------------------------------ host: devices
constexpr int kMaxDevices = 64;  // per-device host caches (launch attributes, SM counts)

// The calling thread's current device; false when the runtime cannot say or
// the index is beyond the per-device host caches (callers then fail the call).
inline bool current_device(int& dev) {
  dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices;
}

// SM count of the current device (cached per device); 0 when the device or
// the attribute cannot be read.
int sm_count();

// ------------------------------------------------------------------ status word
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// ------------------------------------------------------------------ conversions
__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) {
  return __uint_as_float(((uint32_t)h) << 16);
}

// ------------------------------------------------------------------ integer dot products
// d = c + sum_i a.byte[i] * b.byte[i]; a unsigned codes, b signed or unsigned limb.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp4a_uu(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// ------------------------------------------------------------------ warp reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum of one value per thread over a CTA of 256 threads, in a fixed order
// (warps, then the eight warp totals in order); red: 8 floats of shared memory.
__device__ __forceinline__ float row_sum_256(float v, float* red) {
  v = warp_sum(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) t += red[i];
  __syncthreads();
  return t;
}


// ------------------------------------------------------------------ MX FP4 codes
// An E2M1 code q (bit 3 sign, bits 2..1 exponent, bit 0 mantissa) times two
// is an integer in [-12, 12]; shifted by 12 it is an unsigned code
// q' = 2 e2m1(q) + 12 in [0, 24], so a group with E8M0 byte e is the affine
// group w = q' * s + b with s = 2^(e - 128) and b = -12 s, exactly.  The
// paths run MX FP4 through their affine arithmetic on q'.

// q' of the four codes held one per byte in c (each 0..15): two 8-entry
// byte tables (the positive and the negative values) indexed by the low 3
// bits, chosen per byte by the sign bit.
__device__ __forceinline__ uint32_t mx_q8(uint32_t c) {
  const uint32_t m = c & 0x07070707u;
  const uint32_t sel = __byte_perm(m | (m >> 4), 0u, 0x3320u) & 0xFFFFu;  // nibbles m0..m3
  const uint32_t pos = __byte_perm(0x0F0E0D0Cu, 0x18141210u, sel);  // 12,13,14,15,16,18,20,24
  const uint32_t neg = __byte_perm(0x090A0B0Cu, 0x00040608u, sel);  // 12,11,10,9,8,6,4,0
  const uint32_t smask = ((c >> 3) & 0x01010101u) * 0xFFu;
  return (pos & ~smask) | (neg & smask);
}

// Scale array of t advanced by `entries` groups (MX FP4: one byte each,
// affine: one bf16 each).
__host__ __device__ __forceinline__ const uint16_t* scale_at(const moeq_qtensor& t,
                                                             int64_t entries) {
  return t.format == MOEQ_FMT_MXFP4
             ? reinterpret_cast<const uint16_t*>(reinterpret_cast<const uint8_t*>(t.scales) +
                                                 entries)
             : t.scales + entries;
}

// 2^(e - 127) in fp32 (e = 0: 2^-127, subnormal; e = 255: NaN).
__device__ __forceinline__ float mx_scale(uint32_t e) {
  return e == 255u ? __uint_as_float(0x7FC00000u)
                   : e == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(e << 23);
}

// ------------------------------------------------------------------ code registers
// A 16-byte chunk of a packed row holds VPC = 128/BITS codes in 4 words.
// It is split into NC = VPC/4 "code registers", each holding 4 codes in its
// 4 bytes, ready for dp4a:
//   BITS 8: reg k      = word k                      (values 4k .. 4k+3)
//   BITS 4: reg 2k     = word k & 0x0F0F0F0F         (values 8k + 0,2,4,6)
//           reg 2k+1   = (word k >> 4) & 0x0F0F0F0F  (values 8k + 1,3,5,7)
//   BITS 2: reg 4k+i   = (word k >> 2i) & 0x03030303 (values 16k + i + 0,4,8,12)
// value_of(BITS, reg, byte) gives the position of a code within the chunk.
// BITS 3, 5, 6 (cross-word packing): a chunk is 32 values, 12, 20 or 24
// bytes of the row's bit stream, spread to one code per byte in value order
//   reg k = values 4k .. 4k+3.
__host__ __device__ constexpr bool stream_bits(int bits) {
  return bits == 3 || bits == 5 || bits == 6;
}
__host__ __device__ constexpr int chunk_values(int bits) {
  return stream_bits(bits) ? 32 : 128 / bits;
}

template <int BITS>
struct Chunk {
  static constexpr int VPC = chunk_values(BITS);  // values per chunk
  static constexpr int BYTES = VPC * BITS / 8;     // 16; 12, 20 or 24 (3, 5, 6 bits)
  static constexpr int NC = VPC / 4;      // code registers per chunk
  static constexpr int NBLK = VPC >= kXBlock ? VPC / kXBlock : 1;  // x blocks touched
  __host__ __device__ static constexpr int value_of(int reg, int byte) {
    return BITS == 8 || stream_bits(BITS) ? reg * 4 + byte
         : BITS == 4 ? (reg >> 1) * 8 + (reg & 1) + 2 * byte
                     : (reg >> 2) * 16 + (reg & 3) + 4 * byte;
  }
  // Four consecutive b-bit values (the low 4b bits of v) one per byte.
  __device__ __forceinline__ static uint32_t spread4(uint32_t v) {
    if (BITS == 3)
      return (v & 0x7u) | ((v & 0x38u) << 5) | ((v & 0x1C0u) << 10) | ((v & 0xE00u) << 15);
    if (BITS == 5)
      return (v & 0x1Fu) | ((v & 0x3E0u) << 3) | ((v & 0x7C00u) << 6) | ((v & 0xF8000u) << 9);
    return (v & 0x3Fu) | ((v & 0xFC0u) << 2) | ((v & 0x3F000u) << 4) | ((v & 0xFC0000u) << 6);
  }
  // The chunk of 3-, 5- or 6-bit codes in words w[0 .. BYTES/4) as NC registers.
  __device__ __forceinline__ static void split_stream(const uint32_t* w, uint32_t (&c)[NC]) {
    constexpr int GB = 4 * BITS;  // bits of four values
#pragma unroll
    for (int k = 0; k < NC; ++k) {
      const int bit = GB * k, i = bit / 32, off = bit % 32;
      const uint32_t hi = (i + 1) * 4 < BYTES ? w[i + 1] : 0u;
      c[k] = spread4(__funnelshift_r(w[i], hi, off) & ((1u << GB) - 1u));
    }
  }
  __device__ __forceinline__ static void split(const uint4& w, uint32_t (&c)[NC]) {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (BITS == 8) {
        c[k] = ws[k];
      } else if (BITS == 4) {
        c[2 * k] = ws[k] & 0x0F0F0F0Fu;
        c[2 * k + 1] = (ws[k] >> 4) & 0x0F0F0F0Fu;
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) c[4 * k + i] = (ws[k] >> (2 * i)) & 0x03030303u;
      }
    }
  }
};

}  // namespace moeq
