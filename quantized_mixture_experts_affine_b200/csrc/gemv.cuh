// Split-K quantised GEMV engine for the decode path (HBM-bound).
//
// Work decomposition.  A row of a packed matrix is cut into 16-byte chunks
// (VPC = 128/BITS codes each).  A warp owns a "slice" of 32 consecutive
// chunks (lane = chunk) and streams R rows of that slice: one coalesced
// 512-byte load per row.  The warp keeps its slice of the input vector in
// registers for all R rows, accumulates one partial sum per row in each lane,
// and reduces the R partials across lanes with a transposing butterfly (about
// one shuffle per row).  The S slices of a row are handled by S warps of the
// same CTA and summed in fixed slice order, so results do not depend on
// scheduling.
//
// Arithmetic per chunk (the group form of the fma(q, scale*x, bias*x)
// factoring of flash-moe's matvec_4bit_fma):
//   contribution = scale_g * (xs_b * sum_c q_c X_c) + bias_g * sum_c xs_b X_c
// where sum_c q_c X_c is an exact integer dot product (dp4a) of the codes with
// a fixed-point copy X of the input vector (NL byte limbs per value,
// power-of-two block scale xs_b per 32 values), converted to fp32 once per
// block.  NL = 2 keeps 15 significant bits of each value relative to its
// block's largest magnitude (every bf16 value within 2^7 of it exactly);
// NL = 3 keeps 23 bits (every bf16 value within 2^15 of it exactly).
#pragma once

#include "common.cuh"

namespace moeq {

// Slice of one input vector held by a lane, in fixed-point limbs.
template <int BITS, int NL>
struct SliceVec {
  static constexpr int VPC = Chunk<BITS>::VPC;
  static constexpr int NC = Chunk<BITS>::NC;
  static constexpr int NB = (BITS == 2) ? 2 : 1;  // 32-value blocks per chunk
  uint32_t limb[NL][NC];
  float xs[NB];    // block scale 2^-k
  float xsum[NB];  // sum of the represented values in this chunk's part of the block
};

// A lane's slice to and from shared memory, word-major ([word][lane]) so
// that a warp's accesses are conflict-free.  At most 64 words per lane.
template <int BITS, int NL>
__device__ __forceinline__ void slice_store(uint32_t* slot, const SliceVec<BITS, NL>& sv,
                                            int lane) {
  constexpr int NC = SliceVec<BITS, NL>::NC, NB = SliceVec<BITS, NL>::NB;
  static_assert(NL * NC + 2 * NB <= 64, "slice exceeds its shared-memory slot");
#pragma unroll
  for (int l = 0; l < NL; ++l)
#pragma unroll
    for (int r = 0; r < NC; ++r) slot[(l * NC + r) * 32 + lane] = sv.limb[l][r];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    slot[(NL * NC + b) * 32 + lane] = __float_as_uint(sv.xs[b]);
    slot[(NL * NC + NB + b) * 32 + lane] = __float_as_uint(sv.xsum[b]);
  }
}

template <int BITS, int NL>
__device__ __forceinline__ void slice_load(const uint32_t* slot, SliceVec<BITS, NL>& sv,
                                           int lane) {
  constexpr int NC = SliceVec<BITS, NL>::NC, NB = SliceVec<BITS, NL>::NB;
#pragma unroll
  for (int l = 0; l < NL; ++l)
#pragma unroll
    for (int r = 0; r < NC; ++r) sv.limb[l][r] = slot[(l * NC + r) * 32 + lane];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    sv.xs[b] = __uint_as_float(slot[(NL * NC + b) * 32 + lane]);
    sv.xsum[b] = __uint_as_float(slot[(NL * NC + NB + b) * 32 + lane]);
  }
}

// Value c of the source vector row, as float.
struct SrcBF16 {
  __device__ __forceinline__ static void load(const void* row, int c0, float* v, int n) {
    const uint16_t* p = reinterpret_cast<const uint16_t*>(row) + c0;
    // n is a multiple of 8 and c0 a multiple of 8: 16-byte loads
#pragma unroll
    for (int i = 0; i < n; i += 8) {
      const uint4 u = *reinterpret_cast<const uint4*>(p + i);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[i + 2 * j] = __uint_as_float(w[j] << 16);
        v[i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
      }
    }
  }
};
struct SrcF32 {
  __device__ __forceinline__ static void load(const void* row, int c0, float* v, int n) {
    const float* p = reinterpret_cast<const float*>(row) + c0;
#pragma unroll
    for (int i = 0; i < n; i += 4) {
      const float4 u = *reinterpret_cast<const float4*>(p + i);
      v[i] = u.x;
      v[i + 1] = u.y;
      v[i + 2] = u.z;
      v[i + 3] = u.w;
    }
  }
};

// Build the lane's slice (chunk `ch`) of a vector.  All 32 lanes must call
// (8-bit chunks pair up lanes for a 32-value block).  Inactive lanes pass
// active = false and get zeros.
template <int BITS, int NL, class SRC>
__device__ __forceinline__ void build_slice(const void* row, int ch, bool active,
                                            SliceVec<BITS, NL>& sv) {
  constexpr int VPC = Chunk<BITS>::VPC;
  constexpr int NC = Chunk<BITS>::NC;
  constexpr int NB = SliceVec<BITS, NL>::NB;
  constexpr int PV = VPC / NB;  // values per part (16 or 32)
  float v[VPC];
  if (active) {
    SRC::load(row, ch * VPC, v, VPC);
  } else {
#pragma unroll
    for (int i = 0; i < VPC; ++i) v[i] = 0.0f;
  }
  int X[VPC];
#pragma unroll
  for (int pb = 0; pb < NB; ++pb) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < PV; ++i) m = fmaxf(m, fabsf(v[pb * PV + i]));
    if (BITS == 8) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    // m < 2^e with e = biased exponent - 126 (normal m); scale so |X| < 2^(8NL-1)
    const int e = (int)((__float_as_uint(m) >> 23) & 0xFFu) - 126;
    int k = (m > 0.0f) ? 8 * NL - 1 - e : 0;
    k = max(-120, min(k, 120));
    const float up = __uint_as_float((uint32_t)(127 + k) << 23);  // 2^k
    const int lim = (1 << (8 * NL - 1)) - 1;
    float tot = 0.0f;
#pragma unroll
    for (int i = 0; i < PV; ++i) {
      int x = __float2int_rn(v[pb * PV + i] * up);
      x = max(-lim, min(x, lim));
      X[pb * PV + i] = x;
      tot += (float)x;
    }
    const float down = __uint_as_float((uint32_t)(127 - k) << 23);  // 2^-k
    sv.xs[pb] = down;
    sv.xsum[pb] = tot * down;
  }
#pragma unroll
  for (int l = 0; l < NL; ++l)
#pragma unroll
    for (int r = 0; r < NC; ++r) {
      uint32_t w = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b)
        w |= (((uint32_t)X[Chunk<BITS>::value_of(r, b)] >> (8 * l)) & 0xFFu) << (8 * b);
      sv.limb[l][r] = w;
    }
}

// Code registers [lo, hi) that belong to block part pb of a chunk.
template <int BITS>
struct PartRegs {
  static constexpr int NC = Chunk<BITS>::NC;
  static constexpr int lo(int pb) { return BITS == 2 ? pb * (NC / 2) : 0; }
  static constexpr int hi(int pb) { return BITS == 2 ? (pb + 1) * (NC / 2) : NC; }
};

// Integer dot of code registers [LO, HI) with limbs; returns exact integer
// sum as float.
template <int BITS, int NL, int LO, int HI>
__device__ __forceinline__ float part_dot(const uint32_t (&c)[Chunk<BITS>::NC],
                                          const SliceVec<BITS, NL>& sv) {
  int a[NL];
#pragma unroll
  for (int l = 0; l < NL; ++l) a[l] = 0;
#pragma unroll
  for (int r = LO; r < HI; ++r)
#pragma unroll
    for (int l = 0; l < NL; ++l)
      a[l] = (l == NL - 1) ? dp4a_us(c[r], sv.limb[l][r], a[l]) : dp4a_uu(c[r], sv.limb[l][r], a[l]);
  if (NL == 2) return (float)(a[1] * 256 + a[0]);
  float f = (float)a[NL - 1];
#pragma unroll
  for (int l = NL - 2; l >= 0; --l) f = fmaf(f, 256.0f, (float)a[l]);
  return f;
}

// Contribution of one chunk (codes c, groups' scale/bias) to a row's dot
// product with one vector slice.
template <int BITS, int NL>
__device__ __forceinline__ float chunk_contrib(const uint32_t (&c)[Chunk<BITS>::NC],
                                               const SliceVec<BITS, NL>& sv, const float (&s)[2],
                                               const float (&b)[2]) {
  constexpr int NB = SliceVec<BITS, NL>::NB;
  float acc = 0.0f;
  if (NB == 1) {
    const float d = part_dot<BITS, NL, 0, Chunk<BITS>::NC>(c, sv);
    acc = fmaf(s[0], d * sv.xs[0], b[0] * sv.xsum[0]);
  } else {
    const float d0 = part_dot<BITS, NL, PartRegs<BITS>::lo(0), PartRegs<BITS>::hi(0)>(c, sv);
    const float d1 = part_dot<BITS, NL, PartRegs<BITS>::lo(1), PartRegs<BITS>::hi(1)>(c, sv);
    acc = fmaf(s[0], d0 * sv.xs[0], b[0] * sv.xsum[0]);
    acc = fmaf(s[1], d1 * sv.xs[1], fmaf(b[1], sv.xsum[1], acc));
  }
  return acc;
}

__device__ __forceinline__ uint4 gq_lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds32_gv(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 lds64_gv(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint16_t lds_u16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

// Transposing butterfly: every lane holds v[0..R); afterwards lane l holds
// sum over all lanes of v[l % R] (returned).  R in {8, 16, 32}.
template <int R>
__device__ __forceinline__ float transpose_reduce(float (&v)[R]) {
  const int lane = threadIdx.x & 31;
  // plain halvings while more lanes than rows
#pragma unroll
  for (int o = 16; o >= R; o >>= 1)
#pragma unroll
    for (int i = 0; i < R; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
  // reduce-scatter over the remaining lane bits
#pragma unroll
  for (int half = R / 2; half >= 1; half >>= 1) {
    const bool upper = (lane & half) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float keep = upper ? v[i + half] : v[i];
      const float send = upper ? v[i] : v[i + half];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
    }
  }
  return v[0];
}

}  // namespace moeq
