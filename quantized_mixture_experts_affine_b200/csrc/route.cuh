// Top-K routing of one token by one warp (shared by the decode plan and
// the routing kernels).
#pragma once

#include "common.cuh"

namespace moeq {

// One warp routes one token: the K largest of p = softmax(scale * logits)
// (ties to the lower index), listed by p descending; w = p_k (/ sum of the
// chosen p when renorm).  `taken` is a per-warp bitmap of E bits in shared
// memory.
__device__ __forceinline__ void route_token_warp(const float* lg, int E, int K, int renorm, float scale,
                                 int32_t* idx, float* w, uint32_t* taken) {
  const int lane = threadIdx.x & 31;
  const int words = (E + 31) >> 5;
  for (int i = lane; i < words; i += 32) taken[i] = 0u;
  __syncwarp();
  float psel[kMaxK];
  float mx = -INFINITY;
  float chosen_sum = 0.0f;
  for (int k = 0; k < K; ++k) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int e = lane; e < E; e += 32) {
      if (taken[e >> 5] & (1u << (e & 31))) continue;
      const float v = scale * lg[e];
      // the first untaken expert is always a candidate (so a choice exists
      // even when every remaining scaled logit is -inf or NaN)
      if (v > bv || (v == bv && e < bi) || bi == 0x7fffffff) {
        bv = v;
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (oi != 0x7fffffff && (ov > bv || (ov == bv && oi < bi) || bi == 0x7fffffff)) {
        bv = ov;
        bi = oi;
      }
    }
    if (k == 0) mx = bv;
    if (lane == 0) {
      taken[bi >> 5] |= 1u << (bi & 31);
      idx[k] = bi;
    }
    __syncwarp();
    const float p = expf(bv - mx);
    if (lane == 0 && k < kMaxK) psel[k] = p;
    chosen_sum += p;
  }
  // softmax normaliser over all experts
  float z = 0.0f;
  for (int e = lane; e < E; e += 32) z += expf(scale * lg[e] - mx);
  z = warp_sum(z);
  if (lane == 0) {
    const float denom = renorm ? chosen_sum : z;
    for (int k = 0; k < K; ++k) w[k] = psel[k] / denom;
  }
  __syncwarp();
}

// Copies the E logits of one token into the warp's shared-memory row with
// independent (unrolled, 16-byte where aligned) loads, so the K selection
// passes of route_token_warp read shared memory instead of issuing one
// dependent global load per pass and lane.
__device__ __forceinline__ void stage_logits_warp(const float* __restrict__ lg, float* row, int E) {
  const int lane = threadIdx.x & 31;
  if ((((uintptr_t)lg | (uintptr_t)row) & 15) == 0 && (E & 3) == 0) {
    const float4* g4 = reinterpret_cast<const float4*>(lg);
    float4* r4 = reinterpret_cast<float4*>(row);
    const int E4 = E >> 2;
    int i = lane;
    for (; i + 96 < E4; i += 128) {
      const float4 a = g4[i], b = g4[i + 32], c = g4[i + 64], d = g4[i + 96];
      r4[i] = a;
      r4[i + 32] = b;
      r4[i + 64] = c;
      r4[i + 96] = d;
    }
    for (; i < E4; i += 32) r4[i] = g4[i];
  } else {
    for (int e = lane; e < E; e += 32) row[e] = lg[e];
  }
  __syncwarp();
}

}  // namespace moeq
