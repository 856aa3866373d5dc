// Top-K routing of one token by one warp (shared by the decode plan and
// the routing kernels).
#pragma once

#include "common.cuh"

namespace moeq {

constexpr int kNoExpert = 0x7fffffff;

// Order-preserving 32-bit key of a logit for the selection: a larger value
// has a larger key, -0 and +0 share one key, and every NaN maps to 0
// (below -inf).
__device__ __forceinline__ uint32_t route_key(float v) {
  if (v != v) return 0u;
  const uint32_t b = v == 0.0f ? 0u : __float_as_uint(v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Register path (E <= 32 * NJ): lane l holds the scaled logits of experts
// l, l + 32, ...  Each of the K passes takes the warp's largest key with
// one max-reduction and the lowest expert index holding it with one
// min-reduction; only the lane that owned the winner rescans its values.
template <int NJ>
__device__ __forceinline__ void route_token_regs(const float* __restrict__ lg, int E, int K,
                                                 int renorm, float scale, int32_t* idx, float* w) {
  const int lane = threadIdx.x & 31;
  float v[NJ];
  uint32_t key[NJ];
  uint32_t avail = 0;  // bit j: expert lane + 32 j exists and is not taken
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int e = lane + 32 * j;
    v[j] = e < E ? scale * lg[e] : 0.0f;
    key[j] = route_key(v[j]);
    if (e < E) avail |= 1u << j;
  }
  uint32_t lk = 0;
  int li = kNoExpert;
  float lv = 0.0f;
#pragma unroll
  for (int j = 0; j < NJ; ++j)
    if (((avail >> j) & 1u) && (li == kNoExpert || key[j] > lk)) {
      lk = key[j];
      li = lane + 32 * j;
      lv = v[j];
    }
  float mx = 0.0f, chosen_sum = 0.0f, my_p = 0.0f;
  int my_i = 0;
  for (int k = 0; k < K; ++k) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, lk);
    const uint32_t win = __reduce_min_sync(
        0xffffffffu, (li != kNoExpert && lk == m) ? (uint32_t)li : 0xffffffffu);
    const int wl = (int)(win & 31u);
    const float bv = __shfl_sync(0xffffffffu, lv, wl);
    if (k == 0) mx = bv;
    if (wl == lane && win != 0xffffffffu) {
      avail &= ~(1u << (win >> 5));
      lk = 0;
      li = kNoExpert;
#pragma unroll
      for (int j = 0; j < NJ; ++j)
        if (((avail >> j) & 1u) && (li == kNoExpert || key[j] > lk)) {
          lk = key[j];
          li = lane + 32 * j;
          lv = v[j];
        }
    }
    const float p = expf(bv - mx);
    if (lane == k) {
      my_p = p;
      my_i = (int)win;
    }
    chosen_sum += p;
  }
  // softmax normaliser over all experts (only without renormalisation)
  float z = 0.0f;
  if (!renorm) {
#pragma unroll
    for (int j = 0; j < NJ; ++j)
      if (lane + 32 * j < E) z += expf(v[j] - mx);
    z = warp_sum(z);
  }
  const float denom = renorm ? chosen_sum : z;
  if (lane < K) {
    idx[lane] = my_i;
    w[lane] = my_p / denom;
  }
  __syncwarp();
}

// Loop path for large E: logits in (shared) memory, `taken` a per-warp
// bitmap of E bits in shared memory.
__device__ __forceinline__ void route_token_loop(const float* lg, int E, int K, int renorm,
                                                 float scale, int32_t* idx, float* w,
                                                 uint32_t* taken) {
  const int lane = threadIdx.x & 31;
  const int words = (E + 31) >> 5;
  for (int i = lane; i < words; i += 32) taken[i] = 0u;
  __syncwarp();
  float mx = -INFINITY, chosen_sum = 0.0f, my_p = 0.0f;
  int my_i = 0;
  for (int k = 0; k < K; ++k) {
    float bv = -INFINITY;
    int bi = kNoExpert;
    uint32_t bk = 0;
    for (int e = lane; e < E; e += 32) {
      if (taken[e >> 5] & (1u << (e & 31))) continue;
      const float v = scale * lg[e];
      const uint32_t ke = route_key(v);
      if (bi == kNoExpert || ke > bk) {
        bk = ke;
        bv = v;
        bi = e;
      }
    }
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    const uint32_t win = __reduce_min_sync(
        0xffffffffu, (bi != kNoExpert && bk == m) ? (uint32_t)bi : 0xffffffffu);
    bv = __shfl_sync(0xffffffffu, bv, (int)(win & 31u));
    bi = win == 0xffffffffu ? kNoExpert : (int)win;
    if (k == 0) mx = bv;
    if (lane == 0 && bi != kNoExpert) taken[bi >> 5] |= 1u << (bi & 31);
    __syncwarp();
    const float p = expf(bv - mx);
    if (lane == k) {
      my_p = p;
      my_i = bi;
    }
    chosen_sum += p;
  }
  float z = 0.0f;
  for (int e = lane; e < E; e += 32) z += expf(scale * lg[e] - mx);
  z = warp_sum(z);
  const float denom = renorm ? chosen_sum : z;
  if (lane < K) {
    idx[lane] = my_i;
    w[lane] = my_p / denom;
  }
  __syncwarp();
}

// Candidates of one part of a token's logits: the K largest scaled logits
// of experts [base, base + count) in selection order (same rule as the full
// selection), written by lanes 0..K-1 to cidx/cval; lane 0 also writes the
// part's largest value and sum of exp(v - that maximum) over the part.
template <int NJ>
__device__ __forceinline__ void route_part_regs(const float* __restrict__ lg, int base, int count,
                                                int K, float scale, int32_t* cidx, float* cval,
                                                float* pmax, float* psum) {
  const int lane = threadIdx.x & 31;
  float v[NJ];
  uint32_t key[NJ];
  uint32_t avail = 0;
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int e = lane + 32 * j;
    v[j] = e < count ? scale * lg[base + e] : 0.0f;
    key[j] = route_key(v[j]);
    if (e < count) avail |= 1u << j;
  }
  uint32_t lk = 0;
  int li = kNoExpert;
  float lv = 0.0f;
#pragma unroll
  for (int j = 0; j < NJ; ++j)
    if (((avail >> j) & 1u) && (li == kNoExpert || key[j] > lk)) {
      lk = key[j];
      li = base + lane + 32 * j;
      lv = v[j];
    }
  float mx = 0.0f;
  for (int k = 0; k < K; ++k) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, lk);
    const uint32_t win = __reduce_min_sync(
        0xffffffffu, (li != kNoExpert && lk == m) ? (uint32_t)li : 0xffffffffu);
    const int wl = (int)((win - base) & 31u);
    const float bv = __shfl_sync(0xffffffffu, lv, wl);
    if (k == 0) mx = bv;
    if (win != 0xffffffffu && wl == lane) {
      avail &= ~(1u << ((win - base) >> 5));
      lk = 0;
      li = kNoExpert;
#pragma unroll
      for (int j = 0; j < NJ; ++j)
        if (((avail >> j) & 1u) && (li == kNoExpert || key[j] > lk)) {
          lk = key[j];
          li = base + lane + 32 * j;
          lv = v[j];
        }
    }
    if (lane == k) {
      cidx[k] = win == 0xffffffffu ? kNoExpert : (int)win;
      cval[k] = bv;
    }
  }
  float z = 0.0f;
#pragma unroll
  for (int j = 0; j < NJ; ++j)
    if (lane + 32 * j < count) z += expf(v[j] - mx);
  z = warp_sum(z);
  if (lane == 0) {
    *pmax = mx;
    *psum = z;
  }
}

// Final selection of one token from the C <= 128 candidates of its parts
// (one warp): the same rule over the candidates, then the weights; the
// softmax normaliser combines the parts' sums of exp relative to each
// part's maximum.
__device__ __forceinline__ void route_merge_parts(const int32_t* cidx, const float* cval, int C,
                                                  int K, int renorm, const float* pmax,
                                                  const float* psum, int parts, int32_t* idx,
                                                  float* w) {
  const int lane = threadIdx.x & 31;
  float v[4];
  uint32_t key[4];
  int ix[4];
  uint32_t avail = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c = lane + 32 * j;
    const bool ok = c < C && cidx[c] != kNoExpert;
    v[j] = ok ? cval[c] : 0.0f;
    ix[j] = ok ? cidx[c] : kNoExpert;
    key[j] = route_key(v[j]);
    if (ok) avail |= 1u << j;
  }
  auto best = [&](uint32_t& bk, int& bi, float& bv) {
    bk = 0;
    bi = kNoExpert;
    bv = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (((avail >> j) & 1u) &&
          (bi == kNoExpert || key[j] > bk || (key[j] == bk && ix[j] < bi))) {
        bk = key[j];
        bi = ix[j];
        bv = v[j];
      }
  };
  uint32_t lk;
  int li;
  float lv;
  best(lk, li, lv);
  float mx = 0.0f, chosen_sum = 0.0f, my_p = 0.0f;
  int my_i = 0;
  for (int k = 0; k < K; ++k) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, lk);
    const uint32_t win = __reduce_min_sync(
        0xffffffffu, (li != kNoExpert && lk == m) ? (uint32_t)li : 0xffffffffu);
    // the lane holding the winner (candidate indices are distinct experts)
    const uint32_t own = __ballot_sync(0xffffffffu, li != kNoExpert && (uint32_t)li == win);
    const int wl = own ? __ffs(own) - 1 : 0;
    const float bv = __shfl_sync(0xffffffffu, lv, wl);
    if (k == 0) mx = bv;
    if (own && wl == lane) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if ((uint32_t)ix[j] == win) avail &= ~(1u << j);
      best(lk, li, lv);
    }
    const float p = expf(bv - mx);
    if (lane == k) {
      my_p = p;
      my_i = win == 0xffffffffu ? 0 : (int)win;
    }
    chosen_sum += p;
  }
  float z = 0.0f;
  if (!renorm && lane == 0)
    for (int q = 0; q < parts; ++q)
      if (psum[q] > 0.0f) z += expf(pmax[q] - mx) * psum[q];
  z = __shfl_sync(0xffffffffu, z, 0);
  const float denom = renorm ? chosen_sum : z;
  if (lane < K) {
    idx[lane] = my_i;
    w[lane] = my_p / denom;
  }
  __syncwarp();
}

// Copies the E logits of one token into the warp's shared-memory row with
// independent (unrolled, 16-byte where aligned) loads.
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

// One warp routes one token: the K largest of p = softmax(scale * logits)
// (ties to the lower index; NaN logits rank below -inf), listed by p
// descending; w = p_k (/ sum of the
// chosen p when renorm).  lg: the token's E logits (global memory);
// row (E floats) and taken ((E+31)/32 words): the warp's shared scratch,
// used only when E > 1024.
__device__ __forceinline__ void route_token_warp(const float* lg, int E, int K, int renorm,
                                                 float scale, int32_t* idx, float* w, float* row,
                                                 uint32_t* taken) {
  if (E <= 32) route_token_regs<1>(lg, E, K, renorm, scale, idx, w);
  else if (E <= 64) route_token_regs<2>(lg, E, K, renorm, scale, idx, w);
  else if (E <= 128) route_token_regs<4>(lg, E, K, renorm, scale, idx, w);
  else if (E <= 256) route_token_regs<8>(lg, E, K, renorm, scale, idx, w);
  else if (E <= 512) route_token_regs<16>(lg, E, K, renorm, scale, idx, w);
  else if (E <= 1024) route_token_regs<32>(lg, E, K, renorm, scale, idx, w);
  else {
    stage_logits_warp(lg, row, E);
    route_token_loop(row, E, K, renorm, scale, idx, w, taken);
  }
}

// Part `part` of `parts` (one warp each) of a token's routing: candidates of
// experts [part * chunk, ...) with chunk = ceil(E / parts) <= 1024.
__device__ __forceinline__ void route_part(const float* lg, int E, int K, float scale, int part,
                                           int parts, int32_t* cidx, float* cval, float* pmax,
                                           float* psum) {
  const int chunk = (E + parts - 1) / parts;
  const int base = part * chunk;
  const int count = max(0, min(chunk, E - base));
  if (chunk <= 32) route_part_regs<1>(lg, base, count, K, scale, cidx, cval, pmax, psum);
  else if (chunk <= 64) route_part_regs<2>(lg, base, count, K, scale, cidx, cval, pmax, psum);
  else if (chunk <= 128) route_part_regs<4>(lg, base, count, K, scale, cidx, cval, pmax, psum);
  else if (chunk <= 256) route_part_regs<8>(lg, base, count, K, scale, cidx, cval, pmax, psum);
  else if (chunk <= 512) route_part_regs<16>(lg, base, count, K, scale, cidx, cval, pmax, psum);
  else route_part_regs<32>(lg, base, count, K, scale, cidx, cval, pmax, psum);
}

}  // namespace moeq
