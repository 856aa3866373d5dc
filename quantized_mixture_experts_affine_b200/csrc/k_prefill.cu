// Prefill path (many tokens): fp16 copy of the tokens, router GEMM, top-K,
// stable counting sort of the (token, slot) pairs by expert, gate/up
// gather-QMM with the SwiGLU epilogue, down gather-QMM into pair order,
// weighted combine.  Every output row is computed from its own token only,
// with the same kernels and the same K order for any M, so results do not
// depend on how the tokens are split into calls.
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <string.h>

#include "common.cuh"
#include "gqmm.cuh"
#include "kernels.h"
#include "prefill.h"
#include "route.cuh"

namespace moeq {

namespace {

constexpr int kSortChunk = 512;  // pairs per sort block

// ------------------------------------------------------------------ tokens to fp16
__global__ void __launch_bounds__(256) k_to_f16(const uint16_t* __restrict__ x, int64_t n8,
                                                __half* __restrict__ y, int* status) {
  bool bad = false;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 u = reinterpret_cast<const uint4*>(x)[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = __uint_as_float(w[j] << 16), b = __uint_as_float(w[j] & 0xFFFF0000u);
      bad |= !(fabsf(a) <= 65504.0f) || !(fabsf(b) <= 65504.0f);
      __half2 h = __floats2half2_rn(a, b);
      o[j] = *reinterpret_cast<uint32_t*>(&h);
    }
    reinterpret_cast<uint4*>(y)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (bad) set_status(status, MOEQ_ERR_RANGE);
}

// Rows of the fp16 tokens in sorted pair order: out[i] = x16[sorted[i] / K]
// (the gate/up operand as one contiguous matrix, fetched by tensor-map tiles).
__global__ void __launch_bounds__(256) k_gather_rows(const uint4* __restrict__ x16,
                                                     const int32_t* __restrict__ sorted, int K,
                                                     int64_t n, int row_chunks,
                                                     uint4* __restrict__ out) {
  // one warp per two rows: every lane's loads of both rows in flight, then
  // streaming (evict-first) stores; the rows are read once, by the gather-QMM
  constexpr int U = 8;
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 2; r < n;
       r += 2 * warps) {
    const bool two = r + 1 < n;
    const uint4* src0 = x16 + (int64_t)(sorted[r] / K) * row_chunks;
    const uint4* src1 = x16 + (int64_t)(sorted[two ? r + 1 : r] / K) * row_chunks;
    uint4* dst0 = out + r * row_chunks;
    uint4* dst1 = out + (r + 1) * row_chunks;
    for (int c0 = 0; c0 < row_chunks; c0 += 32 * U) {
      uint4 v[U], w2[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < row_chunks) {
          v[u] = src0[c];
          w2[u] = src1[c];
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < row_chunks) {
          __stcs(dst0 + c, v[u]);
          if (two) __stcs(dst1 + c, w2[u]);
        }
      }
    }
  }
}

// y[t] = sum_k w[t][k] d[t*K + k] (+ sigma[t] d[M*K + t]) (+ residual[t]), k in
// order, from fp16 down rows in pair order; eight columns per thread.
__global__ void __launch_bounds__(256) k_combine_h(const uint4* __restrict__ d,
                                                   const float* __restrict__ w,
                                                   const float* __restrict__ sigma,
                                                   int has_shared,
                                                   const float* __restrict__ residual,
                                                   float* __restrict__ y, int M, int K, int H) {
  const int H8 = H >> 3;
  const int64_t total = (int64_t)M * H8;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / H8);
    const int c8 = (int)(i - (int64_t)t * H8);
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
    auto add = [&](float s, const uint4 v) {
      const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(h[j]);
        acc[2 * j] = fmaf(s, f.x, acc[2 * j]);
        acc[2 * j + 1] = fmaf(s, f.y, acc[2 * j + 1]);
      }
    };
    for (int k = 0; k < K; ++k) add(w[(int64_t)t * K + k], d[((int64_t)t * K + k) * H8 + c8]);
    if (has_shared) add(sigma[t], d[((int64_t)M * K + t) * H8 + c8]);
    if (residual) {
      const float4* r = reinterpret_cast<const float4*>(residual + (int64_t)t * H) + 2 * c8;
      const float4 r0 = r[0], r1 = r[1];
      acc[0] += r0.x; acc[1] += r0.y; acc[2] += r0.z; acc[3] += r0.w;
      acc[4] += r1.x; acc[5] += r1.y; acc[6] += r1.z; acc[7] += r1.w;
    }
    float4* o = reinterpret_cast<float4*>(y + (int64_t)t * H) + 2 * c8;
    o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

// k_combine_h followed by the RMS norm of each row, in one pass over the
// fp16 down rows: one CTA per row keeps its NC8 chunks of eight columns per
// thread in registers while the row's sum of squares is reduced (fixed
// order), then writes y and y_norm[t][j] = bf16(y[t][j] / sqrt(mean(y[t]^2)
// + eps) * gamma[j]) ("flash-moe-inference", per-layer pipeline: combine +
// norm; rms_norm_pass1/2).  H <= 2048 * NC8.
template <int NC8>
__global__ void __launch_bounds__(256) k_combine_norm(const uint4* __restrict__ d,
                                                      const float* __restrict__ w,
                                                      const float* __restrict__ sigma,
                                                      int has_shared,
                                                      const float* __restrict__ residual,
                                                      float* __restrict__ y, int M, int K, int H,
                                                      const uint16_t* __restrict__ gamma,
                                                      float eps, uint16_t* __restrict__ y_norm) {
  __shared__ float red[8];
  const int H8 = H >> 3;
  for (int t = blockIdx.x; t < M; t += gridDim.x) {
    float acc[NC8][8];
    float ss = 0.0f;
#pragma unroll
    for (int c = 0; c < NC8; ++c) {
      const int c8 = threadIdx.x + 256 * c;
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[c][j] = 0.0f;
      if (c8 < H8) {
        auto add = [&](float s, const uint4 v) {
          const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = __half22float2(h[j]);
            acc[c][2 * j] = fmaf(s, f.x, acc[c][2 * j]);
            acc[c][2 * j + 1] = fmaf(s, f.y, acc[c][2 * j + 1]);
          }
        };
        for (int k = 0; k < K; ++k) add(w[(int64_t)t * K + k], d[((int64_t)t * K + k) * H8 + c8]);
        if (has_shared) add(sigma[t], d[((int64_t)M * K + t) * H8 + c8]);
        if (residual) {
          const float4* r = reinterpret_cast<const float4*>(residual + (int64_t)t * H) + 2 * c8;
          const float4 r0 = r[0], r1 = r[1];
          acc[c][0] += r0.x; acc[c][1] += r0.y; acc[c][2] += r0.z; acc[c][3] += r0.w;
          acc[c][4] += r1.x; acc[c][5] += r1.y; acc[c][6] += r1.z; acc[c][7] += r1.w;
        }
        float4* o = reinterpret_cast<float4*>(y + (int64_t)t * H) + 2 * c8;
        o[0] = make_float4(acc[c][0], acc[c][1], acc[c][2], acc[c][3]);
        o[1] = make_float4(acc[c][4], acc[c][5], acc[c][6], acc[c][7]);
#pragma unroll
        for (int j = 0; j < 8; ++j) ss = fmaf(acc[c][j], acc[c][j], ss);
      }
    }
    const float inv = 1.0f / sqrtf(row_sum_256(ss, red) / (float)H + eps);
#pragma unroll
    for (int c = 0; c < NC8; ++c) {
      const int c8 = threadIdx.x + 256 * c;
      if (c8 < H8) {
        const uint4 gw = reinterpret_cast<const uint4*>(gamma)[c8];
        const uint32_t gg[4] = {gw.x, gw.y, gw.z, gw.w};
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float lo = acc[c][2 * j] * inv * __uint_as_float(gg[j] << 16);
          const float hi = acc[c][2 * j + 1] * inv * __uint_as_float(gg[j] & 0xFFFF0000u);
          out[j] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
                   ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
        }
        reinterpret_cast<uint4*>(y_norm + (int64_t)t * H)[c8] =
            make_uint4(out[0], out[1], out[2], out[3]);
      }
    }
  }
}

// ------------------------------------------------------------------ routing (strided logits)
__global__ void __launch_bounds__(256) k_route_prefill(const float* __restrict__ logits, int64_t ld,
                                                       int M, int E, int K, int renorm,
                                                       float scale, int32_t* __restrict__ idx,
                                                       float* __restrict__ w, int sg_col,
                                                       float* __restrict__ sigma) {
  extern __shared__ __align__(16) uint8_t rsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int words = (E + 31) >> 5;
  const int wbytes = ((words * 4 + 15) & ~15) + E * 4;
  uint32_t* taken = reinterpret_cast<uint32_t*>(rsm + warp * wbytes);
  float* row = reinterpret_cast<float*>(rsm + warp * wbytes + ((words * 4 + 15) & ~15));
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= M) return;
  route_token_warp(logits + (int64_t)t * ld, E, K, renorm, scale, idx + (int64_t)t * K,
                   w + (int64_t)t * K, row, taken);
  if (sigma && lane == 0) sigma[t] = 1.0f / (1.0f + expf(-logits[(int64_t)t * ld + sg_col]));
}

__global__ void __launch_bounds__(256) k_copy_routing(const int32_t* __restrict__ idx_in,
                                                      const float* __restrict__ w_in, int64_t n,
                                                      int32_t* __restrict__ idx,
                                                      float* __restrict__ w) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    idx[i] = idx_in[i];
    w[i] = w_in[i];
  }
}

__global__ void __launch_bounds__(256) k_sigmoid_col(const float* __restrict__ logits, int64_t ld,
                                                     int col, int M, float* __restrict__ sigma) {
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < M; t += gridDim.x * blockDim.x)
    sigma[t] = 1.0f / (1.0f + expf(-logits[(int64_t)t * ld + col]));
}

// ------------------------------------------------------------------ stable counting sort
__device__ __forceinline__ int checked_expert(const int32_t* idx, int64_t p, int E, int* status) {
  int e = idx[p];
  if (e < 0 || e >= E) {
    set_status(status, MOEQ_ERR_INVALID_ARG);
    e = 0;
  }
  return e;
}

// Per-block expert histogram of kSortChunk pairs.
__global__ void __launch_bounds__(256) k_hist(const int32_t* __restrict__ idx, int64_t n, int E,
                                              int32_t* __restrict__ blockhist, int* status) {
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t p0 = (int64_t)blockIdx.x * kSortChunk;
  const int64_t p1 = min(n, p0 + kSortChunk);
  for (int64_t p = p0 + threadIdx.x; p < p1; p += blockDim.x)
    atomicAdd(&hist[checked_expert(idx, p, E, status)], 1);
  __syncthreads();
  // expert-major [E][nb]: one expert's block counts are contiguous
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    blockhist[(int64_t)e * gridDim.x + blockIdx.x] = hist[e];
}

struct OffsetsArgs {
  const int32_t* blockhist;
  int32_t* blockoff;        // [E][nb]
  int32_t* expert_off;      // [E]
  int32_t nb, E, I, H;
  int32_t tile_rows;         // rows per m-tile (128, or 256 for CTA pairs)
  gq::Seg* segs_gu;         // [E]
  gq::Seg* segs_dn;         // [E]
  int2* tiles;              // [max tiles]
  int32_t* n_tiles;         // [1]
  moeq_qtensor gate, up, down;
};

// One CTA: per-expert block offsets and counts, expert offsets (exclusive
// scan), one gate/up and one down segment per expert and the m-tile list.
__global__ void __launch_bounds__(1024) k_offsets(const __grid_constant__ OffsetsArgs a) {
  __shared__ int32_t count_s[4096];  // pairs per expert (E <= 4096)
  __shared__ int32_t part_rows[64], part_tiles[64];
  const int E = a.E, tid = threadIdx.x;
  const int lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
  // 1. per expert (one warp at a time): exclusive scan of its block counts
  // (the counts of 8 x 32 blocks are loaded before any is scanned, so the
  // warp waits for one memory round trip per 256 blocks, not per 32)
  for (int e = wid; e < E; e += nw) {
    const int32_t* hrow = a.blockhist + (int64_t)e * a.nb;
    int32_t* orow = a.blockoff + (int64_t)e * a.nb;
    int carry = 0;
    for (int b00 = 0; b00 < a.nb; b00 += 32 * 8) {
      int vals[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int b = b00 + 32 * j + lane;
        vals[j] = b < a.nb ? hrow[b] : 0;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int b = b00 + 32 * j + lane;
        const int v = vals[j];
        int inc = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += u;
        }
        if (b < a.nb) orow[b] = carry + inc - v;
        carry += __shfl_sync(0xffffffffu, inc, 31);
      }
    }
    if (lane == 0) count_s[e] = carry;
  }
  __syncthreads();
  // 2. exclusive scan of (rows, m-tiles) over the experts: each thread sums
  //    its experts, then shuffles within warps and over the warp totals
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = tid * per, e1 = min(E, e0 + per);
  int32_t cnt[4];  // E <= 4096 -> at most 4 experts per thread
  int rsum = 0, tsum = 0;
  for (int e = e0; e < e1; ++e) {
    const int run = count_s[e];
    cnt[e - e0] = run;
    rsum += run;
    tsum += (run + a.tile_rows - 1) / a.tile_rows;
  }
  int ir = rsum, itl = tsum;  // inclusive within the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int vr = __shfl_up_sync(0xffffffffu, ir, o);
    const int vt = __shfl_up_sync(0xffffffffu, itl, o);
    if (lane >= o) {
      ir += vr;
      itl += vt;
    }
  }
  if (lane == 31) {
    part_rows[wid] = ir;
    part_tiles[wid] = itl;
  }
  __syncthreads();
  if (wid == 0) {
    int wr = lane < nw ? part_rows[lane] : 0, wt = lane < nw ? part_tiles[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int vr = __shfl_up_sync(0xffffffffu, wr, o);
      const int vt = __shfl_up_sync(0xffffffffu, wt, o);
      if (lane >= o) {
        wr += vr;
        wt += vt;
      }
    }
    if (lane < nw) {
      part_rows[32 + lane] = wr;  // inclusive over warps
      part_tiles[32 + lane] = wt;
    }
    if (lane == nw - 1) *a.n_tiles = wt;
  }
  __syncthreads();
  int row = ir - rsum + (wid ? part_rows[32 + wid - 1] : 0);
  int tile = itl - tsum + (wid ? part_tiles[32 + wid - 1] : 0);
  for (int e = e0; e < e1; ++e) {
    const int c = cnt[e - e0];
    a.expert_off[e] = row;
    gq::Seg g;
    memset(&g, 0, sizeof(g));
    g.w[0] = a.gate.w + (int64_t)e * a.gate.expert_stride_w;
    g.s[0] = scale_at(a.gate, (int64_t)e * a.gate.expert_stride_sb);
    g.b[0] = a.gate.biases + (int64_t)e * a.gate.expert_stride_sb;
    g.w[1] = a.up.w + (int64_t)e * a.up.expert_stride_w;
    g.s[1] = scale_at(a.up, (int64_t)e * a.up.expert_stride_sb);
    g.b[1] = a.up.biases + (int64_t)e * a.up.expert_stride_sb;
    g.n0 = a.I;
    g.n_valid = a.I;
    g.row_begin = row;
    g.rows = c;
    g.a_mode = gq::A_PAIRS;
    g.dest_pairs = 0;
    g.ex[0] = g.ex[1] = e;
    a.segs_gu[e] = g;
    gq::Seg d;
    memset(&d, 0, sizeof(d));
    d.w[0] = d.w[1] = a.down.w + (int64_t)e * a.down.expert_stride_w;
    d.s[0] = d.s[1] = scale_at(a.down, (int64_t)e * a.down.expert_stride_sb);
    d.b[0] = d.b[1] = a.down.biases + (int64_t)e * a.down.expert_stride_sb;
    d.n0 = a.H;
    d.n_valid = a.H;
    d.row_begin = row;
    d.rows = c;
    d.a_mode = gq::A_ROWS;
    d.dest_pairs = 1;
    d.ex[0] = d.ex[1] = e;
    a.segs_dn[e] = d;
    const int nt = (c + a.tile_rows - 1) / a.tile_rows;
    for (int j = 0; j < nt; ++j) a.tiles[tile + j] = make_int2(e, j * a.tile_rows);
    row += c;
    tile += nt;
  }
}

// Stable scatter: one warp per block of kSortChunk pairs, in pair order.
__global__ void __launch_bounds__(32) k_scatter(const int32_t* __restrict__ idx, int64_t n, int E,
                                                const int32_t* __restrict__ expert_off,
                                                const int32_t* __restrict__ blockoff,
                                                int32_t* __restrict__ sorted_pair, int* status) {
  extern __shared__ int32_t run[];  // next sorted position of each expert
  const int lane = threadIdx.x;
  for (int e = lane; e < E; e += 32)
    run[e] = expert_off[e] + blockoff[(int64_t)e * gridDim.x + blockIdx.x];
  __syncwarp();
  const int64_t p0 = (int64_t)blockIdx.x * kSortChunk;
  const int64_t p1 = min(n, p0 + kSortChunk);
  // the block's expert indices, loaded before the ordered pass (one memory
  // round trip instead of one per 32 pairs)
  constexpr int R = kSortChunk / 32;
  int ev[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int64_t p = p0 + 32 * r + lane;
    ev[r] = p < p1 ? checked_expert(idx, p, E, status) : -1 - lane;
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int64_t base = p0 + 32 * r;
    const int64_t p = base + lane;
    const bool on = p < p1;
    const int e = ev[r];
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (on) {
      const int rank = __popc(peers & ((1u << lane) - 1u));
      sorted_pair[(int64_t)run[e] + rank] = (int32_t)p;
    }
    __syncwarp();
    if (on && lane == __ffs(peers) - 1) run[e] += __popc(peers);
    __syncwarp();
  }
}

// ------------------------------------------------------------------ gather-QMM launch

// Launch over `units` work items: one CTA per item up to the co-resident
// count, or (PAIR) one cluster of two CTAs per item up to the co-resident
// cluster count.
template <int BITS, int EPI, bool PAIR, int GS, bool MX = false>
cudaError_t launch_gqmm_t(const gq::Args& a, int units, cudaStream_t st) {
  constexpr int smem = gq::Smem<BITS, PAIR>::ALLOC;
  auto kern = gq::k_gqmm<BITS, EPI, PAIR, GS, MX>;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.blockDim = dim3(gq::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = PAIR ? 1 : 0;
  // co-resident CTAs or clusters, and the shared-memory opt-in, per device
  static std::atomic<int> max_units[kMaxDevices];
  int dev;
  if (!current_device(dev)) return cudaErrorInvalidDevice;
  int cap = max_units[dev].load(std::memory_order_acquire);
  if (cap <= 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cap = sm_count();
    if (cap <= 0) return cudaErrorInvalidDevice;
    if (PAIR) {
      cfg.gridDim = dim3(2);
      e = cudaOccupancyMaxActiveClusters(&cap, kern, &cfg);
      if (e != cudaSuccess) return e;
      if (cap <= 0) return cudaErrorInvalidConfiguration;
    }
    max_units[dev].store(cap, std::memory_order_release);
  }
  const int n = units < cap ? units : cap;
  if (n <= 0) return cudaSuccess;
  cfg.gridDim = dim3(PAIR ? 2 * n : n);
  return cudaLaunchKernelEx(&cfg, kern, a);
}

// Group size 64 runs the kernel compiled for it; 32 and 128 the one that
// reads it from the arguments.
template <int BITS, int EPI, bool PAIR>
cudaError_t launch_gqmm_g(const gq::Args& a, int units, cudaStream_t st) {
  if (a.fmt == MOEQ_FMT_MXFP4) {
    if constexpr (BITS == 4 && EPI != gq::EPI_SPLIT)
      return launch_gqmm_t<4, EPI, PAIR, 32, true>(a, units, st);
    return cudaErrorInvalidValue;
  }
  if (a.G == 64) return launch_gqmm_t<BITS, EPI, PAIR, 64>(a, units, st);
  return launch_gqmm_t<BITS, EPI, PAIR, 0>(a, units, st);
}

template <bool PAIR>
cudaError_t launch_gqmm_p(int bits, int epi, const gq::Args& a, int units, cudaStream_t st) {
  if (epi == gq::EPI_SPLIT) {
    if (bits == 8) return launch_gqmm_g<8, gq::EPI_SPLIT, PAIR>(a, units, st);
    if (bits == 4) return launch_gqmm_g<4, gq::EPI_SPLIT, PAIR>(a, units, st);
    return launch_gqmm_g<2, gq::EPI_SPLIT, PAIR>(a, units, st);
  }
  if (epi == gq::EPI_SWIGLU) {
    if (bits == 8) return launch_gqmm_g<8, gq::EPI_SWIGLU, PAIR>(a, units, st);
    if (bits == 4) return launch_gqmm_g<4, gq::EPI_SWIGLU, PAIR>(a, units, st);
    return launch_gqmm_g<2, gq::EPI_SWIGLU, PAIR>(a, units, st);
  }
  if (bits == 8) return launch_gqmm_g<8, gq::EPI_STORE, PAIR>(a, units, st);
  if (bits == 4) return launch_gqmm_g<4, gq::EPI_STORE, PAIR>(a, units, st);
  return launch_gqmm_g<2, gq::EPI_STORE, PAIR>(a, units, st);
}

// PAIR launches need the A operand as tensor-map tiles (a.tma_a).
cudaError_t launch_gqmm(int bits, int epi, bool pair, const gq::Args& a, int64_t units,
                        cudaStream_t st) {
  if (units <= 0) return cudaSuccess;
  const int u = units > (1 << 30) ? (1 << 30) : (int)units;
  if (pair) {
    if (!a.tma_a) return cudaErrorInvalidValue;
    return launch_gqmm_p<true>(bits, epi, a, u, st);
  }
  return launch_gqmm_p<false>(bits, epi, a, u, st);
}


gq::Seg seg_single(const moeq_qtensor& t0, const moeq_qtensor* t1, int rows, int a_mode) {
  gq::Seg s;
  memset(&s, 0, sizeof(s));
  s.w[0] = t0.w;
  s.s[0] = t0.scales;
  s.b[0] = t0.biases;
  const moeq_qtensor& u = t1 ? *t1 : t0;
  s.w[1] = u.w;
  s.s[1] = u.scales;
  s.b[1] = u.biases;
  s.n0 = t0.out_dim;
  s.n_valid = t0.out_dim + (t1 ? t1->out_dim : 0);
  s.row_begin = 0;
  s.rows = rows;
  s.a_mode = a_mode;
  s.dest_pairs = 0;
  return s;
}

// ------------------------------------------------------------------ workspace
struct Carve {
  size_t off = 0;
  size_t take(size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~(size_t)255;
    return o;
  }
};

struct PrefillWs {
  size_t x16, logits, idx, w, sigma, blockhist, blockoff, expert_off, segs_gu, segs_dn, tiles,
      n_tiles, sorted, a_sorted, h, h_sh, y, total;
  int64_t ld_logits;
  int nb;
};

bool sg_with_router(const moeq_layer* L) {
  return L->has_shared && L->sh_expert_gate.bits == L->router.bits &&
         L->sh_expert_gate.group_size == L->router.group_size;
}

PrefillWs prefill_ws(const moeq_layer* L, int M) {
  const int E = L->n_experts, K = L->top_k, H = L->hidden, I = L->inter;
  const int Is = L->has_shared ? L->sh_gate.out_dim : 0;
  const int64_t n = (int64_t)M * K;
  PrefillWs w;
  w.nb = (int)((n + kSortChunk - 1) / kSortChunk);
  // row stride a multiple of 4 floats: the epilogue stores 16-byte vectors
  w.ld_logits = (E + (L->has_shared ? 1 : 0) + 3) & ~3;
  const int64_t max_tiles = n / gq::BM + E + 1;
  Carve c;
  w.x16 = c.take((size_t)M * H * 2);
  w.logits = c.take((size_t)M * w.ld_logits * 4);
  w.idx = c.take((size_t)n * 4);
  w.w = c.take((size_t)n * 4);
  w.sigma = c.take((size_t)M * 4);
  w.blockhist = c.take((size_t)w.nb * E * 4);
  w.blockoff = c.take((size_t)w.nb * E * 4);
  w.expert_off = c.take((size_t)E * 4);
  w.segs_gu = c.take((size_t)E * sizeof(gq::Seg));
  w.segs_dn = c.take((size_t)E * sizeof(gq::Seg));
  w.tiles = c.take((size_t)max_tiles * sizeof(int2));
  w.n_tiles = c.take(16);
  w.sorted = c.take((size_t)n * 4);
  w.a_sorted = c.take((size_t)n * H * 2);
  w.h = c.take((size_t)n * I * 2);
  w.h_sh = c.take((size_t)M * Is * 2);
  w.y = c.take((size_t)(n + M) * H * 2);  // fp16 down rows, pair order then shared
  w.total = c.off;
  return w;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (null if
// the driver does not provide it).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Tensor map of an fp16 matrix [rows][K] (row stride lda elements) with a
// 128-row x 64-column box in the 128-byte swizzled layout of the A stages;
// rows past the end read as zeros.  Sets a.tma_a on success.
void set_a_tensor_map(gq::Args& a, const __half* A, int64_t rows, int K, int64_t lda) {
  a.tma_a = 0;
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn || ((uintptr_t)A & 15) || ((lda * 2) & 15) || rows <= 0 || K % gq::BK) return;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)lda * 2};
  const cuuint32_t box[2] = {(cuuint32_t)gq::BK, (cuuint32_t)gq::BM};
  const cuuint32_t es[2] = {1, 1};
  if (fn(&a.tmA, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(A), dims, strides, box, es,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
    a.tma_a = 1;
}

// Tensor map of a packed code tensor [n_mat][out_dim][in_dim*bits/32 words]
// with a box of 128 rows x one 64-wide group, written in the swizzle of the
// raw code stages.  False when the tensor does not meet the map's rules.
bool code_tensor_map(CUtensorMap* m, const moeq_qtensor& t, int n_mat) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  const int64_t row_words = (int64_t)t.in_dim * t.bits / 32;
  const int64_t row_bytes = row_words * 4;
  const int64_t mat_bytes = n_mat > 1 ? t.expert_stride_w * 4 : (int64_t)t.out_dim * row_bytes;
  if (!fn || ((uintptr_t)t.w & 15) || (row_bytes & 15) || (mat_bytes & 15) || mat_bytes <= 0 ||
      t.in_dim % gq::BK || n_mat < 1)
    return false;
  const cuuint64_t dims[3] = {(cuuint64_t)row_words, (cuuint64_t)t.out_dim, (cuuint64_t)n_mat};
  const cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)mat_bytes};
  const cuuint32_t box[3] = {(cuuint32_t)(gq::BK * t.bits / 32), 128, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  const CUtensorMapSwizzle swz = t.bits == 8   ? CU_TENSOR_MAP_SWIZZLE_64B
                                 : t.bits == 4 ? CU_TENSOR_MAP_SWIZZLE_32B
                                               : CU_TENSOR_MAP_SWIZZLE_NONE;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t*>(t.w), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Groups per scale/bias window copy of a gather-QMM launch over tensors ts
// (reduction length K, one group size G for all of them): the largest of 8,
// 4, 2 that divides K/G, keeps every matrix's scale and bias rows aligned to
// the copy size and spans at least two k-blocks (W * G / 64 >= 2).  0 when
// none does or the tensors' group sizes differ.
int sb_window(const moeq_qtensor* const* ts, int n, int K) {
  const int G = ts[0]->group_size;
  for (int i = 1; i < n; ++i)
    if (ts[i]->group_size != G || ts[i]->format != ts[0]->format) return 0;
  if (G != 32 && G != 64 && G != 128) return 0;
  const int groups = K / G;
  if (ts[0]->format == MOEQ_FMT_MXFP4) {
    // one exponent byte per group: W-byte copies (W = 8 or 4, two or more
    // k-blocks per window at G = 32) from W-aligned rows
    for (int W = 8; W >= 4; W >>= 1) {
      bool ok = groups % W == 0;
      for (int i = 0; i < n && ok; ++i)
        ok = ((uintptr_t)ts[i]->scales % W) == 0 && ts[i]->expert_stride_sb % W == 0;
      if (ok) return W;
    }
    return 0;
  }
  for (int W = 8; W >= 2; W >>= 1) {
    if (gq::win_kb_log2(W, G) < 1) continue;
    bool ok = groups % W == 0;
    for (int i = 0; i < n && ok; ++i)
      ok = ((uintptr_t)ts[i]->scales % (2 * W)) == 0 && ((uintptr_t)ts[i]->biases % (2 * W)) == 0 &&
           (ts[i]->expert_stride_sb * 2) % (2 * W) == 0;
    if (ok || (W == 2 && groups % 2 == 0)) return W;
  }
  return 0;
}

// Scale/bias window and group size of a launch over tensors ts.
bool set_window(gq::Args& a, const moeq_qtensor* const* ts, int n, int K) {
  a.sb_w = sb_window(ts, n, K);
  a.G = ts[0]->group_size;
  a.fmt = ts[0]->format;
  return a.sb_w != 0;
}

moeq_status check_prefill(const moeq_layer* L) {
  const moeq_qtensor* ts[8] = {&L->router, &L->gate, &L->up, &L->down,
                               &L->sh_gate, &L->sh_up, &L->sh_down, &L->sh_expert_gate};
  const int n = L->has_shared ? 8 : 4;
  for (int i = 0; i < n; ++i) {
    const int G = ts[i]->group_size;
    if (G != 32 && G != 64 && G != 128) return MOEQ_ERR_UNSUPPORTED;
    if (G == 32 && ts[i]->bits == 2) return MOEQ_ERR_UNSUPPORTED;
    if (stream_bits(ts[i]->bits)) return MOEQ_ERR_UNSUPPORTED;  // decode only
    if (ts[i]->format == MOEQ_FMT_AFFINE &&
        (((uintptr_t)ts[i]->scales & 3) || ((uintptr_t)ts[i]->biases & 3)))
      return MOEQ_ERR_ALIGNMENT;
    if (ts[i]->in_dim % 128) return MOEQ_ERR_UNSUPPORTED;
    if (ts[i]->expert_stride_sb % 2) return MOEQ_ERR_ALIGNMENT;
  }
  if (L->inter % 128) return MOEQ_ERR_UNSUPPORTED;
  if (L->has_shared && L->sh_gate.out_dim % 128) return MOEQ_ERR_UNSUPPORTED;
  // every launch's tensors share a group size and admit a scale/bias window
  const moeq_qtensor* gu[2] = {&L->gate, &L->up};
  const moeq_qtensor* dn[1] = {&L->down};
  const moeq_qtensor* rt[2] = {&L->router, &L->sh_expert_gate};
  if (!sb_window(gu, 2, L->hidden) || !sb_window(dn, 1, L->inter)) return MOEQ_ERR_UNSUPPORTED;
  if (!sb_window(rt, 1, L->hidden)) return MOEQ_ERR_UNSUPPORTED;
  if (L->has_shared) {
    const moeq_qtensor* sgu[2] = {&L->sh_gate, &L->sh_up};
    const moeq_qtensor* sdn[1] = {&L->sh_down};
    const moeq_qtensor* sg[1] = {&L->sh_expert_gate};
    if (!sb_window(sgu, 2, L->hidden) || !sb_window(sdn, 1, L->sh_gate.out_dim) ||
        !sb_window(sg, 1, L->hidden))
      return MOEQ_ERR_UNSUPPORTED;
    if (sg_with_router(L) && !sb_window(rt, 2, L->hidden)) return MOEQ_ERR_UNSUPPORTED;
  }
  return MOEQ_OK;
}

}  // namespace

int sm_count() {
  static std::atomic<int> sms[kMaxDevices];
  int dev;
  if (!current_device(dev)) return 0;
  int n = sms[dev].load(std::memory_order_relaxed);
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      return 0;
    sms[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

size_t prefill_workspace_bytes(const moeq_layer* L, int M) {
  if (check_prefill(L) != MOEQ_OK) return 0;
  return prefill_ws(L, M).total;
}

#define PCK(x)                                              \
  do {                                                      \
    if ((x) != cudaSuccess) return MOEQ_ERR_CUDA;           \
    count_launches(1);                                      \
  } while (0)

moeq_status prefill_forward(const moeq_layer* L, const uint16_t* x, int M, const int32_t* idx_in,
                            const float* w_in, const float* residual, float* y, int32_t* idx_out,
                            float* w_out, void* ws, size_t ws_bytes, int* status,
                            cudaStream_t st, const NormOut* norm) {
  moeq_status s = check_prefill(L);
  if (s != MOEQ_OK) return s;
  const int E = L->n_experts, K = L->top_k, H = L->hidden, I = L->inter;
  const int64_t n = (int64_t)M * K;
  const PrefillWs lay = prefill_ws(L, M);
  if (ws_bytes < lay.total) return MOEQ_ERR_WORKSPACE;
  char* base = (char*)ws;
  __half* x16 = (__half*)(base + lay.x16);
  float* logits = (float*)(base + lay.logits);
  int32_t* idx = idx_out ? idx_out : (int32_t*)(base + lay.idx);
  float* wts = w_out ? w_out : (float*)(base + lay.w);
  float* sigma = (float*)(base + lay.sigma);
  int32_t* blockhist = (int32_t*)(base + lay.blockhist);
  int32_t* blockoff = (int32_t*)(base + lay.blockoff);
  int32_t* expert_off = (int32_t*)(base + lay.expert_off);
  gq::Seg* segs_gu = (gq::Seg*)(base + lay.segs_gu);
  gq::Seg* segs_dn = (gq::Seg*)(base + lay.segs_dn);
  int2* tiles = (int2*)(base + lay.tiles);
  int32_t* n_tiles = (int32_t*)(base + lay.n_tiles);
  int32_t* sorted = (int32_t*)(base + lay.sorted);
  __half* h = (__half*)(base + lay.h);
  __half* h_sh = (__half*)(base + lay.h_sh);
  __half* yrows = (__half*)(base + lay.y);
  const int sms = sm_count();
  // CTA pairs (m-tiles of 256 rows) when the operands can be tensor-map
  // tiles and the layer routes enough rows to each expert: a 16,384-token
  // call averages at least 256 rows per expert (64 K >= E).  The choice
  // depends on the layer only, so chunked and one-shot calls use the same
  // kernels; every gather-QMM launch of the call uses the same tiling.
  const bool pair = encode_fn() != nullptr && 64 * K >= E;
  const int TR = pair ? 2 * gq::BM : gq::BM;
  const int mtiles = (M + TR - 1) / TR;

  // 1. fp16 copy of the tokens (range-checked)
  {
    const int64_t n8 = (int64_t)M * H / 8;
    int64_t grid = (n8 + 255) / 256;
    if (grid > sms * 8) grid = sms * 8;
    k_to_f16<<<(int)grid, 256, 0, st>>>(x, n8, x16, status);
    PCK(cudaGetLastError());
  }

  // 2. router logits (+ the shared-expert gate logit as one more column)
  const bool sgr = sg_with_router(L);
  auto gemm_args = [&](const gq::Seg& s0, int n_tiles_n, int Kdim, const __half* A, int64_t lda,
                       void* out, int64_t ldo) {
    gq::Args a;
    memset(&a, 0, sizeof(a));
    a.seg0 = s0;
    a.static_mtiles = mtiles;
    a.n_tiles_n = n_tiles_n;
    a.K = Kdim;
    a.A = A;
    a.lda = lda;
    a.topk = K;
    a.out = out;
    a.ldo = ldo;
    a.status = status;
    set_a_tensor_map(a, A, M, Kdim, lda);
    return a;
  };
  if (!idx_in) {
    // hi/lo split weights: fp32-accurate logits for the top-K decision
    const gq::Seg rs = seg_single(L->router, sgr ? &L->sh_expert_gate : nullptr, M, gq::A_TOKENS);
    const int nt = (rs.n_valid + 127) / 128;
    gq::Args a = gemm_args(rs, nt, H, x16, H, logits, lay.ld_logits);
    const moeq_qtensor* ts[2] = {&L->router, &L->sh_expert_gate};
    if (!set_window(a, ts, sgr ? 2 : 1, H)) return MOEQ_ERR_UNSUPPORTED;
    const int items = mtiles * nt;
    PCK(launch_gqmm(L->router.bits, gq::EPI_SPLIT, pair, a, items, st));
  }
  if (L->has_shared && (idx_in || !sgr)) {
    const gq::Seg gs = seg_single(L->sh_expert_gate, nullptr, M, gq::A_TOKENS);
    gq::Args a = gemm_args(gs, 1, H, x16, H, logits + E, lay.ld_logits);
    const moeq_qtensor* ts[1] = {&L->sh_expert_gate};
    if (!set_window(a, ts, 1, H)) return MOEQ_ERR_UNSUPPORTED;
    PCK(launch_gqmm(L->sh_expert_gate.bits, gq::EPI_SPLIT, pair, a, mtiles, st));
  }

  // 3. routing
  if (!idx_in) {
    const int warps = route_warps_per_cta(E);
    const size_t smem = (size_t)warps * ((((E + 31) / 32 * 4 + 15) & ~15) + (size_t)E * 4);
    k_route_prefill<<<(M + warps - 1) / warps, warps * 32, smem, st>>>(
        logits, lay.ld_logits, M, E, K, L->renorm, L->router_scale, idx, wts, E,
        L->has_shared ? sigma : nullptr);
    PCK(cudaGetLastError());
  } else {
    int64_t grid = (n + 255) / 256;
    if (grid > sms * 8) grid = sms * 8;
    k_copy_routing<<<(int)grid, 256, 0, st>>>(idx_in, w_in, n, idx, wts);
    PCK(cudaGetLastError());
    if (L->has_shared) {
      k_sigmoid_col<<<(M + 255) / 256, 256, 0, st>>>(logits, lay.ld_logits, E, M, sigma);
      PCK(cudaGetLastError());
    }
  }

  // 4. stable counting sort of the pairs by expert, segments and m-tiles
  const size_t hsmem = (size_t)E * 4;
  k_hist<<<lay.nb, 256, hsmem, st>>>(idx, n, E, blockhist, status);
  PCK(cudaGetLastError());
  OffsetsArgs oa;
  memset(&oa, 0, sizeof(oa));
  oa.blockhist = blockhist;
  oa.blockoff = blockoff;
  oa.expert_off = expert_off;
  oa.nb = lay.nb;
  oa.E = E;
  oa.I = I;
  oa.H = H;
  oa.tile_rows = TR;
  oa.segs_gu = segs_gu;
  oa.segs_dn = segs_dn;
  oa.tiles = tiles;
  oa.n_tiles = n_tiles;
  oa.gate = L->gate;
  oa.up = L->up;
  oa.down = L->down;
  k_offsets<<<1, 1024, 0, st>>>(oa);
  PCK(cudaGetLastError());
  k_scatter<<<lay.nb, 32, hsmem, st>>>(idx, n, E, expert_off, blockoff, sorted, status);
  PCK(cudaGetLastError());

  const int64_t max_mtiles = n / TR + E;
  // 5. gate/up + SwiGLU for the routed experts (the profiled kernel), then the shared expert
  {
    gq::Args a;
    memset(&a, 0, sizeof(a));
    a.segs = segs_gu;
    a.tiles = tiles;
    a.n_tiles = n_tiles;
    a.n_tiles_n = I / 128;
    a.K = H;
    a.A = x16;
    a.lda = H;
    // the token rows in sorted pair order as one matrix: tensor-map tiles
    __half* a_sorted = (__half*)(base + lay.a_sorted);
    set_a_tensor_map(a, a_sorted, n, H, H);
    if (a.tma_a) {
      int64_t grid = (n + 7) / 8;
      if (grid > (int64_t)sms * 16) grid = (int64_t)sms * 16;
      k_gather_rows<<<(int)grid, 256, 0, st>>>((const uint4*)x16, sorted, K, n, H / 8,
                                               (uint4*)a_sorted);
      PCK(cudaGetLastError());
    }
    a.sorted_pair = sorted;
    a.topk = K;
    a.out = h;
    a.ldo = I;
    a.status = status;
    a.tma_b = code_tensor_map(&a.tmB[0], L->gate, E) && code_tensor_map(&a.tmB[1], L->up, E);
    const moeq_qtensor* ts[2] = {&L->gate, &L->up};
    if (!set_window(a, ts, 2, H)) return MOEQ_ERR_UNSUPPORTED;
    const int64_t items = max_mtiles * a.n_tiles_n;
    if (profile_mark(true, st) != cudaSuccess) return MOEQ_ERR_CUDA;
    PCK(launch_gqmm(L->gate.bits, gq::EPI_SWIGLU, pair, a, items, st));
    if (profile_mark(false, st) != cudaSuccess) return MOEQ_ERR_CUDA;
  }
  if (L->has_shared) {
    const int Is = L->sh_gate.out_dim;
    gq::Seg gs = seg_single(L->sh_gate, &L->sh_up, M, gq::A_TOKENS);
    gs.n0 = Is;
    gq::Args a = gemm_args(gs, Is / 128, H, x16, H, h_sh, Is);
    a.tma_b = code_tensor_map(&a.tmB[0], L->sh_gate, 1) && code_tensor_map(&a.tmB[1], L->sh_up, 1);
    const moeq_qtensor* ts[2] = {&L->sh_gate, &L->sh_up};
    if (!set_window(a, ts, 2, H)) return MOEQ_ERR_UNSUPPORTED;
    const int items = mtiles * (Is / 128);
    PCK(launch_gqmm(L->sh_gate.bits, gq::EPI_SWIGLU, pair, a, items, st));
  }
  // 6. down projections into pair order (shared rows after the M*K pair rows)
  {
    gq::Args a;
    memset(&a, 0, sizeof(a));
    a.segs = segs_dn;
    a.tiles = tiles;
    a.n_tiles = n_tiles;
    a.n_tiles_n = (H + gq::BN - 1) / gq::BN;
    a.K = I;
    a.A = h;
    a.lda = I;
    set_a_tensor_map(a, h, n, I, I);
    a.sorted_pair = sorted;
    a.topk = K;
    a.out = yrows;
    a.ldo = H;
    a.out_f16 = 1;
    a.status = status;
    a.tma_b = code_tensor_map(&a.tmB[0], L->down, E);
    const moeq_qtensor* ts[1] = {&L->down};
    if (!set_window(a, ts, 1, I)) return MOEQ_ERR_UNSUPPORTED;
    const int64_t items = max_mtiles * a.n_tiles_n;
    PCK(launch_gqmm(L->down.bits, gq::EPI_STORE, pair, a, items, st));
  }
  if (L->has_shared) {
    const int Is = L->sh_gate.out_dim;
    const gq::Seg ds = seg_single(L->sh_down, nullptr, M, gq::A_ROWS);
    gq::Args a = gemm_args(ds, (H + gq::BN - 1) / gq::BN, Is, h_sh, Is,
                           yrows + n * (int64_t)H, H);
    a.out_f16 = 1;
    a.tma_b = code_tensor_map(&a.tmB[0], L->sh_down, 1);
    const moeq_qtensor* ts[1] = {&L->sh_down};
    if (!set_window(a, ts, 1, Is)) return MOEQ_ERR_UNSUPPORTED;
    const int items = mtiles * ((H + gq::BN - 1) / gq::BN);
    PCK(launch_gqmm(L->sh_down.bits, gq::EPI_STORE, pair, a, items, st));
  }
  // 7. combine in k order (+ sigmoid-gated shared expert, + residual)
  {
    const int64_t total = (int64_t)M * (H / 8);
    int64_t grid = (total + 255) / 256;
    if (grid > (int64_t)sms * 16) grid = (int64_t)sms * 16;
    const int H8 = H / 8;
    if (norm && H8 <= 256 * 4) {
      // combine and norm in one pass: one CTA per row
      const int g = M < sms * 8 ? M : sms * 8;
      if (H8 <= 256)
        k_combine_norm<1><<<g, 256, 0, st>>>((const uint4*)yrows, wts, sigma, L->has_shared,
                                             residual, y, M, K, H, norm->gamma, norm->eps,
                                             norm->y_norm);
      else if (H8 <= 512)
        k_combine_norm<2><<<g, 256, 0, st>>>((const uint4*)yrows, wts, sigma, L->has_shared,
                                             residual, y, M, K, H, norm->gamma, norm->eps,
                                             norm->y_norm);
      else
        k_combine_norm<4><<<g, 256, 0, st>>>((const uint4*)yrows, wts, sigma, L->has_shared,
                                             residual, y, M, K, H, norm->gamma, norm->eps,
                                             norm->y_norm);
      PCK(cudaGetLastError());
    } else {
      k_combine_h<<<(int)grid, 256, 0, st>>>((const uint4*)yrows, wts, sigma, L->has_shared,
                                             residual, y, M, K, H);
      PCK(cudaGetLastError());
      if (norm) PCK(launch_rmsnorm_rows(y, M, H, *norm, st));
    }
  }
  return MOEQ_OK;
}

}  // namespace moeq
