// Decode path kernels: split-K quantised GEMV (router, gate/up + SwiGLU,
// down), top-K routing with the grouped work plan, and the weighted combine.
#include "gemv.cuh"
#include "kernels.h"
#include "route.cuh"

namespace moeq {

GemvShape gemv_shape(int slices, int R) {
  GemvShape s;
  s.R = R;
  s.rbs = slices >= 8 ? 1 : 8 / slices;
  s.warps = slices * s.rbs;
  return s;
}

// ============================================================== GEMV kernel
__device__ __forceinline__ int find_seg(const Seg* segs, int n, int unit) {
  int lo = 0, hi = n - 1;  // last seg with unit_begin <= unit
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (segs[mid].unit_begin <= unit) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int BITS, int NL, int NMAT, int R, int SRC, int EPI>
__global__ void __launch_bounds__(256) k_gemv(const __grid_constant__ GemvArgs a) {
  constexpr int VPC = Chunk<BITS>::VPC;
  constexpr int NC = Chunk<BITS>::NC;
  constexpr int NB = SliceVec<BITS, NL>::NB;
  constexpr int RB = 4;  // rows per load batch
  using SrcT = typename std::conditional<SRC == SRC_BF16, SrcBF16, SrcF32>::type;
  __shared__ float part[8][NMAT][R];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.slices;
  const int rbs = (blockDim.x >> 5) / S;
  const int slice = warp % S, rbl = warp / S;

  const Seg* segs = a.dyn_segs ? a.dyn_segs : a.segs;
  const int n_segs = a.dyn_segs ? a.dyn_count[0] : a.n_segs;
  const int total_units = a.dyn_segs ? a.dyn_count[1] : a.total_units;

  for (int unit = blockIdx.x; unit < total_units; unit += gridDim.x) {
    const Seg& sg = segs[find_seg(segs, n_segs, unit)];
    const int lu = unit - sg.unit_begin;
    const int out_dim = sg.out_dim;
    const int row0 = (lu * rbs + rbl) * R;
    const int cpr = sg.in_dim / VPC;
    const int ch = slice * 32 + lane;
    const bool lane_on = ch < cpr;
    const int64_t wpr = (int64_t)sg.in_dim * BITS / 32;
    const int gpr = sg.in_dim / sg.G;
    int gi[2];
#pragma unroll
    for (int pb = 0; pb < 2; ++pb) gi[pb] = (ch * VPC + (pb < NB ? pb : 0) * kXBlock) / sg.G;
    const uint32_t* wbase[NMAT];
    const uint16_t* sbase[NMAT];
    const uint16_t* bbase[NMAT];
#pragma unroll
    for (int m = 0; m < NMAT; ++m) {
      wbase[m] = sg.w[m];
      sbase[m] = sg.s[m];
      bbase[m] = sg.b[m];
    }

    for (int v = 0; v < sg.n_vec; ++v) {
      const void* src;
      float* dst;
      if (sg.vec_mode == 0) {
        src = (SRC == SRC_BF16)
                  ? (const void*)((const uint16_t*)sg.src_base + (int64_t)v * sg.src_stride)
                  : (const void*)((const float*)sg.src_base + (int64_t)v * sg.src_stride);
        dst = sg.dst_base + (int64_t)v * sg.dst_stride;
      } else {
        src = sg.vecs[v].src;
        dst = sg.vecs[v].dst;
      }
      SliceVec<BITS, NL> sv;
      build_slice<BITS, NL, SrcT>(src, ch, lane_on, sv);

      float acc[NMAT][R];
#pragma unroll
      for (int rr = 0; rr < R; rr += RB) {
        uint4 wv[NMAT][RB];
        float sf[NMAT][RB][2], bf[NMAT][RB][2];
#pragma unroll
        for (int i = 0; i < RB; ++i) {
          const int r = row0 + rr + i;
          const bool on = lane_on && r < out_dim;
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            if (on) {
              wv[m][i] = ldg_stream16(wbase[m] + (int64_t)r * wpr + (int64_t)ch * 4);
#pragma unroll
              for (int pb = 0; pb < NB; ++pb) {
                sf[m][i][pb] = bf16_bits_to_float(ldg_u16(sbase[m] + (int64_t)r * gpr + gi[pb]));
                bf[m][i][pb] = bf16_bits_to_float(ldg_u16(bbase[m] + (int64_t)r * gpr + gi[pb]));
              }
            } else {
              wv[m][i] = make_uint4(0, 0, 0, 0);
#pragma unroll
              for (int pb = 0; pb < NB; ++pb) sf[m][i][pb] = bf[m][i][pb] = 0.0f;
            }
            if (NB == 1) sf[m][i][1] = bf[m][i][1] = 0.0f;
          }
        }
#pragma unroll
        for (int i = 0; i < RB; ++i)
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            uint32_t c[NC];
            Chunk<BITS>::split(wv[m][i], c);
            const float s2[2] = {sf[m][i][0], sf[m][i][1]};
            const float b2[2] = {bf[m][i][0], bf[m][i][1]};
            acc[m][rr + i] = chunk_contrib<BITS, NL>(c, sv, s2, b2);
          }
      }
      float tot[NMAT];
#pragma unroll
      for (int m = 0; m < NMAT; ++m) tot[m] = transpose_reduce<R>(acc[m]);
      // lane l now holds row (l % R) of this warp's slice
      bool writer = (lane < R);
      if (S > 1) {
        if (lane < R)
#pragma unroll
          for (int m = 0; m < NMAT; ++m) part[warp][m][lane] = tot[m];
        __syncthreads();
        writer = writer && slice == 0;
        if (writer) {
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            float t = 0.0f;
            for (int sl = 0; sl < S; ++sl) t += part[rbl * S + sl][m][lane];
            tot[m] = t;
          }
        }
      }
      if (writer) {
        const int r = row0 + lane;
        if (r < out_dim) {
          float o;
          if (EPI == EPI_SWIGLU) {
            const float g = tot[0];
            o = g / (1.0f + expf(-g)) * tot[NMAT - 1];
          } else {
            o = tot[0];
          }
          dst[r] = o;
        }
      }
      if (S > 1) __syncthreads();
    }
  }
}

template <int BITS, int NL, int NMAT, int R, int SRC, int EPI>
static cudaError_t launch_one(const GemvArgs& a, int grid, int warps, cudaStream_t st) {
  k_gemv<BITS, NL, NMAT, R, SRC, EPI><<<grid, warps * 32, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gemv(int bits, int nl, int nmat, int R, int src, const GemvArgs& a, int grid,
                        cudaStream_t st) {
  const GemvShape sh = gemv_shape(a.slices, R);
  if (grid <= 0) return cudaSuccess;
  if (R != 8) return cudaErrorInvalidValue;
  // instantiated forms: router / qmv (3 limbs, bf16 tokens), gate/up + SwiGLU
  // (2 limbs, bf16 tokens), down (2 limbs, fp32 hidden rows)
  if (nmat == 2 && nl == 2 && src == SRC_BF16) {
    if (bits == 8) return launch_one<8, 2, 2, 8, SRC_BF16, EPI_SWIGLU>(a, grid, sh.warps, st);
    if (bits == 4) return launch_one<4, 2, 2, 8, SRC_BF16, EPI_SWIGLU>(a, grid, sh.warps, st);
    return launch_one<2, 2, 2, 8, SRC_BF16, EPI_SWIGLU>(a, grid, sh.warps, st);
  }
  if (nmat == 1 && nl == 3 && src == SRC_BF16) {
    if (bits == 8) return launch_one<8, 3, 1, 8, SRC_BF16, EPI_PLAIN>(a, grid, sh.warps, st);
    if (bits == 4) return launch_one<4, 3, 1, 8, SRC_BF16, EPI_PLAIN>(a, grid, sh.warps, st);
    return launch_one<2, 3, 1, 8, SRC_BF16, EPI_PLAIN>(a, grid, sh.warps, st);
  }
  if (nmat == 1 && nl == 2 && src == SRC_F32) {
    if (bits == 8) return launch_one<8, 2, 1, 8, SRC_F32, EPI_PLAIN>(a, grid, sh.warps, st);
    if (bits == 4) return launch_one<4, 2, 1, 8, SRC_F32, EPI_PLAIN>(a, grid, sh.warps, st);
    return launch_one<2, 2, 1, 8, SRC_F32, EPI_PLAIN>(a, grid, sh.warps, st);
  }
  return cudaErrorInvalidValue;
}

// ============================================================== top-K routing
__global__ void __launch_bounds__(256) k_route_topk(const float* __restrict__ logits, int M, int E,
                                                    int K, int renorm, float scale,
                                                    int32_t* __restrict__ idx,
                                                    float* __restrict__ w) {
  extern __shared__ uint32_t taken_all[];
  const int warp = threadIdx.x >> 5;
  const int words = (E + 31) >> 5;
  uint32_t* taken = taken_all + warp * words;
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= M) return;
  route_token_warp(logits + (int64_t)t * E, E, K, renorm, scale, idx + (int64_t)t * K,
                   w + (int64_t)t * K, taken);
}

cudaError_t launch_route_topk(const float* logits, int M, int E, int K, int renorm, float scale,
                              int32_t* idx, float* w, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  const int warps = 8;
  const int grid = (M + warps - 1) / warps;
  const size_t smem = (size_t)warps * ((E + 31) / 32) * 4;
  k_route_topk<<<grid, warps * 32, smem, st>>>(logits, M, E, K, renorm, scale, idx, w);
  return cudaGetLastError();
}

// ============================================================== decode plan
// One CTA (1024 threads).  Routes the M tokens (unless the routing is given),
// computes the shared-expert gate, sorts the M*K (token, slot) pairs by
// expert (stable) and writes one gate/up segment and one down segment per
// distinct expert, then the shared expert's segments.
__global__ void __launch_bounds__(1024) k_decode_plan(const __grid_constant__ DecodePlanArgs a) {
  extern __shared__ uint32_t sm[];
  const int M = a.M, K = a.K, n = M * K;
  const int tid = threadIdx.x, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int words = (a.E + 31) >> 5;
  int32_t* key = reinterpret_cast<int32_t*>(sm);      // [n] expert of pair
  int32_t* sorted = key + n;                          // [n] pairs sorted by (expert, pair)
  int32_t* head = sorted + n;                         // [n] 1 at the first pair of an expert
  int32_t* entry_of = head + n;                       // [n] entry index of sorted position
  uint32_t* taken = reinterpret_cast<uint32_t*>(entry_of + n);  // [nwarps][words]

  // 1. routing
  if (a.logits) {
    for (int t = warp; t < M; t += nwarps)
      route_token_warp(a.logits + (int64_t)t * a.E, a.E, K, a.renorm, a.router_scale,
                       a.idx_out + (int64_t)t * K, a.w_out + (int64_t)t * K,
                       taken + warp * words);
  } else {
    for (int p = tid; p < n; p += blockDim.x) {
      a.idx_out[p] = a.idx_in[p];
      a.w_out[p] = a.w_in[p];
    }
  }
  if (a.has_shared && a.sg_logit)
    for (int t = tid; t < M; t += blockDim.x) a.sigma[t] = 1.0f / (1.0f + expf(-a.sg_logit[t]));
  __syncthreads();

  // 2. stable sort of pairs by expert: rank of key (expert * n + pair)
  for (int p = tid; p < n; p += blockDim.x) {
    int e = a.idx_out[p];
    if (e < 0 || e >= a.E) {
      set_status(a.status, MOEQ_ERR_INVALID_ARG);
      e = 0;
    }
    key[p] = e;
  }
  __syncthreads();
  for (int p = tid; p < n; p += blockDim.x) {
    const int e = key[p];
    int rank = 0;
    for (int q = 0; q < n; ++q) {
      const int f = key[q];
      rank += (f < e) || (f == e && q < p);
    }
    sorted[rank] = p;
  }
  __syncthreads();
  for (int i = tid; i < n; i += blockDim.x)
    head[i] = (i == 0) || (key[sorted[i]] != key[sorted[i - 1]]);
  __syncthreads();
  // entry index = inclusive prefix count of heads - 1 (serial scan by warp 0; n <= 2048)
  if (warp == 0) {
    int run = 0;
    for (int base = 0; base < n; base += 32) {
      const int i = base + (tid & 31);
      int h = (i < n) ? head[i] : 0;
      int incl = h;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if ((tid & 31) >= o) incl += y;
      }
      if (i < n) entry_of[i] = run + incl - 1;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  __syncthreads();
  const int n_entries = n > 0 ? entry_of[n - 1] + 1 : 0;

  // 3. vector lists and segments, one per distinct expert
  for (int i = tid; i < n; i += blockDim.x) {
    const int p = sorted[i];
    const int t = p / K;
    a.vecs_gu[i].src = a.x + (int64_t)t * a.H;
    a.vecs_gu[i].dst = a.h + (int64_t)p * a.I;
    a.vecs_dn[i].src = a.h + (int64_t)p * a.I;
    a.vecs_dn[i].dst = a.d + (int64_t)p * a.H;
    if (head[i]) {
      const int u = entry_of[i];
      const int e = key[p];
      int cnt = 1;
      while (i + cnt < n && !head[i + cnt]) ++cnt;
      Seg g;
      g.w[0] = a.gate.w + (int64_t)e * a.gate.expert_stride_w;
      g.s[0] = a.gate.scales + (int64_t)e * a.gate.expert_stride_sb;
      g.b[0] = a.gate.biases + (int64_t)e * a.gate.expert_stride_sb;
      g.w[1] = a.up.w + (int64_t)e * a.up.expert_stride_w;
      g.s[1] = a.up.scales + (int64_t)e * a.up.expert_stride_sb;
      g.b[1] = a.up.biases + (int64_t)e * a.up.expert_stride_sb;
      g.out_dim = a.I;
      g.in_dim = a.H;
      g.G = a.gate.group_size;
      g.n_vec = cnt;
      g.unit_begin = u * a.units_per_seg_gu;
      g.vec_mode = 1;
      g.src_base = nullptr;
      g.src_stride = 0;
      g.dst_base = nullptr;
      g.dst_stride = 0;
      g.vecs = a.vecs_gu + i;
      a.segs_gu[u] = g;
      Seg dn;
      dn.w[0] = dn.w[1] = a.down.w + (int64_t)e * a.down.expert_stride_w;
      dn.s[0] = dn.s[1] = a.down.scales + (int64_t)e * a.down.expert_stride_sb;
      dn.b[0] = dn.b[1] = a.down.biases + (int64_t)e * a.down.expert_stride_sb;
      dn.out_dim = a.H;
      dn.in_dim = a.I;
      dn.G = a.down.group_size;
      dn.n_vec = cnt;
      dn.unit_begin = u * a.units_per_seg_dn;
      dn.vec_mode = 1;
      dn.src_base = nullptr;
      dn.src_stride = 0;
      dn.dst_base = nullptr;
      dn.dst_stride = 0;
      dn.vecs = a.vecs_dn + i;
      a.segs_dn[u] = dn;
    }
  }
  if (tid == 0) {
    int nseg_gu = n_entries, nseg_dn = n_entries;
    int units_gu = n_entries * a.units_per_seg_gu, units_dn = n_entries * a.units_per_seg_dn;
    int sep_gu[2] = {0, 0}, sep_dn[2] = {0, 0};
    if (a.has_shared) {
      // the shared expert: all M tokens, strided rows after the M*K pair rows
      Seg g;
      g.w[0] = a.sh_gate.w;
      g.s[0] = a.sh_gate.scales;
      g.b[0] = a.sh_gate.biases;
      g.w[1] = a.sh_up.w;
      g.s[1] = a.sh_up.scales;
      g.b[1] = a.sh_up.biases;
      g.out_dim = a.sh_gate.out_dim;
      g.in_dim = a.H;
      g.G = a.sh_gate.group_size;
      g.n_vec = M;
      g.vec_mode = 0;
      g.src_base = a.x;
      g.src_stride = a.H;
      g.dst_base = a.h + (int64_t)n * a.I;
      g.dst_stride = a.sh_gate.out_dim;
      g.vecs = nullptr;
      Seg dn;
      dn.w[0] = dn.w[1] = a.sh_down.w;
      dn.s[0] = dn.s[1] = a.sh_down.scales;
      dn.b[0] = dn.b[1] = a.sh_down.biases;
      dn.out_dim = a.H;
      dn.in_dim = a.sh_down.in_dim;
      dn.G = a.sh_down.group_size;
      dn.n_vec = M;
      dn.vec_mode = 0;
      dn.src_base = a.h + (int64_t)n * a.I;
      dn.src_stride = a.sh_gate.out_dim;
      dn.dst_base = a.d + (int64_t)n * a.H;
      dn.dst_stride = a.H;
      dn.vecs = nullptr;
      // same bit width as the routed experts: appended to the routed list;
      // otherwise stored at index n (one past the largest routed list) for a
      // launch of its own
      const bool same_gu = a.shared_same_gu != 0;
      const bool same_dn = a.shared_same_dn != 0;
      g.unit_begin = same_gu ? units_gu : 0;
      dn.unit_begin = same_dn ? units_dn : 0;
      a.segs_gu[same_gu ? n_entries : n] = g;
      a.segs_dn[same_dn ? n_entries : n] = dn;
      if (same_gu) {
        nseg_gu += 1;
        units_gu += a.units_per_seg_gu_sh;
      } else {
        sep_gu[0] = 1;
        sep_gu[1] = a.units_per_seg_gu_sh;
      }
      if (same_dn) {
        nseg_dn += 1;
        units_dn += a.units_per_seg_dn_sh;
      } else {
        sep_dn[0] = 1;
        sep_dn[1] = a.units_per_seg_dn_sh;
      }
    }
    a.count_gu[0] = nseg_gu;
    a.count_gu[1] = units_gu;
    a.count_gu[2] = sep_gu[0];
    a.count_gu[3] = sep_gu[1];
    a.count_dn[0] = nseg_dn;
    a.count_dn[1] = units_dn;
    a.count_dn[2] = sep_dn[0];
    a.count_dn[3] = sep_dn[1];
  }
}

cudaError_t launch_decode_plan(const DecodePlanArgs& a, cudaStream_t st) {
  const int n = a.M * a.K;
  const int threads = 1024;
  const size_t smem = (size_t)n * 4 * 4 + (size_t)(threads / 32) * ((a.E + 31) / 32) * 4;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_decode_plan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  k_decode_plan<<<1, threads, smem, st>>>(a);
  return cudaGetLastError();
}

// ============================================================== combine
__global__ void __launch_bounds__(256) k_combine(const float* __restrict__ d,
                                                 const float* __restrict__ w,
                                                 const float* __restrict__ sigma, int has_shared,
                                                 const float* __restrict__ residual,
                                                 float* __restrict__ y, int M, int K, int H) {
  const int H4 = H >> 2;
  const int64_t total = (int64_t)M * H4;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / H4);
    const int c4 = (int)(i % H4);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = 0; k < K; ++k) {
      const float wk = w[(int64_t)t * K + k];
      const float4 v = reinterpret_cast<const float4*>(d + ((int64_t)t * K + k) * H)[c4];
      acc.x = fmaf(wk, v.x, acc.x);
      acc.y = fmaf(wk, v.y, acc.y);
      acc.z = fmaf(wk, v.z, acc.z);
      acc.w = fmaf(wk, v.w, acc.w);
    }
    if (has_shared) {
      const float sg = sigma[t];
      const float4 v = reinterpret_cast<const float4*>(d + ((int64_t)M * K + t) * H)[c4];
      acc.x = fmaf(sg, v.x, acc.x);
      acc.y = fmaf(sg, v.y, acc.y);
      acc.z = fmaf(sg, v.z, acc.z);
      acc.w = fmaf(sg, v.w, acc.w);
    }
    if (residual) {
      const float4 r = reinterpret_cast<const float4*>(residual + (int64_t)t * H)[c4];
      acc.x += r.x;
      acc.y += r.y;
      acc.z += r.z;
      acc.w += r.w;
    }
    reinterpret_cast<float4*>(y + (int64_t)t * H)[c4] = acc;
  }
}

cudaError_t launch_combine(const float* d, const float* w, const float* sigma, int has_shared,
                           const float* residual, float* y, int M, int K, int H, cudaStream_t st) {
  const int64_t total = (int64_t)M * (H / 4);
  if (total <= 0) return cudaSuccess;
  int64_t grid = (total + 255) / 256;
  if (grid > 148 * 16) grid = 148 * 16;
  k_combine<<<(int)grid, 256, 0, st>>>(d, w, sigma, has_shared, residual, y, M, K, H);
  return cudaGetLastError();
}

}  // namespace moeq
