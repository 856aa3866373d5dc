// Single-token decode (M = 1) in three lean launches.
//
// The per-layer pipeline of the flash-moe-inference page ("Per-layer
// pipeline") runs, for one token, the router matvec, the top-K selection,
// the K experts' gate/up matvecs with SwiGLU, their down matvecs, and the
// weighted combine with the sigmoid-gated shared expert.  For one token each
// phase reads a few MB of weights exactly once, so its time is set by how
// soon all of its loads are in flight, not by arithmetic.  Each launch here:
//   - splits every matrix it reads into per-CTA blocks of whole rows (codes,
//     scales and biases in 16-byte runs), and bulk-copies all of a CTA's
//     blocks into shared memory at once, one mbarrier per matrix;
//   - issues the blocks that do not depend on the preceding launch (router
//     rows, the shared expert's rows) before its programmatic-dependency
//     wait;
//   - computes rows with the decode engine's arithmetic (gemv.cuh: exact
//     dp4a sums of the codes with a fixed-point copy of the input, scale and
//     bias per group), one warp per row; the input's limbs are built once
//     per CTA into shared memory and then held in registers.
// The launches:
//   R  router rows and the shared-expert gate row -> logits;
//   G  top-K (one warp per CTA, route.cuh's selection), then the shared and
//      routed gate/up rows with SwiGLU -> h; also pulls into L2 the routed
//      down rows that D's CTA of the same index reads;
//   D  the shared and routed down rows of the CTA's output rows, summed
//      with the routing weights and the shared gate by the warp that owns
//      the row (no cross-CTA combine), plus the residual -> y.
#include <atomic>
#include <cstring>

#include "gemv.cuh"
#include "kernels.h"
#include "route.cuh"
#include "tc.cuh"

namespace moeq {

namespace {

constexpr int kS1Threads = 256;        // R: 8 warps
constexpr int kS1WideThreads = 512;    // G and D: 16 warps
constexpr int kS1RowsPerWarp = 4;      // D: output rows per warp
constexpr int kS1SlicesBar = 2;        // G: named barrier of warps 1.. "slices built"
constexpr int kS1CopyBar = 1;          // D: named barrier of the copying warps
// G's registers per thread: 512 x 96 leaves room for an R CTA (256 x 48)
// on the same SM, so G's CTAs start while R runs
constexpr int kS1GateUpRegs = 96;
constexpr uint32_t kS1SmemMax = 227 * 1024;
constexpr int kS1HeadBytes = 512;      // barriers, routing, shared gate value

struct S1Smem {
  // head: [0, 256) mbarriers; [256, 320) expert ids; [320, 384) weights;
  // [384] shared gate value
  static constexpr int IDX_OFF = 256;
  static constexpr int W_OFF = 320;
  static constexpr int SIG_OFF = 384;
};

__host__ __device__ inline uint32_t s1_al(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// Rows [lo, hi) of an n-row matrix for CTA c of `grid`, in units of q rows.
__host__ __device__ inline void s1_rows(int n, int q, int grid, int c, int& lo, int& hi) {
  const int64_t nu = n / q;
  lo = (int)((int64_t)c * nu / grid) * q;
  hi = (int)((int64_t)(c + 1) * nu / grid) * q;
}

// Shared-memory region of a block of at most `rows` rows of one matrix
// (codes, then scales and biases, each 16-byte aligned), `nmat` matrices
// (gate and up: 2) side by side.
struct S1Blk {
  uint32_t codes, sc, bi, bytes;  // offsets of matrix 0; matrix 1 follows at +stride
  uint32_t stride;
};
__host__ __device__ inline S1Blk s1_blk(int rows, int row_bytes, int gpr, int nmat) {
  S1Blk b;
  const uint32_t cb = (uint32_t)rows * row_bytes;
  const uint32_t sbb = s1_al((uint32_t)rows * gpr * 2, 16);
  b.stride = cb + 2 * sbb;
  b.codes = 0;
  b.sc = cb;
  b.bi = cb + sbb;
  b.bytes = s1_al(b.stride * nmat, 128);
  return b;
}

template <int BITS, int NL>
constexpr int s1_slw() {
  return NL * Chunk<BITS>::NC + 2 * SliceVec<BITS, NL>::NB;
}

// Issues the bulk copies of rows [lo, hi) of one packed matrix (expert e)
// into a block region; returns the bytes.
__device__ __forceinline__ uint32_t s1_issue(const moeq_qtensor& t, int64_t e, int lo, int hi,
                                             uint32_t dst_codes, uint32_t dst_s, uint32_t dst_b,
                                             uint64_t* bar) {
  const int n = hi - lo;
  if (n <= 0) return 0;
  const int rw = t.in_dim * t.bits / 32;  // words per row
  const int gpr = t.in_dim / t.group_size;
  const uint32_t cb = (uint32_t)n * rw * 4, sb = (uint32_t)n * gpr * 2;
  tc::bulk_g2s(dst_codes, t.w + e * t.expert_stride_w + (int64_t)lo * rw, cb, bar);
  tc::bulk_g2s(dst_s, t.scales + e * t.expert_stride_sb + (int64_t)lo * gpr, sb, bar);
  tc::bulk_g2s(dst_b, t.biases + e * t.expert_stride_sb + (int64_t)lo * gpr, sb, bar);
  return cb + 2 * sb;
}

__host__ __device__ inline uint32_t s1_bytes(const moeq_qtensor& t, int n) {
  return n <= 0 ? 0u
                : (uint32_t)n * (uint32_t)(t.in_dim * t.bits / 8) +
                      2u * (uint32_t)n * (uint32_t)(t.in_dim / t.group_size) * 2u;
}

// The CTA's slices of one input vector (cpr chunks) into shared memory,
// by the threads [t0, t0 + nthr) (whole warps); slot s holds chunks
// 32 s .. 32 s + 31, word-major.
template <int BITS, int NL, class SRC>
__device__ __forceinline__ void s1_build_slices(const void* src, int cpr, uint32_t* base, int t0,
                                                int nthr) {
  constexpr int SLW = s1_slw<BITS, NL>();
  const int lane = threadIdx.x & 31;
  const int wb = ((int)threadIdx.x - t0) & ~31;
  for (int c0 = wb; c0 < cpr; c0 += nthr) {
    const int ch = c0 + lane;
    SliceVec<BITS, NL> sv;
    build_slice<BITS, NL, SRC>(src, ch, ch < cpr, sv);
    slice_store<BITS, NL>(base + (c0 >> 5) * SLW * 32, sv, lane);
  }
}

// One lane's part of a row's dot product with the input whose slices the
// lane holds (chunks ch0 + lane, ch0 + lane + 32, ...).  codes/sc/bi: shared
// addresses of the row's codes, scales and biases.
template <int BITS, int NL, int NSL>
__device__ __forceinline__ float s1_row_part(uint32_t codes, uint32_t sc, uint32_t bi,
                                             const SliceVec<BITS, NL> (&sv)[NSL], int lane,
                                             int cpr, int gsh, int ch0 = 0) {
  constexpr int VPC = Chunk<BITS>::VPC, NC = Chunk<BITS>::NC, NB = SliceVec<BITS, NL>::NB;
  float acc = 0.0f;
#pragma unroll
  for (int s = 0; s < NSL; ++s) {
    const int ch = ch0 + s * 32 + lane;
    if (ch < cpr) {
      const uint4 wv = gq_lds128(codes + ch * 16);
      uint32_t c[NC];
      Chunk<BITS>::split(wv, c);
      float s2[2] = {0.0f, 0.0f}, b2[2] = {0.0f, 0.0f};
#pragma unroll
      for (int pb = 0; pb < NB; ++pb) {
        const int g = (ch * VPC + pb * kXBlock) >> gsh;
        s2[pb] = bf16_bits_to_float(lds_u16(sc + g * 2));
        b2[pb] = bf16_bits_to_float(lds_u16(bi + g * 2));
      }
      acc += chunk_contrib<BITS, NL>(c, sv[s], s2, b2);
    }
  }
  return acc;
}

template <int BITS, int NL, int NSL>
__device__ __forceinline__ void s1_load_slices(const uint32_t* base, SliceVec<BITS, NL> (&sv)[NSL],
                                               int lane) {
  constexpr int SLW = s1_slw<BITS, NL>();
#pragma unroll
  for (int s = 0; s < NSL; ++s) slice_load<BITS, NL>(base + s * SLW * 32, sv[s], lane);
}

__device__ __forceinline__ int s1_log2(int g) { return 31 - __clz(g); }

// Waits (bounded) for the copies a CTA issued on the barriers in `mask`
// before it exits, so that no bulk copy lands in freed shared memory (the
// phases have completed already unless a wait ran out).
__device__ __forceinline__ void s1_drain(uint64_t* bars, uint32_t mask, int* status) {
  for (int m = 0; m < 32; ++m)
    if ((mask >> m) & 1u) tc::mbar_wait(&bars[m], 0, status);
}

// ------------------------------------------------------------------ R: router rows
// Warp w holds input slot w % ns (chunks 32 s .. 32 s + 31, ns = nsR) in
// registers and takes the rows of row group w / ns; each row's ns partial
// sums meet in shared memory and are added in slot order.
__global__ void __launch_bounds__(kS1Threads, 1) k_s1_router(const __grid_constant__ S1Args a) {
  constexpr int BITS = 8, NL = 3;
  extern __shared__ __align__(128) uint8_t sm[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm);
  float* red = reinterpret_cast<float*>(sm + kS1HeadBytes);  // [row][8]
  const uint32_t sb = tc::smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const moeq_qtensor& R = a.router;
  const int rb = a.H * BITS / 8, gpr = a.H / R.group_size;
  // router rows only when the launch routes (a given routing needs the
  // shared-gate row alone)
  int r0, r1;
  s1_rows(a.idx_in ? 0 : a.E, a.qR, gridDim.x, blockIdx.x, r0, r1);
  // the shared-gate row goes to CTA 0, whose block of router rows is the
  // smallest (row blocks round down)
  const bool sg = a.has_shared && blockIdx.x == 0;
  const uint32_t blk_off = s1_al(kS1HeadBytes + (a.r_rows_max + 1) * 8 * 4, 128);
  const S1Blk rbk = s1_blk(a.r_rows_max, rb, gpr, 1);
  const S1Blk gbk = s1_blk(1, rb, gpr, 1);
  const uint32_t sg_off = blk_off + rbk.bytes;
  if (tid == 0) {
    tc::mbar_init(bar, 1);
    tc::fence_mbar_init();
    // the router's weights do not depend on the preceding launch
    uint32_t bytes = s1_bytes(R, r1 - r0) + (sg ? s1_bytes(a.sg, 1) : 0u);
    tc::mbar_arrive_expect_tx(bar, bytes);
    s1_issue(R, 0, r0, r1, sb + blk_off + rbk.codes, sb + blk_off + rbk.sc, sb + blk_off + rbk.bi,
             bar);
    if (sg)
      s1_issue(a.sg, 0, 0, 1, sb + sg_off + gbk.codes, sb + sg_off + gbk.sc, sb + sg_off + gbk.bi,
               bar);
  }
  tc::grid_dep_wait();
  tc::grid_dep_launch();
  const int ns = a.nsR, rg = 8 / ns;
  const int slot = warp % ns, grp = warp / ns;
  const int cpr = a.H / Chunk<BITS>::VPC;
  const int ch0 = slot * 32;
  SliceVec<BITS, NL> sv[1];
  if (grp < rg) build_slice<BITS, NL, SrcBF16>(a.x, ch0 + lane, ch0 + lane < cpr, sv[0]);
  __syncthreads();  // the barrier's initialisation is visible to every thread
  const bool ok = tc::mbar_wait(bar, 0, a.status);
  const int nr = r1 - r0 + (sg ? 1 : 0);
  const int gsh = s1_log2(R.group_size);
  for (int i = grp; ok && grp < rg && i < nr; i += rg) {
    const bool is_sg = i >= r1 - r0;
    const uint32_t base = is_sg ? sb + sg_off : sb + blk_off;
    const S1Blk& k = is_sg ? gbk : rbk;
    const int j = is_sg ? 0 : i;
    const float p = s1_row_part<BITS, NL, 1>(base + k.codes + j * rb, base + k.sc + j * gpr * 2,
                                             base + k.bi + j * gpr * 2, sv, lane, cpr, gsh, ch0);
    const float t = warp_sum(p);
    if (lane == 0) red[i * 8 + slot] = t;
  }
  __syncthreads();
  if (ok && tid < nr) {
    float t = 0.0f;
    for (int q = 0; q < ns; ++q) t += red[tid * 8 + q];
    if (tid >= r1 - r0) *a.sg_logit = t;
    else a.logits[r0 + tid] = t;
  }
  if (tid == 0) s1_drain(bar, 1u, a.status);
}

// Rows [lo, hi) of one packed matrix (expert e) into a block region with
// 16-byte asynchronous copies spread over the CTA's threads (scales and
// biases are whole 16-byte runs: the row quanta guarantee it).
__device__ __forceinline__ void s1_async_rows(const moeq_qtensor& t, int64_t e, int lo, int hi,
                                              uint32_t dst_codes, uint32_t dst_s, uint32_t dst_b,
                                              int tid, int nthr) {
  const int n = hi - lo;
  if (n <= 0) return;
  const int rw = t.in_dim * t.bits / 32;
  const int gpr = t.in_dim / t.group_size;
  const uint8_t* wc = reinterpret_cast<const uint8_t*>(t.w + e * t.expert_stride_w + (int64_t)lo * rw);
  const uint8_t* ws = reinterpret_cast<const uint8_t*>(t.scales + e * t.expert_stride_sb +
                                                       (int64_t)lo * gpr);
  const uint8_t* wb = reinterpret_cast<const uint8_t*>(t.biases + e * t.expert_stride_sb +
                                                       (int64_t)lo * gpr);
  const int cb = n * rw * 4, sbb = n * gpr * 2;
  for (int o = tid * 16; o < cb; o += nthr * 16) tc::cp_async16(dst_codes + o, wc + o, 16);
  for (int o = tid * 16; o < sbb; o += nthr * 16) {
    tc::cp_async16(dst_s + o, ws + o, 16);
    tc::cp_async16(dst_b + o, wb + o, 16);
  }
}

// Top-K of one token's E <= 32 NJ logits by one warp with route.cuh's rule
// (the K largest scaled logits, ties to the lower index, listed by value;
// weights p_k over the chosen sum with renormalisation, else over the
// softmax normaliser).  Lane l holds experts NJ l .. NJ l + NJ - 1, loaded
// with 16-byte loads when NJ is a multiple of 4 (lg 16-byte aligned).
template <int NJ>
__device__ __forceinline__ void s1_topk(const float* __restrict__ lg, int E, int K, int renorm,
                                        float scale, int32_t* idx, float* w) {
  const int lane = threadIdx.x & 31;
  const int e0 = lane * NJ;
  float v[NJ];
  if (NJ % 4 == 0 && e0 + NJ <= E) {
#pragma unroll
    for (int q = 0; q < NJ / 4; ++q) {
      const float4 f = __ldcg(reinterpret_cast<const float4*>(lg + e0) + q);
      v[4 * q] = f.x;
      v[4 * q + 1] = f.y;
      v[4 * q + 2] = f.z;
      v[4 * q + 3] = f.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < NJ; ++j) v[j] = e0 + j < E ? lg[e0 + j] : 0.0f;
  }
  uint32_t key[NJ];
  uint32_t avail = 0;  // bit j: expert e0 + j exists and is not taken
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    v[j] *= scale;
    key[j] = route_key(v[j]);
    if (e0 + j < E) avail |= 1u << j;
  }
  uint32_t lk = 0;
  int li = kNoExpert;
  float lv = 0.0f;
#pragma unroll
  for (int j = 0; j < NJ; ++j)
    if (((avail >> j) & 1u) && (li == kNoExpert || key[j] > lk)) {
      lk = key[j];
      li = e0 + j;
      lv = v[j];
    }
  float mx = 0.0f, chosen_sum = 0.0f, my_p = 0.0f;
  int my_i = 0;
  for (int k = 0; k < K; ++k) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, lk);
    const uint32_t win = __reduce_min_sync(
        0xffffffffu, (li != kNoExpert && lk == m) ? (uint32_t)li : 0xffffffffu);
    const int wl = (int)(win / NJ);
    const float bv = __shfl_sync(0xffffffffu, lv, wl & 31);
    if (k == 0) mx = bv;
    if (win != 0xffffffffu && wl == lane) {
      avail &= ~(1u << (win - e0));
      lk = 0;
      li = kNoExpert;
#pragma unroll
      for (int j = 0; j < NJ; ++j)
        if (((avail >> j) & 1u) && (li == kNoExpert || key[j] > lk)) {
          lk = key[j];
          li = e0 + j;
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
  float z = 0.0f;
  if (!renorm) {
#pragma unroll
    for (int j = 0; j < NJ; ++j)
      if (e0 + j < E) z += expf(v[j] - mx);
    z = warp_sum(z);
  }
  if (lane < K) {
    idx[lane] = my_i;
    w[lane] = my_p / (renorm ? chosen_sum : z);
  }
  __syncwarp();
}

// ------------------------------------------------------------------ G: top-K, gate/up + SwiGLU
// 16 warps.  A row pair (gate row, up row) is split over SGc warps, each
// holding s1_slots(BITS) input slots (chunks ch0 .. ch0 + 32 slots - 1) in
// registers; the SGc partial sums meet in shared memory and are added in
// slot order.  The shared expert (BSH-bit codes, which may differ from the
// routed experts' BITS) has slices of its own layout and its own split.
__host__ __device__ constexpr int s1_slots(int bits) { return bits == 2 ? 1 : 2; }

template <int B, int NSLW>
__device__ __noinline__ bool s1_gateup_items(int H, int* status, int n_items, int nrt, int m0,
                                             const uint32_t* slices, int sgc, uint32_t sb,
                                             uint32_t base0, uint32_t stride_m, S1Blk k,
                                             uint64_t* bars, float* red, int warp, int lane,
                                             int gsh, int nw) {
  constexpr int NL = 2, SLW = s1_slw<B, NL>();
  if (warp >= nw) return true;
  const int ig = warp / sgc, sgi = warp % sgc, IG = nw / sgc;
  if (ig >= IG) return true;
  const int rb = H * B / 8, gpr = H >> gsh, cpr = H / Chunk<B>::VPC;
  const int ch0 = sgi * NSLW * 32;
  SliceVec<B, NL> sv[NSLW];
  s1_load_slices<B, NL, NSLW>(slices + sgi * NSLW * SLW * 32, sv, lane);
  for (int it = ig; it < n_items; it += IG) {
    const int mi = it / nrt, j = it % nrt;
    if (!tc::mbar_wait(&bars[m0 + mi], 0, status)) return false;
    const uint32_t r = sb + base0 + (uint32_t)mi * stride_m;
    const float pg = s1_row_part<B, NL, NSLW>(r + k.codes + j * rb, r + k.sc + j * gpr * 2,
                                              r + k.bi + j * gpr * 2, sv, lane, cpr, gsh, ch0);
    const float pu = s1_row_part<B, NL, NSLW>(
        r + k.stride + k.codes + j * rb, r + k.stride + k.sc + j * gpr * 2,
        r + k.stride + k.bi + j * gpr * 2, sv, lane, cpr, gsh, ch0);
    const float g = warp_sum(pg), u = warp_sum(pu);
    if (lane == 0) {
      red[(it * sgc + sgi) * 2] = g;
      red[(it * sgc + sgi) * 2 + 1] = u;
    }
  }
  return true;
}

template <int BITS, int BSH>
__global__ void __maxnreg__(kS1GateUpRegs) k_s1_gateup(const __grid_constant__ S1Args a) {
  constexpr int NL = 2;
  extern __shared__ __align__(128) uint8_t sm[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm);
  int32_t* sidx = reinterpret_cast<int32_t*>(sm + S1Smem::IDX_OFF);
  float* sw = reinterpret_cast<float*>(sm + S1Smem::W_OFF);
  float* ssig = reinterpret_cast<float*>(sm + S1Smem::SIG_OFF);
  const uint32_t sb = tc::smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.K, hs = a.has_shared ? 1 : 0;
  const int gpr = a.H / a.gate.group_size;
  int g0, g1, s0 = 0, s1 = 0;
  s1_rows(a.I, a.qG, gridDim.x, blockIdx.x, g0, g1);
  if (hs) s1_rows(a.Ish, a.qGs, gridDim.x, blockIdx.x, s0, s1);
  uint32_t* sl_r = reinterpret_cast<uint32_t*>(sm + a.g_sl_r);
  uint32_t* sl_s = reinterpret_cast<uint32_t*>(sm + a.g_sl_s);
  float* red_s = reinterpret_cast<float*>(sm + a.g_red);
  float* red_r = red_s + a.g_sh_max * a.g_sgc_s * 2;
  const S1Blk shb = s1_blk(a.g_sh_max, a.H * BSH / 8, gpr, 2);
  const S1Blk rtb = s1_blk(a.g_rt_max, a.H * BITS / 8, gpr, 2);
  const uint32_t rt_off = a.g_blk + hs * shb.bytes;  // routed block k at rt_off + k * rtb.bytes
  // A shared expert of the routed width is computed by warps 1.. while warp
  // 0 selects the experts (when a row pair's slot groups fit there): 397B-like
  // layer 23.7 -> 23.1 us per step.  A wider shared expert is computed by the
  // lower half of the warps while the upper half copies the routed rows
  // (2-bit bank with its 4-bit shared expert: 27.1 -> 25.4 us).  The item
  // loop is one out-of-line body for its three uses.
  constexpr int kShWarps = kS1WideThreads / 32 - 1;
  const bool early_sh = hs && BSH == BITS && a.g_sgc_s <= kShWarps;
  const int copy_lo = (hs && BSH != BITS) ? kS1WideThreads / 2 : 0;
  if (tid == 0) {
    for (int m = 0; m < hs + K; ++m)
      tc::mbar_init(&bars[m], m < hs ? kS1WideThreads : kS1WideThreads - copy_lo);
    tc::fence_mbar_init();
  }
  __syncthreads();
  // the shared expert's rows do not depend on the routing
  if (hs) {
    const uint32_t r = sb + a.g_blk;
    s1_async_rows(a.sh_gate, 0, s0, s1, r + shb.codes, r + shb.sc, r + shb.bi, tid, kS1WideThreads);
    s1_async_rows(a.sh_up, 0, s0, s1, r + shb.stride + shb.codes, r + shb.stride + shb.sc,
                  r + shb.stride + shb.bi, tid, kS1WideThreads);
    tc::cp_async_arrive_noinc(&bars[0]);
  }
  tc::grid_dep_wait();
  tc::grid_dep_launch();
  bool ok = true;
  if (warp == 0) {
    // the routing (every CTA computes it; CTA 0 publishes it); the shared
    // gate's logit is loaded alongside the router logits
    const float sgl = (hs && lane == 0) ? *a.sg_logit : 0.0f;
    const float* lg = a.logits;
    const int E = a.E;
    if (a.idx_in) {
      // the caller's routing; an expert index out of range is reported and
      // read as expert 0
      if (lane < K) {
        int e = a.idx_in[lane];
        if (e < 0 || e >= E) {
          set_status(a.status, MOEQ_ERR_INVALID_ARG);
          e = 0;
        }
        sidx[lane] = e;
        sw[lane] = a.w_in[lane];
      }
      __syncwarp();
    } else if (E <= 32) s1_topk<1>(lg, E, K, a.renorm, a.router_scale, sidx, sw);
    else if (E <= 64) s1_topk<2>(lg, E, K, a.renorm, a.router_scale, sidx, sw);
    else if (E <= 128) s1_topk<4>(lg, E, K, a.renorm, a.router_scale, sidx, sw);
    else if (E <= 256) s1_topk<8>(lg, E, K, a.renorm, a.router_scale, sidx, sw);
    else s1_topk<16>(lg, E, K, a.renorm, a.router_scale, sidx, sw);  // E <= 512
    if (lane == 0 && hs) *ssig = 1.0f / (1.0f + expf(-sgl));
    __syncwarp();
    if (blockIdx.x == 0) {
      if (lane < K) {
        a.idx[lane] = sidx[lane];
        a.w[lane] = sw[lane];
      }
      if (lane == 0 && hs) *a.sigma = *ssig;
    }
  } else {
    s1_build_slices<BITS, NL, SrcBF16>(a.x, a.H / Chunk<BITS>::VPC, sl_r, 32, kS1WideThreads - 32);
    if (BSH != BITS && hs)
      s1_build_slices<BSH, NL, SrcBF16>(a.x, a.H / Chunk<BSH>::VPC, sl_s, 32,
                                        kS1WideThreads - 32);
    if (early_sh && s1 > s0) {
      tc::named_sync(kS1SlicesBar, kS1WideThreads - 32);  // the token's slices are built
      ok = s1_gateup_items<BSH, s1_slots(BSH)>(a.H, a.status, s1 - s0, s1 - s0, 0,
                                               BSH == BITS ? sl_r : sl_s, a.g_sgc_s, sb,
                                               a.g_blk, 0u, shb, bars, red_s, warp - 1, lane,
                                               s1_log2(a.gate.group_size), kShWarps);
    }
  }
  __syncthreads();
  // the routed experts' rows, by threads copy_lo ..
  if (tid >= copy_lo)
    for (int k = 0; k < K; ++k) {
      const uint32_t r = sb + rt_off + (uint32_t)k * rtb.bytes;
      const int64_t e = sidx[k];
      const int t = tid - copy_lo, nt = kS1WideThreads - copy_lo;
      s1_async_rows(a.gate, e, g0, g1, r + rtb.codes, r + rtb.sc, r + rtb.bi, t, nt);
      s1_async_rows(a.up, e, g0, g1, r + rtb.stride + rtb.codes, r + rtb.stride + rtb.sc,
                    r + rtb.stride + rtb.bi, t, nt);
      tc::cp_async_arrive_noinc(&bars[hs + k]);
    }
  if (warp == 1 && lane < K && (int)blockIdx.x < a.gridD) {
    // the routed down rows that D's CTA of this index will read, into L2
    int d0, d1;
    s1_rows(a.H, a.qD, a.gridD, blockIdx.x, d0, d1);
    const moeq_qtensor& D = a.down;
    const int64_t e = sidx[lane];
    const int rw = D.in_dim * D.bits / 32, dg = D.in_dim / D.group_size;
    if (d1 > d0) {
      tc::prefetch_l2(D.w + e * D.expert_stride_w + (int64_t)d0 * rw, (uint32_t)(d1 - d0) * rw * 4);
      tc::prefetch_l2(D.scales + e * D.expert_stride_sb + (int64_t)d0 * dg,
                      (uint32_t)(d1 - d0) * dg * 2);
      tc::prefetch_l2(D.biases + e * D.expert_stride_sb + (int64_t)d0 * dg,
                      (uint32_t)(d1 - d0) * dg * 2);
    }
  }
  const int gsh = s1_log2(a.gate.group_size);
  const int nsh = s1 - s0, nrt = g1 - g0;
  // the shared rows here unless computed during the selection (on the lower
  // half of the warps while the upper half copies, when their slot groups
  // fit there), then the routed experts' rows
  const int nw_sh = copy_lo && a.g_sgc_s <= copy_lo / 32 ? copy_lo / 32 : kS1WideThreads / 32;
  if (ok && hs && !early_sh && nsh > 0)
    ok = s1_gateup_items<BSH, s1_slots(BSH)>(a.H, a.status, nsh, nsh, 0, BSH == BITS ? sl_r : sl_s,
                                             a.g_sgc_s, sb, a.g_blk, 0u, shb, bars, red_s, warp,
                                             lane, gsh, nw_sh);
  if (ok && nrt > 0)
    ok = s1_gateup_items<BITS, s1_slots(BITS)>(a.H, a.status, K * nrt, nrt, hs, sl_r, a.g_sgc_r, sb, rt_off,
                                               rtb.bytes, rtb, bars, red_r, warp, lane, gsh,
                                               kS1WideThreads / 32);
  if (!ok && lane == 0) set_status(a.status, MOEQ_ERR_TIMEOUT);
  const bool all_ok = __syncthreads_and(ok);
  if (all_ok) {
    for (int t = tid; t < nsh + K * nrt; t += kS1WideThreads) {
      const bool shr = t < nsh;
      const int q0 = shr ? t : t - nsh, nq = shr ? a.g_sgc_s : a.g_sgc_r;
      const float* rr = (shr ? red_s : red_r) + q0 * nq * 2;
      float g = 0.0f, u = 0.0f;
      for (int q = 0; q < nq; ++q) {
        g += rr[2 * q];
        u += rr[2 * q + 1];
      }
      float* dst = shr ? a.h + (int64_t)K * a.I + s0 + t
                       : a.h + (int64_t)(q0 / nrt) * a.I + g0 + q0 % nrt;
      *dst = __fdividef(g, 1.0f + __expf(-g)) * u;
    }
  }
  tc::cp_async_wait_all();
}

// ------------------------------------------------------------------ D: down rows + combine
// 16 warps; warp w owns output rows w, w + 16, ... of the CTA's block and
// sums, for each of them, every matrix's row (shared first, then the routed
// experts in slot order) weighted by the shared gate or the routing weight.
// The shared down matrix has BSH-bit codes, the routed ones BITS.
template <int B, int NSL>
__device__ __forceinline__ bool s1_down_matrix(float (&acc)[kS1RowsPerWarp], const uint32_t* set,
                                               uint32_t r, const S1Blk& k, int in_dim, float coef,
                                               uint64_t* bar, int nd, int warp, int lane, int gsh,
                                               int* status) {
  constexpr int NL = 2, NW = kS1WideThreads / 32;
  const int rb = in_dim * B / 8, gpr = in_dim >> gsh, cpr = in_dim / Chunk<B>::VPC;
  SliceVec<B, NL> sv[NSL];
  s1_load_slices<B, NL, NSL>(set, sv, lane);
  if (!tc::mbar_wait(bar, 0, status)) return false;
#pragma unroll
  for (int j = 0; j < kS1RowsPerWarp; ++j) {
    const int row = warp + NW * j;
    if (row < nd)
      acc[j] += coef * s1_row_part<B, NL, NSL>(r + k.codes + row * rb, r + k.sc + row * gpr * 2,
                                               r + k.bi + row * gpr * 2, sv, lane, cpr, gsh);
  }
  return true;
}

template <int B>
__device__ __forceinline__ void s1_down_slices(const float* src, int cpr, int c0, uint32_t* set,
                                               int lane) {
  constexpr int NL = 2, SLW = s1_slw<B, NL>();
  if (c0 >= cpr) return;
  const int ch = c0 + lane;
  SliceVec<B, NL> v;
  build_slice<B, NL, SrcF32>(src, ch, ch < cpr, v);
  slice_store<B, NL>(set + (c0 >> 5) * SLW * 32, v, lane);
}

template <int BITS, int BSH, int NSL>
__global__ void __launch_bounds__(kS1WideThreads, 1) k_s1_down(const __grid_constant__ S1Args a) {
  constexpr int NW = kS1WideThreads / 32;
  extern __shared__ __align__(128) uint8_t sm[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm);
  int32_t* sidx = reinterpret_cast<int32_t*>(sm + S1Smem::IDX_OFF);
  float* sw = reinterpret_cast<float*>(sm + S1Smem::W_OFF);
  float* ssig = reinterpret_cast<float*>(sm + S1Smem::SIG_OFF);
  const uint32_t sb = tc::smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.K, hs = a.has_shared ? 1 : 0, NM = hs + K;
  const moeq_qtensor& D = a.down;
  int d0, d1;
  s1_rows(a.H, a.qD, gridDim.x, blockIdx.x, d0, d1);
  const int gsh = s1_log2(D.group_size);
  const uint32_t set_words = a.d_set_bytes / 4;
  const S1Blk shb = s1_blk(a.d_rows_max, hs ? a.Ish * BSH / 8 : 16, hs ? a.Ish >> gsh : 8, 1);
  const S1Blk rtb = s1_blk(a.d_rows_max, a.I * BITS / 8, a.I >> gsh, 1);
  auto region = [&](int m) -> uint32_t {
    return sb + a.d_blk + (m < hs ? 0u : hs * shb.bytes + (uint32_t)(m - hs) * rtb.bytes);
  };
  // the shared matrix's barrier counts every thread's copies, a routed
  // matrix's those of the copying warps (the upper half)
  constexpr int kCopyThreads = kS1WideThreads / 2;
  if (tid == 0) {
    for (int m = 0; m < NM; ++m) tc::mbar_init(&bars[m], m < hs ? kS1WideThreads : kCopyThreads);
    tc::fence_mbar_init();
  }
  __syncthreads();
  if (hs) {
    const uint32_t r = region(0);
    s1_async_rows(a.sh_down, 0, d0, d1, r + shb.codes, r + shb.sc, r + shb.bi, tid,
                  kS1WideThreads);
    tc::cp_async_arrive_noinc(&bars[0]);
  }
  tc::grid_dep_wait();
  tc::grid_dep_launch();
  uint32_t* slices = reinterpret_cast<uint32_t*>(sm + kS1HeadBytes);
  const int cpr_r = a.I / Chunk<BITS>::VPC, cpr_s = hs ? a.Ish / Chunk<BSH>::VPC : 0;
  if (tid >= kCopyThreads) {
    // the upper half reads the routing and copies the routed rows while the
    // lower half builds the hidden vectors' slices
    const int t = tid - kCopyThreads;
    if (t < K) {
      sidx[t] = a.idx[t];
      sw[t] = a.w[t];
    }
    if (t == 0 && hs) *ssig = *a.sigma;
    tc::named_sync(kS1CopyBar, kCopyThreads);
    for (int k = 0; k < K; ++k) {
      const uint32_t r = region(hs + k);
      s1_async_rows(D, sidx[k], d0, d1, r + rtb.codes, r + rtb.sc, r + rtb.bi, t, kCopyThreads);
      tc::cp_async_arrive_noinc(&bars[hs + k]);
    }
  } else {
    // the slices of every hidden vector (fp32): matrix m's set at
    // m * set_words; the warps take (matrix, 32-chunk group) pairs in turn
    const int ngrp = ((cpr_r > cpr_s ? cpr_r : cpr_s) + 31) / 32;
    for (int t = warp; t < NM * ngrp; t += kCopyThreads / 32) {
      const int m = t / ngrp, c0 = (t % ngrp) * 32;
      if (m < hs)
        s1_down_slices<BSH>(a.h + (int64_t)K * a.I, cpr_s, c0, slices + m * set_words, lane);
      else
        s1_down_slices<BITS>(a.h + (int64_t)(m - hs) * a.I, cpr_r, c0, slices + m * set_words,
                             lane);
    }
  }
  __syncthreads();
  const int nd = d1 - d0;
  float acc[kS1RowsPerWarp];
#pragma unroll
  for (int j = 0; j < kS1RowsPerWarp; ++j) acc[j] = 0.0f;
  bool ok = true;
  for (int m = 0; m < NM && ok && warp < nd; ++m) {
    if (m < hs)
      ok = s1_down_matrix<BSH, NSL>(acc, slices + m * set_words, region(m), shb, a.Ish, *ssig,
                                    &bars[m], nd, warp, lane, gsh, a.status);
    else
      ok = s1_down_matrix<BITS, NSL>(acc, slices + m * set_words, region(m), rtb, a.I,
                                     sw[m - hs], &bars[m], nd, warp, lane, gsh, a.status);
  }
  if (ok) {
#pragma unroll
    for (int j = 0; j < kS1RowsPerWarp; ++j) {
      const int row = warp + NW * j;
      if (row < nd) {
        const float t = warp_sum(acc[j]);
        if (lane == 0) a.y[d0 + row] = t + (a.residual ? a.residual[d0 + row] : 0.0f);
      }
    }
  }
  tc::cp_async_wait_all();
}

// ------------------------------------------------------------------ host side
int gcd_i(int x, int y) {
  while (y) {
    const int t = x % y;
    x = y;
    y = t;
  }
  return x;
}
// Rows per block unit so that a block's scales start on a 16-byte boundary.
int row_quantum(int gpr) { return 16 / gcd_i(16, 2 * gpr); }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

bool s1_tensor_ok(const moeq_qtensor& t, bool bank) {
  if (t.format != MOEQ_FMT_AFFINE) return false;
  if (!(t.bits == 2 || t.bits == 4 || t.bits == 8)) return false;
  if (!aligned16(t.w) || !aligned16(t.scales) || !aligned16(t.biases)) return false;
  if (bank && ((t.expert_stride_w % 4) || (t.expert_stride_sb % 8))) return false;
  return true;
}

template <class Kern>
cudaError_t s1_launch(Kern kern, std::atomic<bool>* attr, int grid, int threads, uint32_t smem,
                      const S1Args& a, cudaStream_t st) {
  int dev;
  if (!current_device(dev)) return cudaErrorInvalidDevice;
  if (!attr[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kS1SmemMax);
    // every launch asks for the largest shared-memory carveout, so that a
    // launch's CTAs can start on an SM the previous launch still occupies
    // (a different carveout would wait for the SM to drain)
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    attr[dev].store(true, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

cudaError_t launch_r(const S1Args& a, cudaStream_t st) {
  static std::atomic<bool> attr[kMaxDevices];
  return s1_launch(k_s1_router, attr, a.gridR, kS1Threads, a.smem_R, a, st);
}
template <int BITS, int BSH>
cudaError_t launch_g(const S1Args& a, cudaStream_t st) {
  static std::atomic<bool> attr[kMaxDevices];
  return s1_launch(k_s1_gateup<BITS, BSH>, attr, a.gridG, kS1WideThreads, a.smem_G, a, st);
}
template <int BITS, int BSH, int NSL>
cudaError_t launch_d(const S1Args& a, cudaStream_t st) {
  static std::atomic<bool> attr[kMaxDevices];
  return s1_launch(k_s1_down<BITS, BSH, NSL>, attr, a.gridD, kS1WideThreads, a.smem_D, a, st);
}

// Down warps hold a hidden vector's slots: 1, 2 or 4 (2-bit rows of
// 64-value chunks: 1 or 2, intermediate up to 4096).
int d_slots(int ns) { return ns <= 1 ? 1 : ns <= 2 ? 2 : 4; }
template <int BITS, int BSH>
cudaError_t launch_d_bits(const S1Args& a, cudaStream_t st) {
  if (a.nsD <= 1) return launch_d<BITS, BSH, 1>(a, st);
  if (BITS == 2 || a.nsD <= 2) return launch_d<BITS, BSH, 2>(a, st);
  return launch_d<BITS == 2 ? 4 : BITS, BSH == 2 ? 4 : BSH, 4>(a, st);
}

// Code widths the launches are built for: routed = shared in {2, 4, 8}, and
// 2-bit routed experts with a 4-bit shared expert (the requantised bank).
bool s1_bits_pair(int be, int bs) { return (be == bs && (be == 2 || be == 4 || be == 8)) || (be == 2 && bs == 4); }

int slw_of(int bits) { return 2 * (32 / bits) + 2 * (bits == 2 ? 2 : 1); }  // words per slot

}  // namespace

bool single_decode_plan(const moeq_layer* L, int sms, S1Args& a) {
  memset(&a, 0, sizeof(a));
  const int H = L->hidden, I = L->inter, E = L->n_experts, K = L->top_k;
  if (sms < 1 || K < 1 || K > kS1MaxK || E > 512 || E < K) return false;
  const moeq_qtensor &R = L->router, &Gt = L->gate, &U = L->up, &D = L->down;
  // router: 8-bit, and the shared-expert gate row in the same format
  if (R.bits != 8 || !s1_tensor_ok(R, false) || R.out_dim != E || R.in_dim != H) return false;
  const int BE = Gt.bits, GE = Gt.group_size;
  for (const moeq_qtensor* t : {&Gt, &U, &D})
    if (!s1_tensor_ok(*t, true) || t->bits != BE || t->group_size != GE) return false;
  const bool hs = L->has_shared != 0;
  const int Ish = hs ? L->sh_gate.out_dim : 0;
  const int BS = hs ? L->sh_gate.bits : BE;
  if (!s1_bits_pair(BE, BS)) return false;
  if (hs) {
    const moeq_qtensor& SG = L->sh_expert_gate;
    if (!s1_tensor_ok(SG, false) || SG.bits != R.bits || SG.group_size != R.group_size ||
        SG.in_dim != H || ((H / SG.group_size) % 8))
      return false;
    for (const moeq_qtensor* t : {&L->sh_gate, &L->sh_up, &L->sh_down})
      if (!s1_tensor_ok(*t, false) || t->bits != BS || t->group_size != GE) return false;
    if (L->sh_up.out_dim != Ish || L->sh_down.in_dim != Ish || L->sh_down.out_dim != H)
      return false;
  }
  a.H = H;
  a.I = I;
  a.Ish = Ish;
  a.E = E;
  a.K = K;
  a.has_shared = hs;
  a.renorm = L->renorm;
  a.router_scale = L->router_scale;
  a.router = R;
  if (hs) a.sg = L->sh_expert_gate;
  a.gate = Gt;
  a.up = U;
  a.down = D;
  if (hs) {
    a.sh_gate = L->sh_gate;
    a.sh_up = L->sh_up;
    a.sh_down = L->sh_down;
  }
  // row quanta: every block's scales on a 16-byte boundary
  a.qR = row_quantum(H / R.group_size);
  a.qG = row_quantum(H / GE);
  a.qGs = a.qG;
  int qD = row_quantum(I / GE);
  if (hs) {
    const int qs = row_quantum(Ish / GE);
    qD = qD / gcd_i(qD, qs) * qs;
  }
  a.qD = qD;
  if (E % a.qR || I % a.qG || (hs && Ish % a.qGs) || H % a.qD) return false;
  // grids and the largest block of a CTA
  a.gridR = E / a.qR < sms ? E / a.qR : sms;
  a.gridG = sms;
  a.gridD = H / a.qD < sms ? H / a.qD : sms;
  auto most = [](int n, int q, int grid) { return (int)(((n / q) + grid - 1) / grid) * q; };
  a.r_rows_max = most(E, a.qR, a.gridR);
  a.g_rt_max = most(I, a.qG, a.gridG);
  a.g_sh_max = hs ? most(Ish, a.qGs, a.gridG) : 0;
  a.d_rows_max = most(H, a.qD, a.gridD);
  if (a.d_rows_max > (kS1WideThreads / 32) * kS1RowsPerWarp) return false;
  // input slices per lane
  const int vpc = 128 / BE, vps = 128 / BS;
  if (H % 32 || H % vps || I % vpc || (hs && Ish % vps)) return false;
  a.nsR = (H / 16 + 31) / 32;
  a.nsG = (H / vpc + 31) / 32;
  const int nsGs = (H / vps + 31) / 32;
  const int cpr_d = (I / vpc > Ish / vps) ? I / vpc : Ish / vps;
  a.nsD = (cpr_d + 31) / 32;
  if (a.nsR > 8 || a.nsD > (BE == 2 || BS == 2 ? 2 : 4)) return false;
  // G: warps per row (slot groups) of the routed and of the shared layout
  a.g_sgc_r = (a.nsG + s1_slots(BE) - 1) / s1_slots(BE);
  a.g_sgc_s = hs ? (nsGs + s1_slots(BS) - 1) / s1_slots(BS) : 1;
  if (a.g_sgc_r > kS1WideThreads / 32 || a.g_sgc_s > kS1WideThreads / 32) return false;
  // shared memory per launch; the kernels take these offsets as they are
  {
    const int rb = H, gpr = H / R.group_size;
    uint32_t s = s1_al(kS1HeadBytes + (a.r_rows_max + 1) * 8 * 4, 128);
    s += s1_blk(a.r_rows_max, rb, gpr, 1).bytes + s1_blk(1, rb, gpr, 1).bytes;
    a.smem_R = s;
  }
  {
    const int gpr = H / GE;
    a.g_sl_r = kS1HeadBytes;
    uint32_t end = a.g_sl_r + (uint32_t)a.g_sgc_r * s1_slots(BE) * slw_of(BE) * 32 * 4;
    a.g_sl_s = a.g_sl_r;
    if (hs && BS != BE) {
      a.g_sl_s = s1_al(end, 16);
      end = a.g_sl_s + (uint32_t)a.g_sgc_s * s1_slots(BS) * slw_of(BS) * 32 * 4;
    }
    a.g_red = s1_al(end, 16);
    const uint32_t red_floats =
        2u * ((uint32_t)a.g_sh_max * a.g_sgc_s + (uint32_t)K * a.g_rt_max * a.g_sgc_r);
    a.g_blk = s1_al(a.g_red + red_floats * 4, 128);
    a.smem_G = a.g_blk + (hs ? s1_blk(a.g_sh_max, H * BS / 8, gpr, 2).bytes : 0u) +
               (uint32_t)K * s1_blk(a.g_rt_max, H * BE / 8, gpr, 2).bytes;
  }
  {
    const int NM = K + (hs ? 1 : 0);
    const int slw = slw_of(BE) > slw_of(BS) ? slw_of(BE) : slw_of(BS);
    a.d_set_bytes = (uint32_t)d_slots(a.nsD) * slw * 32 * 4;
    a.d_blk = s1_al(kS1HeadBytes + (uint32_t)NM * a.d_set_bytes, 128);
    a.smem_D = a.d_blk + (hs ? s1_blk(a.d_rows_max, Ish * BS / 8, Ish / GE, 1).bytes : 0u) +
               (uint32_t)K * s1_blk(a.d_rows_max, I * BE / 8, I / GE, 1).bytes;
  }
  if (a.smem_R > kS1SmemMax || a.smem_G > kS1SmemMax || a.smem_D > kS1SmemMax) return false;
  return true;
}

cudaError_t launch_single_router(const S1Args& a, cudaStream_t st) { return launch_r(a, st); }

cudaError_t launch_single_gateup(const S1Args& a, cudaStream_t st) {
  const int bs = a.has_shared ? a.sh_gate.bits : a.gate.bits;
  switch (a.gate.bits) {
    case 2: return bs == 4 ? launch_g<2, 4>(a, st) : launch_g<2, 2>(a, st);
    case 4: return launch_g<4, 4>(a, st);
    default: return launch_g<8, 8>(a, st);
  }
}

cudaError_t launch_single_down(const S1Args& a, cudaStream_t st) {
  const int bs = a.has_shared ? a.sh_down.bits : a.down.bits;
  switch (a.down.bits) {
    case 2: return bs == 4 ? launch_d_bits<2, 4>(a, st) : launch_d_bits<2, 2>(a, st);
    case 4: return launch_d_bits<4, 4>(a, st);
    default: return launch_d_bits<8, 8>(a, st);
  }
}

}  // namespace moeq
