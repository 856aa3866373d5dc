// Gather quantised matrix multiply on tcgen05 tensor cores (prefill path).
//
// Persistent, warp-specialised.  A work item is an m-tile of one expert's
// sorted token rows by an n-tile of 256 weight rows, over 64-wide groups
// (k-blocks).  Two forms:
//   PAIR   the two CTAs of a cluster share each item: 256 token rows, each
//          CTA loading 128 of them and dequantising 128 of the weight rows;
//          rank 0 issues tcgen05.mma.cta_group::2 (M 256, N 256, K 16) over
//          both CTAs' shared memory and commits to both CTAs' barriers;
//   single one CTA per item: 128 token rows, 256 weight rows, M 128.
// Warp roles (per CTA):
//   warps 0-1  A loader: token rows (or the expert's contiguous hidden rows)
//              as tensor-map tiles (one thread issues; PAIR: completion
//              counted on rank 0's barrier), or, without tensor maps, 16-byte
//              cp.async gathers;
//   warp  2    B loader: the packed codes of the CTA's weight rows for one
//              k-block (tensor-map tiles of 128 rows, or cp.async per row) and
//              the rows' scales and biases once per window of up to 8 groups;
//   warp  3    MMA issuer (PAIR: rank 0 only), fp32 accumulators in TMEM
//              (two 256-column buffers);
//   warps 4-7  epilogue: tcgen05.ld of the accumulator rows, SwiGLU to fp16
//              hidden rows, or output rows (fp16 or fp32) scattered to pair
//              order, as 32-byte stores;
//   warps 8-15 dequantiser: codes -> fp16 weights w = q*scale + bias (one
//              fused fp16 multiply-add of exact operands) written into the
//              swizzled B stage.
// The scale and bias of a 64-wide group are constant along K within a
// k-block, so dequantising tiles in shared memory applies the affine map of
// the pages' format exactly once per weight before the tensor-core product.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "tc.cuh"

namespace moeq {
namespace gq {

constexpr int BM = 128, BN = 256, BK = 64;  // per MMA issuer: M = BM (PAIR: 2 BM)
constexpr int A_STAGE = BM * BK * 2;   // 16 KB: 128 rows of A per CTA
constexpr int DQ_WARPS = 8;            // dequantiser warps
constexpr int THREADS = (8 + DQ_WARPS) * 32;

// Packed codes of one k-block in shared memory, one dense row per
// dequantiser thread, in the layout a tensor-map load writes: 8-bit rows
// (64 bytes) with the 64-byte swizzle (chunk c of row r at c ^ ((r >> 1) & 3)),
// 4-bit rows (32 bytes) with the 32-byte swizzle (c ^ ((r >> 2) & 1)), 2-bit
// rows (16 bytes) plain.  Either way the eight rows a quarter-warp reads
// touch distinct 16-byte bank groups.
template <int BITS>
struct Raw {
  static constexpr int ROW = BK * BITS / 8;       // packed bytes of one row per k-block
  static constexpr int CHUNKS = ROW / 16;         // 16-byte chunks per row
  __device__ __forceinline__ static int offset(int r, int c) {
    return BITS == 8   ? r * ROW + ((c ^ ((r >> 1) & 3)) << 4)
           : BITS == 4 ? r * ROW + ((c ^ ((r >> 2) & 1)) << 4)
                       : r * ROW + (c << 4);
  }
};

// Shared-memory plan.  PAIR: each CTA of the pair holds 128 of the 256 B
// rows, which frees room for deeper rings.
template <int BITS, bool PAIR>
struct Smem {
  static constexpr int BR = PAIR ? BN / 2 : BN;          // B rows in this CTA
  static constexpr int S1 = PAIR ? 6 : 3;                // A stages
  static constexpr int SR = PAIR ? 4 : 3;                // packed-code stages
  static constexpr int S2 = PAIR ? 4 : 3;                // dequantised B stages
  static constexpr int B_STAGE = BR * BK * 2;
  static constexpr int RAW_STAGE = BR * Raw<BITS>::ROW;
  // scale/bias windows of up to 8 groups (k-blocks): per row 16 bytes of
  // scales, then 16 of biases.  Two window buffers suffice: the dequantiser
  // reads a window in its first k-block, before releasing that k-block's raw
  // stage, and the loader refills the buffer two windows (>= 4 k-blocks)
  // later, after waiting for the release of the k-block SR (<= 4) back.
  static constexpr int SB_WIN = BR * 32;
  static constexpr int NWB = 2;
  static constexpr uint32_t IDESC = tc::idesc_f16_f32(PAIR ? 2 * BM : BM, BN);
  static constexpr int A_OFF = 0;
  static constexpr int B_OFF = A_OFF + S1 * A_STAGE;
  static constexpr int RAW_OFF = B_OFF + S2 * B_STAGE;
  static constexpr int SB_OFF = RAW_OFF + SR * RAW_STAGE;
  static constexpr int BAR_OFF = SB_OFF + NWB * SB_WIN;
  static constexpr int N_BARS = 2 * S1 + 2 * SR + 2 * S2 + 4;
  static constexpr int ATAB_OFF = BAR_OFF + N_BARS * 8;   // 2 x 128 A-row pointers
  static constexpr int TMEM_OFF = ATAB_OFF + 2 * BM * 8;
  static constexpr int BYTES = TMEM_OFF + 16;
  static constexpr int ALLOC = BYTES + 1024;  // room to align the base to 1024
};

enum Epi { EPI_SWIGLU = 0, EPI_STORE = 1, EPI_SPLIT = 2 };
enum AMode { A_PAIRS = 0, A_TOKENS = 1, A_ROWS = 2 };

// One expert (or the shared expert, or the router) over a run of sorted rows.
struct Seg {
  const uint32_t* w[2];
  const uint16_t* s[2];
  const uint16_t* b[2];
  int32_t n0;         // SWIGLU: rows per source (I); STORE: rows taken from source 0
  int32_t n_valid;    // STORE: valid weight rows in total (source 0 then source 1)
  int32_t row_begin;  // first row of the segment in the sorted row space
  int32_t rows;       // rows of the segment
  int32_t a_mode;     // AMode
  int32_t dest_pairs; // STORE: 1 = output row is the pair index sorted_pair[m]
  int32_t ex[2];      // matrix index of each source in its code tensor map
};

struct Args {
  // contiguous A rows (A_TOKENS, A_ROWS): tiles fetched by the tensor-memory
  // accelerator from this map (box 64 x 128 fp16, 128-byte swizzle) when
  // tma_a is set; gathered rows (A_PAIRS) always use cp.async
  CUtensorMap tmA;
  int32_t tma_a;
  // packed codes (SWIGLU: gate and up, STORE: the single source) fetched by
  // tensor-map tiles of 128 rows x one 64-wide group when tma_b is set
  CUtensorMap tmB[2];
  int32_t tma_b;
  const Seg* segs;
  const int2* tiles;        // (segment, first row within the segment); null: seg0 only
  const int32_t* n_tiles;   // device count of tiles
  Seg seg0;                 // the single segment when tiles == null
  int32_t static_mtiles;    // m-tiles of seg0 when tiles == null
  int32_t n_tiles_n;        // n-tiles per m-tile
  int32_t K;                // reduction length, multiple of 128
  const __half* A;
  int64_t lda;              // elements
  const int32_t* sorted_pair;
  int32_t topk;
  void* out;
  int64_t ldo;              // elements
  int32_t out_f16;          // STORE: fp16 output rows (range-checked) instead of fp32
  int32_t sb_w;             // groups per scale/bias window copy: 8, 4 or 2 (dividing K/G;
                            // scale/bias rows aligned to 2*sb_w bytes; a window spans
                            // sb_w*G/64 >= 2 k-blocks)
  int32_t G;                // group size of the launch's tensors: 32, 64 or 128 (32: not
                            // 2-bit, whose 16-byte code chunks span two groups)
  int32_t fmt;              // MOEQ_FMT_*: MX FP4 windows hold one exponent byte per group
  int* status;
};

// k-blocks (of BK = 64 values) spanned by a window of W groups of size G,
// as a power of two: log2(W * G / 64).
__host__ __device__ __forceinline__ int win_kb_log2(int W, int G) {
  const int wl = W == 8 ? 3 : W == 4 ? 2 : 1;
  return wl + (G == 128 ? 1 : G == 32 ? -1 : 0);
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// 32-byte global store (32-byte aligned address): one full sector per lane.
__device__ __forceinline__ void stg256(void* p, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t a4, uint32_t a5, uint32_t a6, uint32_t a7) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(a0), "r"(a1),
               "r"(a2), "r"(a3), "r"(a4), "r"(a5), "r"(a6), "r"(a7)
               : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Weight row of tile row r (0..255) of n-tile nt: source index, row within
// the source matrix, validity.
template <int EPI>
__device__ __forceinline__ void b_row(const Seg& sg, int nt, int r, int& src, int& q, bool& ok) {
  if (EPI == EPI_SWIGLU) {
    src = r >= 128;
    q = nt * 128 + (r & 127);
    ok = q < sg.n0;
  } else if (EPI == EPI_SPLIT) {
    const int g = nt * 128 + (r & 127);
    src = g >= sg.n0;
    q = src ? g - sg.n0 : g;
    ok = g < sg.n_valid;
  } else {
    const int g = nt * BN + r;
    src = g >= sg.n0;
    q = src ? g - sg.n0 : g;
    ok = g < sg.n_valid;
  }
}

// fp16 operands of the affine map for one group, with the range check of
// the prefill tiles: the scale exactly representable as fp16 (every bf16
// scale from 2^-17 to 65504 is, subnormals included, so the fma q*s + b
// rounds once, as for any normal scale), |bias| and |bias + (2^b - 1) scale|
// at most the fp16 maximum.
template <int BITS>
__device__ __forceinline__ void group_h2(uint32_t sbits, uint32_t bbits, __half2& s2, __half2& b2,
                                         int* status) {
  const float s = bf16_bits_to_float((uint16_t)sbits);
  const float b = bf16_bits_to_float((uint16_t)bbits);
  const float top = fabsf(b + (float)((1 << BITS) - 1) * s);
  const bool bad = __half2float(__float2half_rn(s)) != s || !(fabsf(b) <= 65504.0f) ||
                   !(top <= 65504.0f);
  if (bad) set_status(status, MOEQ_ERR_RANGE);
  s2 = __float2half2_rn(s);
  b2 = __float2half2_rn(b);
}

// MX FP4 group with E8M0 byte e, as the affine group of its codes q' = 2
// e2m1 + 12: s = 2^(e - 128), b = -12 s, both exact in fp16 for e in
// [102, 140] (the weights between 6 * 2^-25 and 6 * 2^13); other bytes
// are outside the prefill tiles' range (MOEQ_ERR_RANGE).
__device__ __forceinline__ void group_h2_mx(uint32_t e, __half2& s2, __half2& b2, int* status) {
  if (e < 102u || e > 140u) set_status(status, MOEQ_ERR_RANGE);
  const float s = __uint_as_float((e >= 1u ? e - 1u : 0u) << 23);  // 2^(e - 128)
  s2 = __float2half2_rn(s);
  b2 = __float2half2_rn(-12.0f * s);
}

// One 16-byte chunk of E2M1 codes (32 values, low nibble first) as two
// 16-byte chunks of 8-bit codes q' in value order (u0: values 0..15).
__device__ __forceinline__ void mx_chunk_q8(uint4 raw, uint4& u0, uint4& u1) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t n[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t lo = mx_q8(w[k] & 0x0F0F0F0Fu);         // values 8k + 0, 2, 4, 6
    const uint32_t hi = mx_q8((w[k] >> 4) & 0x0F0F0F0Fu);  // values 8k + 1, 3, 5, 7
    n[2 * k] = __byte_perm(lo, hi, 0x5140u);
    n[2 * k + 1] = __byte_perm(lo, hi, 0x7362u);
  }
  u0 = make_uint4(n[0], n[1], n[2], n[3]);
  u1 = make_uint4(n[4], n[5], n[6], n[7]);
}

// Dequantise one 16-byte chunk of packed codes into fp16 weights: 16 (8-bit),
// 32 (4-bit) or 64 (2-bit) values, written as 16-byte chunks starting at
// chunk `c16` of row `r` of the swizzled B stage.
template <int BITS>
__device__ __forceinline__ void dequant_chunk(uint4 raw, __half2 s2, __half2 b2, uint32_t bstage,
                                              int r, int c16) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  if (BITS == 8) {
    // codes q0..q15; half2 (1024 + q_j, 1024 + q_j+1) by byte permutes
    const __half2 k1024 = __float2half2_rn(1024.0f);
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 lo = __hsub2(u2h(__byte_perm(w[i], 0x64646464u, 0x4140)), k1024);
      const __half2 hi = __hsub2(u2h(__byte_perm(w[i], 0x64646464u, 0x4342)), k1024);
      o[2 * i] = h2u(__hfma2(lo, s2, b2));
      o[2 * i + 1] = h2u(__hfma2(hi, s2, b2));
    }
    sts128(bstage + tc::sw128_offset(r, c16), o[0], o[1], o[2], o[3]);
    sts128(bstage + tc::sw128_offset(r, c16 + 1), o[4], o[5], o[6], o[7]);
  } else if (BITS == 4) {
    // byte j holds q_2j (low nibble) and q_2j+1 (high nibble)
    const __half2 sc = __halves2half2(__float2half_rn(1.0f), __float2half_rn(1.0f / 16.0f));
    const __half2 of = __halves2half2(__float2half_rn(-1024.0f), __float2half_rn(-64.0f));
    uint32_t o[16];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t sel = 0x4040u | (uint32_t)j | ((uint32_t)j << 8);
        const uint32_t t = (__byte_perm(w[i], 0u, sel) & 0x00F0000Fu) | 0x64006400u;
        const __half2 q = __hfma2(u2h(t), sc, of);  // exact (q_lo, q_hi)
        o[4 * i + j] = h2u(__hfma2(q, s2, b2));
      }
#pragma unroll
    for (int k = 0; k < 4; ++k)
      sts128(bstage + tc::sw128_offset(r, c16 + k), o[4 * k], o[4 * k + 1], o[4 * k + 2],
             o[4 * k + 3]);
  } else {
    // byte j holds q_4j .. q_4j+3 in bit pairs
    const __half2 sc0 = __halves2half2(__float2half_rn(1.0f), __float2half_rn(0.25f));
    const __half2 of0 = __halves2half2(__float2half_rn(-1024.0f), __float2half_rn(-256.0f));
    const __half2 sc1 = __halves2half2(__float2half_rn(1.0f / 16.0f), __float2half_rn(1.0f / 64.0f));
    const __half2 of1 = __halves2half2(__float2half_rn(-64.0f), __float2half_rn(-16.0f));
    uint32_t o[32];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t sel = 0x4040u | (uint32_t)j | ((uint32_t)j << 8);
        const uint32_t t = __byte_perm(w[i], 0u, sel);
        const __half2 q01 = __hfma2(u2h((t & 0x000C0003u) | 0x64006400u), sc0, of0);
        const __half2 q23 = __hfma2(u2h((t & 0x00C00030u) | 0x64006400u), sc1, of1);
        o[8 * i + 2 * j] = h2u(__hfma2(q01, s2, b2));
        o[8 * i + 2 * j + 1] = h2u(__hfma2(q23, s2, b2));
      }
#pragma unroll
    for (int k = 0; k < 8; ++k)
      sts128(bstage + tc::sw128_offset(r, c16 + k), o[4 * k], o[4 * k + 1], o[4 * k + 2],
             o[4 * k + 3]);
  }
}

// (segment, first row within it) of m-tile mt; `rows` rows per m-tile
__device__ __forceinline__ int2 tile_of(const Args& a, int mt, int rows) {
  return a.tiles ? a.tiles[mt] : make_int2(0, mt * rows);
}

// Split dequantisation for the router tiles: w = fmaf(q, scale, bias) in
// fp32, written as fp16(w) (LO = false) or fp16(w - fp16(w)) (LO = true).
template <int BITS, bool LO>
__device__ __forceinline__ void dequant_chunk_split(uint4 raw, float s, float b, uint32_t bstage,
                                                    int r, int c16) {
  constexpr int VPC = 128 / BITS;
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t o[VPC / 2];
#pragma unroll
  for (int i = 0; i < VPC / 2; ++i) {
    float v[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int k = 2 * i + j;  // value index within the chunk
      const int word = k / (32 / BITS), pos = k % (32 / BITS);
      const uint32_t q = (w[word] >> (BITS * pos)) & ((1u << BITS) - 1u);
      const float wf = __fmaf_rn((float)q, s, b);
      const float hi = __half2float(__float2half_rn(wf));
      v[j] = LO ? wf - hi : wf;
    }
    o[i] = h2u(__floats2half2_rn(v[0], v[1]));
  }
#pragma unroll
  for (int k = 0; k < VPC / 8; ++k)
    sts128(bstage + tc::sw128_offset(r, c16 + k), o[4 * k], o[4 * k + 1], o[4 * k + 2],
           o[4 * k + 3]);
}

// GS: the group size when fixed at compile time (64, the common case, with
// no group arithmetic left at run time), or 0 to take a.G (32 or 128).
template <int BITS, int EPI, bool PAIR, int GS, bool MX = false>
__global__ void __launch_bounds__(THREADS, 1) k_gqmm(const __grid_constant__ Args a) {
  const int G = GS ? GS : a.G;
  static_assert(!MX || (BITS == 4 && GS == 32 && EPI != EPI_SPLIT), "MX FP4: 4-bit, G 32");
  using SM = Smem<BITS, PAIR>;
  using RW = Raw<BITS>;
  constexpr int S1 = SM::S1, SR = SM::SR, S2 = SM::S2, BR = SM::BR;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = tc::smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::BAR_OFF);
  uint64_t* full_a = bars;               // S1, A loader -> MMA
  uint64_t* a_empty = bars + S1;         // S1, MMA -> A loader
  uint64_t* raw_full = bars + 2 * S1;    // SR, B loader -> dequant
  uint64_t* raw_empty = raw_full + SR;   // SR, dequant -> B loader
  uint64_t* b_full = raw_empty + SR;     // S2, dequant -> MMA
  uint64_t* b_empty = b_full + S2;       // S2, MMA -> dequant
  uint64_t* tmem_full = b_empty + S2;    // 2, MMA -> epilogue
  uint64_t* tmem_empty = tmem_full + 2;  // 2, epilogue -> MMA
  const __half** atab = reinterpret_cast<const __half**>(smem + SM::ATAB_OFF);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SM::TMEM_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // PAIR: the cluster's two CTAs share every work item; rank 0 issues the
  // MMAs, each CTA holds half of the A rows, half of the B rows and the
  // accumulator rows of its A half.  The barriers the MMA issuer waits on
  // (full_a, b_full, tmem_empty) are rank 0's; the others are per CTA.
  const uint32_t rank = PAIR ? tc::cluster_ctarank() : 0u;
  const int unit0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int n_units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  if (threadIdx.x == 0) {
    for (int i = 0; i < S1; ++i) {
      tc::mbar_init(&full_a[i], PAIR ? 1 : 64);
      tc::mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < SR; ++i) {
      tc::mbar_init(&raw_full[i], 32);
      tc::mbar_init(&raw_empty[i], DQ_WARPS * 32);
    }
    for (int i = 0; i < S2; ++i) {
      tc::mbar_init(&b_full[i], PAIR ? 2 * DQ_WARPS : DQ_WARPS * 32);
      tc::mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&tmem_full[i], 1);
      tc::mbar_init(&tmem_empty[i], PAIR ? 256 : 128);
    }
    tc::fence_mbar_init();
  }
  if (warp == 3) {
    if (PAIR) {
      tc::tmem_alloc_pair(tmem_holder, 512);
      tc::tmem_relinquish_pair();
    } else {
      tc::tmem_alloc(tmem_holder, 512);
      tc::tmem_relinquish();
    }
  }
  tc::tc_fence_before();
  if (PAIR) tc::cluster_sync();
  else __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int n_items = (a.tiles ? *a.n_tiles : a.static_mtiles) * a.n_tiles_n;
  const int KB = a.K / BK;
  int* status = a.status;

  if (warp < 2 && PAIR) {
    // ------------------------------------------------------------ A loader (pair)
    // warp 0: lane 0 of each CTA fetches its 128 rows per stage; rank 0's
    // stage barrier expects both CTAs' bytes (warp 1 idles)
    if (warp == 0) {
      uint32_t it = 0;
      for (int item = unit0; item < n_items; item += n_units) {
        const int2 tile = tile_of(a, item / a.n_tiles_n, PAIR ? 2 * BM : BM);
        const Seg& sg = a.tiles ? a.segs[tile.x] : a.seg0;
        const int row0 =
            (sg.a_mode == A_TOKENS ? 0 : sg.row_begin) + tile.y + (int)rank * BM;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const uint32_t s = it % S1, ph = (it / S1) & 1u;
          if (!tc::mbar_wait(&a_empty[s], ph ^ 1u, status)) goto done;
          if (lane == 0) {
            if (rank == 0) tc::mbar_arrive_expect_tx(&full_a[s], (uint32_t)(2 * A_STAGE));
            tc::tma_load_2d_pair(sbase + SM::A_OFF + s * A_STAGE, &a.tmA, kb * BK, row0,
                                 tc::mapa_shared(tc::smem_u32(&full_a[s]), 0));
          }
          __syncwarp();
        }
      }
      // every release of this CTA's stages has landed before it may exit
      for (int j = 0; j < S1; ++j, ++it)
        if (!tc::mbar_wait(&a_empty[it % S1], ((it / S1) & 1u) ^ 1u, status)) goto done;
    }
  } else if (warp < 2 && a.tma_a) {
    // ------------------------------------------------------------ A loader (tensor map)
    // thread 0 issues one 128-row x 64-column tile per stage; the other 63
    // threads arrive so the stage barrier keeps its count of 64
    uint32_t it = 0;
    for (int item = unit0; item < n_items; item += n_units) {
      const int2 tile = tile_of(a, item / a.n_tiles_n, PAIR ? 2 * BM : BM);
      const Seg& sg = a.tiles ? a.segs[tile.x] : a.seg0;
      const int row0 = sg.a_mode == A_TOKENS ? tile.y : sg.row_begin + tile.y;
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const uint32_t s = it % S1, ph = (it / S1) & 1u;
        if (!tc::mbar_wait(&a_empty[s], ph ^ 1u, status)) goto done;
        if (threadIdx.x == 0) {
          tc::mbar_arrive_expect_tx(&full_a[s], (uint32_t)A_STAGE);
          tc::tma_load_2d(sbase + SM::A_OFF + s * A_STAGE, &a.tmA, kb * BK, row0, &full_a[s]);
        } else {
          tc::mbar_arrive(&full_a[s]);
        }
      }
    }
  } else if (warp < 2) {
    // ------------------------------------------------------------ A loader
    // 64 threads; the 1024 16-byte chunks of a stage are spread so that each
    // group of 8 lanes writes the 8 chunks of one row (conflict-free).
    const int t = threadIdx.x;
    bool dead = false;
    uint32_t it = 0, tl = 0;
    for (int item = unit0; item < n_items; item += n_units, ++tl) {
      const int2 tile = tile_of(a, item / a.n_tiles_n, PAIR ? 2 * BM : BM);
      const Seg& sg = a.tiles ? a.segs[tile.x] : a.seg0;
      const __half** tab = atab + (tl & 1) * BM;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int i = 2 * t + j;
        const bool ok = tile.y + i < sg.rows;
        const int64_t m = (int64_t)sg.row_begin + tile.y + i;
        const __half* p = nullptr;
        if (ok) {
          int64_t arow;
          if (sg.a_mode == A_PAIRS) arow = a.sorted_pair[m] / a.topk;
          else if (sg.a_mode == A_TOKENS) arow = tile.y + i;
          else arow = m;
          p = a.A + arow * a.lda;
        }
        tab[i] = p;
      }
      tc::named_sync(2, 64);
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const uint32_t s = it % S1, ph = (it / S1) & 1u;
        // after a wait that ran out both loader warps keep walking the items
        // (no copies) so they meet at every named barrier
        if (!dead) dead = !tc::mbar_wait(&a_empty[s], ph ^ 1u, status);
        if (dead) continue;
        const uint32_t st = sbase + SM::A_OFF + s * A_STAGE;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int q = t + 64 * i;
          const int row = q >> 3, c = q & 7;
          const __half* p = tab[row];
          tc::cp_async16(st + tc::sw128_offset(row, c), p ? p + kb * BK + c * 8 : a.A,
                         p ? 16u : 0u);
        }
        tc::cp_async_arrive_noinc(&full_a[s]);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ B loader
    // this CTA's BR weight rows of the tile: rows rank*BR + (lane + 32 j)
    const int groups = a.K / G;
    const int W = a.sb_w, wl = win_kb_log2(W, G);
    const int64_t wrow = (int64_t)a.K * BITS / 32;  // words per weight row
    constexpr int JR = BR / 32;
    uint32_t it = 0;
    for (int item = unit0; item < n_items; item += n_units) {
      const int2 tile = tile_of(a, item / a.n_tiles_n, PAIR ? 2 * BM : BM);
      const int nt = item % a.n_tiles_n;
      const Seg& sg = a.tiles ? a.segs[tile.x] : a.seg0;
      const uint32_t* wp[JR];
      const uint16_t* sp[JR];
      const uint16_t* bp[JR];
      uint32_t ok16[JR];
#pragma unroll
      for (int j = 0; j < JR; ++j) {
        const int r = (int)rank * BR + lane + 32 * j;
        int src, q;
        bool ok;
        b_row<EPI>(sg, nt, r, src, q, ok);
        if (!ok) q = 0;
        wp[j] = sg.w[src] + (int64_t)q * wrow;
        // (MX FP4: one exponent byte per group, no biases)
        sp[j] = MX ? reinterpret_cast<const uint16_t*>(
                         reinterpret_cast<const uint8_t*>(sg.s[src]) + (int64_t)q * groups)
                   : sg.s[src] + (int64_t)q * groups;
        bp[j] = MX ? nullptr : sg.b[src] + (int64_t)q * groups;
        ok16[j] = ok ? 16u : 0u;
      }
      // tensor-map halves: (source, first row) of tile rows 0..127 and 128..255
      const int src1 = EPI == EPI_SWIGLU ? 1 : 0;
      const int y0 = EPI == EPI_SWIGLU ? nt * 128 : nt * BN;
      const int y1 = EPI == EPI_SWIGLU ? nt * 128 : nt * BN + 128;
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const uint32_t s = it % SR, ph = (it / SR) & 1u;
        if (!tc::mbar_wait(&raw_empty[s], ph ^ 1u, status)) goto done;
        const uint32_t rst = sbase + SM::RAW_OFF + s * SM::RAW_STAGE;
        // a new scale/bias window (W groups) every 2^wl k-blocks (windows
        // counted over the whole item loop, like the dequantiser); its
        // first group is group kb * 64 / G of the row
        const bool new_win = (kb & ((1 << wl) - 1)) == 0;
        const uint32_t sbw = sbase + SM::SB_OFF + ((it >> wl) % SM::NWB) * SM::SB_WIN;
        const int g0 = G == 64 ? kb : G == 128 ? kb >> 1 : kb << 1;
        if (a.tma_b) {
          if (lane == 0) {
            tc::mbar_expect_tx(&raw_full[s], (uint32_t)SM::RAW_STAGE);
            if (PAIR) {
              const int src = rank ? src1 : 0;
              tc::tma_load_3d(rst, &a.tmB[src], kb * (RW::ROW / 4), rank ? y1 : y0, sg.ex[src],
                              &raw_full[s]);
            } else {
              tc::tma_load_3d(rst, &a.tmB[0], kb * (RW::ROW / 4), y0, sg.ex[0], &raw_full[s]);
              tc::tma_load_3d(rst + 128 * RW::ROW, &a.tmB[src1], kb * (RW::ROW / 4), y1,
                              sg.ex[src1], &raw_full[s]);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < JR; ++j) {
            const int r = lane + 32 * j;
#pragma unroll
            for (int c = 0; c < RW::CHUNKS; ++c)
              tc::cp_async16(rst + RW::offset(r, c), wp[j] + kb * (RW::ROW / 4) + c * 4, ok16[j]);
          }
        }
        if (new_win) {
#pragma unroll
          for (int j = 0; j < JR; ++j) {
            const int r = lane + 32 * j;
            const uint32_t d = sbw + r * 32;
            if (MX) {
              const uint8_t* e0 = reinterpret_cast<const uint8_t*>(sp[j]) + g0;
              if (W == 8) tc::cp_async8(d, e0, ok16[j] ? 8u : 0u);
              else tc::cp_async4(d, e0, ok16[j] ? 4u : 0u);
            } else if (W == 8) {
              tc::cp_async16(d, sp[j] + g0, ok16[j]);
              tc::cp_async16(d + 16, bp[j] + g0, ok16[j]);
            } else if (W == 4) {
              tc::cp_async8(d, sp[j] + g0, ok16[j] ? 8u : 0u);
              tc::cp_async8(d + 16, bp[j] + g0, ok16[j] ? 8u : 0u);
            } else {
              tc::cp_async4(d, sp[j] + g0, ok16[j] ? 4u : 0u);
              tc::cp_async4(d + 16, bp[j] + g0, ok16[j] ? 4u : 0u);
            }
          }
        }
        tc::cp_async_arrive_noinc(&raw_full[s]);
      }
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ MMA issuer
    if (!PAIR || rank == 0) {
      uint32_t it = 0, tcount = 0;
      for (int item = unit0; item < n_items; item += n_units, ++tcount) {
        const uint32_t acc = tcount & 1u, acc_ph = (tcount >> 1) & 1u;
        if (!tc::mbar_wait(&tmem_empty[acc], acc_ph ^ 1u, status)) goto done;
        tc::tc_fence_after();
        const uint32_t d = tmem_base + acc * 256u;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const uint32_t s1 = it % S1, ph1 = (it / S1) & 1u;
          const uint32_t s2 = it % S2, ph2 = (it / S2) & 1u;
          if (!tc::mbar_wait(&full_a[s1], ph1, status)) goto done;
          if (!tc::mbar_wait(&b_full[s2], ph2, status)) goto done;
          // the dequantisers fenced their shared-memory writes to the async
          // proxy before arriving on b_full
          tc::tc_fence_after();
          if (lane == 0) {
            const uint32_t aa = sbase + SM::A_OFF + s1 * A_STAGE;
            const uint32_t ba = sbase + SM::B_OFF + s2 * SM::B_STAGE;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              if (PAIR)
                tc::mma_f16_pair(d, tc::sw128_kmajor_desc(aa + kk * 32),
                                 tc::sw128_kmajor_desc(ba + kk * 32), SM::IDESC, (kb | kk) != 0);
              else
                tc::mma_f16(d, tc::sw128_kmajor_desc(aa + kk * 32),
                            tc::sw128_kmajor_desc(ba + kk * 32), SM::IDESC, (kb | kk) != 0);
            }
            if (PAIR) {
              tc::mma_commit_pair(&a_empty[s1], 3);
              tc::mma_commit_pair(&b_empty[s2], 3);
            } else {
              tc::mma_commit(&a_empty[s1]);
              tc::mma_commit(&b_empty[s2]);
            }
          }
          __syncwarp();
        }
        if (lane == 0) {
          if (PAIR) tc::mma_commit_pair(&tmem_full[acc], 3);
          else tc::mma_commit(&tmem_full[acc]);
        }
        __syncwarp();
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int i = q * 32 + lane;  // accumulator row of this CTA = TMEM lane
    uint32_t tcount = 0;
    for (int item = unit0; item < n_items; item += n_units, ++tcount) {
      const int2 tile = tile_of(a, item / a.n_tiles_n, PAIR ? 2 * BM : BM);
      const int nt = item % a.n_tiles_n;
      const Seg& sg = a.tiles ? a.segs[tile.x] : a.seg0;
      const uint32_t acc = tcount & 1u, acc_ph = (tcount >> 1) & 1u;
      if (!tc::mbar_wait(&tmem_full[acc], acc_ph, status)) goto done;
      tc::tc_fence_after();
      const int ty = tile.y + (int)rank * BM + i;  // row within the segment
      const bool ok = ty < sg.rows;
      const int64_t m = (int64_t)sg.row_begin + ty;
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * 256u;
      if (EPI == EPI_SWIGLU) {
        __half* out = reinterpret_cast<__half*>(a.out) + m * a.ldo + nt * 128;
        bool bad = false;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t g[32], u[32];
          tc::tmem_ld32(tb + c0, g);
          tc::tmem_ld32(tb + 128 + c0, u);
          tc::tmem_wait_ld();
          if (ok && nt * 128 + c0 < sg.n0) {
            uint32_t o[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const float g0 = __uint_as_float(g[2 * k]), g1 = __uint_as_float(g[2 * k + 1]);
              const float h0 = __fdividef(g0, 1.0f + __expf(-g0)) * __uint_as_float(u[2 * k]);
              const float h1 = __fdividef(g1, 1.0f + __expf(-g1)) * __uint_as_float(u[2 * k + 1]);
              bad |= !(fabsf(h0) <= 65504.0f) || !(fabsf(h1) <= 65504.0f);
              o[k] = h2u(__floats2half2_rn(h0, h1));
            }
            if ((((uintptr_t)(out + c0)) & 31) == 0) {
              stg256(out + c0, o[0], o[1], o[2], o[3], o[4], o[5], o[6], o[7]);
              stg256(out + c0 + 16, o[8], o[9], o[10], o[11], o[12], o[13], o[14], o[15]);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(out + c0);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                dst[k] = make_uint4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
            }
          }
        }
        if (bad) set_status(status, MOEQ_ERR_RANGE);
      } else if (EPI == EPI_SPLIT) {
        float* out = reinterpret_cast<float*>(a.out) + m * a.ldo + nt * 128;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t hv[32], lv[32];
          tc::tmem_ld32(tb + c0, hv);
          tc::tmem_ld32(tb + 128 + c0, lv);
          tc::tmem_wait_ld();
          const int col = nt * 128 + c0;
          if (ok && col < sg.n_valid) {
            const int nv = min(32, sg.n_valid - col);
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (k < nv) out[c0 + k] = __uint_as_float(hv[k]) + __uint_as_float(lv[k]);
          }
        }
      } else if (a.out_f16) {
        int64_t dest = m;
        if (ok && sg.dest_pairs) dest = a.sorted_pair[m];
        __half* out = reinterpret_cast<__half*>(a.out) + dest * a.ldo + nt * BN;
        bool bad = false;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t v[32];
          tc::tmem_ld32(tb + c0, v);
          tc::tmem_wait_ld();
          const int col = nt * BN + c0;
          if (ok && col < sg.n_valid) {
            uint32_t o[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const float f0 = __uint_as_float(v[2 * k]), f1 = __uint_as_float(v[2 * k + 1]);
              bad |= !(fabsf(f0) <= 65504.0f) || !(fabsf(f1) <= 65504.0f);
              o[k] = h2u(__floats2half2_rn(f0, f1));
            }
            if (col + 32 <= sg.n_valid && (((uintptr_t)(out + c0)) & 31) == 0) {
              stg256(out + c0, o[0], o[1], o[2], o[3], o[4], o[5], o[6], o[7]);
              stg256(out + c0 + 16, o[8], o[9], o[10], o[11], o[12], o[13], o[14], o[15]);
            } else {
              const int nv = min(32, sg.n_valid - col);
#pragma unroll
              for (int k = 0; k < 32; ++k)
                if (k < nv) out[c0 + k] = __float2half_rn(__uint_as_float(v[k]));
            }
          }
        }
        if (bad) set_status(status, MOEQ_ERR_RANGE);
      } else {
        int64_t dest = m;
        if (ok && sg.dest_pairs) dest = a.sorted_pair[m];
        float* out = reinterpret_cast<float*>(a.out) + dest * a.ldo + nt * BN;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t v[32];
          tc::tmem_ld32(tb + c0, v);
          tc::tmem_wait_ld();
          const int col = nt * BN + c0;
          if (ok && col < sg.n_valid) {
            if (col + 32 <= sg.n_valid && (((uintptr_t)(out + c0)) & 31) == 0) {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                stg256(out + c0 + 8 * k, v[8 * k], v[8 * k + 1], v[8 * k + 2], v[8 * k + 3],
                       v[8 * k + 4], v[8 * k + 5], v[8 * k + 6], v[8 * k + 7]);
            } else if (col + 32 <= sg.n_valid && (((uintptr_t)(out + c0)) & 15) == 0) {
              uint4* dst = reinterpret_cast<uint4*>(out + c0);
#pragma unroll
              for (int k = 0; k < 8; ++k)
                dst[k] = make_uint4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
            } else {
              const int nv = min(32, sg.n_valid - col);
#pragma unroll
              for (int k = 0; k < 32; ++k)
                if (k < nv) out[c0 + k] = __uint_as_float(v[k]);
            }
          }
        }
      }
      tc::tc_fence_before();
      if (PAIR) tc::mbar_arrive_cluster(tc::mapa_shared(tc::smem_u32(&tmem_empty[acc]), 0));
      else tc::mbar_arrive(&tmem_empty[acc]);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ dequantiser
    // one weight row per thread, or (PAIR: 128 rows per CTA) half a row
    const int t = threadIdx.x - 256;
    const int r = PAIR ? (t & 127) : t;            // row of this CTA's stages
    const int rg = (int)rank * BR + r;             // row of the 256-row tile
    constexpr int CPT = PAIR ? (RW::CHUNKS > 1 ? RW::CHUNKS / 2 : 1) : RW::CHUNKS;
    const int c_lo = PAIR ? (t >> 7) * CPT : 0;   // first raw chunk of this thread
    const bool active = c_lo < RW::CHUNKS;
    const int W = a.sb_w, wl = win_kb_log2(W, G);
    uint4 swin = make_uint4(0u, 0u, 0u, 0u), bwin = swin;  // scale/bias window (bf16 pairs)
    // scale and bias bits of group j of the window
    auto pick = [&](int j, uint32_t& sbits, uint32_t& bbits) {
      const uint32_t sw2 = (j & 4) ? ((j & 2) ? swin.w : swin.z) : ((j & 2) ? swin.y : swin.x);
      const uint32_t bw2 = (j & 4) ? ((j & 2) ? bwin.w : bwin.z) : ((j & 2) ? bwin.y : bwin.x);
      sbits = (j & 1) ? (sw2 >> 16) : (sw2 & 0xFFFFu);
      bbits = (j & 1) ? (bw2 >> 16) : (bw2 & 0xFFFFu);
    };
    constexpr int VPC = 128 / BITS;  // values of one 16-byte code chunk
    uint32_t it = 0;
    for (int item = unit0; item < n_items; item += n_units) {
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const uint32_t sr = it % SR, phr = (it / SR) & 1u;
        const uint32_t s2 = it % S2, ph2 = (it / S2) & 1u;
        if (!tc::mbar_wait(&raw_full[sr], phr, status)) goto done;
        if (!tc::mbar_wait(&b_empty[s2], ph2 ^ 1u, status)) goto done;
        const uint32_t rst = sbase + SM::RAW_OFF + sr * SM::RAW_STAGE;
        const uint32_t bst = sbase + SM::B_OFF + s2 * SM::B_STAGE;
        const int kbw = kb & ((1 << wl) - 1);  // k-block within the window
        if (kbw == 0) {
          // this row's window of W scales and W biases, kept in registers
          const uint32_t sbw =
              sbase + SM::SB_OFF + ((it >> wl) % SM::NWB) * SM::SB_WIN + r * 32;
          if (MX) {
            // W exponent bytes: groups 0..3 in swin.x, 4..7 in swin.y
            swin = W == 8 ? make_uint4(lds64(sbw).x, lds64(sbw).y, 0u, 0u)
                          : make_uint4(lds32(sbw), 0u, 0u, 0u);
          } else if (W == 8) {
            swin = lds128(sbw);
            bwin = lds128(sbw + 16);
          } else if (W == 4) {
            const uint2 sv = lds64(sbw), bv = lds64(sbw + 16);
            swin = make_uint4(sv.x, sv.y, 0u, 0u);
            bwin = make_uint4(bv.x, bv.y, 0u, 0u);
          } else {
            swin = make_uint4(lds32(sbw), 0u, 0u, 0u);
            bwin = make_uint4(lds32(sbw + 16), 0u, 0u, 0u);
          }
        }
        // group of chunk c: value kbw * 64 + c * VPC of the window, over G
        uint32_t sbits, bbits;
        pick(G == 64 ? kbw : G == 128 ? kbw >> 1 : 2 * kbw + (c_lo * VPC >= 32), sbits, bbits);
        uint4 raw[CPT];
#pragma unroll
        for (int c = 0; c < CPT; ++c)
          raw[c] = active ? lds128(rst + RW::offset(r, c_lo + c)) : make_uint4(0, 0, 0, 0);
        tc::mbar_arrive(&raw_empty[sr]);
        if (active) {
          // packed chunk c holds values [c*128/BITS, (c+1)*128/BITS): fp16 chunk c*16/BITS
          // G = 32 (8- and 4-bit only): chunks of one thread may fall in
          // both groups of the k-block
          const bool per_chunk = G == 32 && CPT > 1;
          if (MX) {
            // exponent byte of group j of the window: byte j % 4 of word j / 4
            auto ebyte = [&](int j) { return ((j < 4 ? swin.x : swin.y) >> (8 * (j & 3))) & 255u; };
            const int j0 = 2 * kbw + (c_lo * VPC >= 32);
            __half2 s2h, b2h;
            group_h2_mx(ebyte(j0), s2h, b2h, status);
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
              if (per_chunk && (c_lo + c) * VPC >= 32 && c_lo * VPC < 32)
                group_h2_mx(ebyte(2 * kbw + 1), s2h, b2h, status);
              uint4 u0, u1;
              mx_chunk_q8(raw[c], u0, u1);
              dequant_chunk<8>(u0, s2h, b2h, bst, r, (c_lo + c) * 4);
              dequant_chunk<8>(u1, s2h, b2h, bst, r, (c_lo + c) * 4 + 2);
            }
          } else if (EPI == EPI_SPLIT) {
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
              uint32_t sb = sbits, bb = bbits;
              if (per_chunk) pick(2 * kbw + ((c_lo + c) * VPC >= 32), sb, bb);
              const float sf = bf16_bits_to_float((uint16_t)sb);
              const float bf = bf16_bits_to_float((uint16_t)bb);
              if (rg < 128)
                dequant_chunk_split<BITS, false>(raw[c], sf, bf, bst, r, (c_lo + c) * (16 / BITS));
              else
                dequant_chunk_split<BITS, true>(raw[c], sf, bf, bst, r, (c_lo + c) * (16 / BITS));
            }
          } else {
            __half2 s2h, b2h;
            group_h2<BITS>(sbits, bbits, s2h, b2h, status);
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
              if (per_chunk && (c_lo + c) * VPC >= 32 && c_lo * VPC < 32) {
                uint32_t sb, bb;
                pick(2 * kbw + 1, sb, bb);
                group_h2<BITS>(sb, bb, s2h, b2h, status);
              }
              dequant_chunk<BITS>(raw[c], s2h, b2h, bst, r, (c_lo + c) * (16 / BITS));
            }
          }
        }
        tc::fence_proxy_async_smem();
        if (PAIR) {
          __syncwarp();
          if (lane == 0) tc::mbar_arrive_cluster(tc::mapa_shared(tc::smem_u32(&b_full[s2]), 0));
        } else {
          tc::mbar_arrive(&b_full[s2]);
        }
      }
    }
    if (PAIR)
      for (int j = 0; j < S2; ++j, ++it)
        if (!tc::mbar_wait(&b_empty[it % S2], ((it / S2) & 1u) ^ 1u, status)) goto done;
  }
done:
  tc::tc_fence_before();
  if (PAIR) tc::cluster_sync();
  else __syncthreads();
  if (warp == 3) {
    tc::tc_fence_after();
    if (PAIR) tc::tmem_dealloc_pair(tmem_base, 512);
    else tc::tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace gq
}  // namespace moeq
