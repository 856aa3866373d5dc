// Single-token decode of the whole layer in one launch (HBM-bound).
//
// Sources: "markbaseengine/MOE_ROUTER_WORKS_BREAKTHROUGH.md", Forward Pass
// Sequence (router -> softmax/top-K -> experts -> combine);
// "flash-moe-inference", per-layer pipeline, matvec_4bit_fma, swiglu and
// moe_combine_residual listings (the group form of the fma(q, scale*x,
// bias*x) factoring, SwiGLU of the gate half, the sigmoid-gated shared
// expert).
//
// Work split.  One CTA per SM; every CTA owns balanced contiguous ranges of
// router rows, shared-expert intermediate indices, routed intermediate
// indices (expert-major over the K selected experts) and output rows of the
// down projections -- the same output rows for the shared expert and every
// routed expert, so a CTA combines its rows with no cross-CTA reduction.
// Ranges are cut into units: 4 router rows (the shared-gate row is a unit of
// its own on the last CTA), 8 gate/up indices (a gate box and an up box),
// 8 down rows.
//
// Arithmetic.  Each input vector (the token, the hidden vectors) is turned
// into a table of block fixed point: per group of 64 values (the weights'
// scale/bias group) a power-of-two scale xs, and every value as an integer
// of at most 22 bits written as three signed byte limbs X = L0 + 256 L1 +
// 65536 L2.  For one group and one row, sum_c q_c X_c is an exact integer:
// an mma.sync m16n8k32 (u8 codes x s8 limbs, s32 accumulate) takes 16 tile
// rows by 32 inputs against the three limb columns, and the group's value is
// scale * xs * (sum over limbs) + bias * xs * sum_c X_c.  The integer MMA
// serves as a wide integer dot-product instruction (one instruction and a
// few unpacking operations per 16 rows x 32 inputs, where byte-wise dp4a
// needs about 1.7 instructions per weight and made the SM, not HBM, the
// bound).  Input order inside a 32-value block follows the code packing (the
// MMA sums over k, so any common order of codes and limbs is exact): 4-bit
// words give their even then odd nibbles, 2-bit words their bit planes.
//
// Stream.  A producer warp loads each unit with one tensor-map copy per box:
// a 4-D map (slab words, row, slab, matrix) whose box overhangs the slab by
// 16 bytes, so the copy itself writes every (slab, row) at a padded stride
// (the overhang reads as zeros, nothing extra is fetched) and the MMA
// fragment reads are bank-conflict free; each box's scale and bias rows
// come the same way (3-D maps, rows padded by 8 entries).  Units stream
// through a 4-stage ring.  The 16 compute warps take one unit at a time
// together, each a contiguous run of the unit's groups, then sum their
// partial row values in warp order (deterministic).
//
// Phases: (1) before the dependency wait the producer streams the units of
// weights that do not depend on the routing (router, shared gate, shared
// gate/up, shared down); (2) the compute warps build the token tables,
// compute router logits, the shared gate logit and the shared hidden values,
// publish them and raise this CTA's flag in the first flag array; (3) the
// producer waits until every CTA's first flag carries this call's tag,
// selects the top K (one warp), pulls the CTA's routed bytes into L2
// (gate/up first, then down) and streams the routed units; the compute warps
// run the shared down rows and the routed gate/up + SwiGLU units, publish
// the hidden values and raise the second flag; (4) once every second flag
// carries the tag, they build the K hidden tables, run the routed down rows
// and write y[r] = sigma * shared[r] + sum_k w_k d_k[r] (+ residual[r]), k in
// order.
//
// Flags are 64-bit tags, so the workspace needs no clearing: workspace word
// 0 holds the previous call's tag, this call's tag is a fixed bijective mix
// of it, and CTA 0 stores it back at the end.  A stale flag holds an earlier
// tag of the chain or unrelated data, neither of which equals the new tag
// except with probability ~2^-64.
//
// Waits sleep in hardware (mbarrier try_wait with a suspend time) and are
// bounded (about two seconds); one that runs out sets MOEQ_ERR_TIMEOUT in
// the status word, and the CTA skips its remaining work after its copies in
// flight have landed.
#include <cudaTypedefs.h>
#include <string.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "route.cuh"
#include "tc.cuh"

namespace moeq {

namespace {

constexpr int FZ_CW = 16;                    // compute warps
constexpr int FZ_PROD = FZ_CW;               // producer warp index
constexpr int FZ_CT = FZ_CW * 32;            // compute threads
constexpr int FZ_THREADS = FZ_CT + 32;
constexpr int FZ_NS = 4;                     // ring stages
constexpr int FZ_UMAX = 96;                  // units per CTA
constexpr int FZ_BAR_C = 1;                  // named barrier: compute warps
constexpr int FZ_SMEM_MAX = 227 * 1024;      // the per-CTA limit (at most ~110 KB lets two CTAs share an SM)
constexpr int FZ_G = 64;                     // group size of every tensor on this path

struct FzUnit {
  int32_t r0;
  int16_t n;   // rows (indices for gate/up units)
  int8_t kind;
  int8_t k;    // expert slot of routed units
};

// ------------------------------------------------------------------ small helpers
__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
__device__ __forceinline__ int ld_vol(const int* p) { return *reinterpret_cast<const volatile int*>(p); }
__device__ __forceinline__ void mark_dead(int* p) { *reinterpret_cast<volatile int*>(p) = 1; }

// D += A * B: 16x32 unsigned byte codes times 32x8 signed byte limbs.
__device__ __forceinline__ void imma(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four-dimensional tensor-map tile load into this CTA's shared memory,
// completing on `bar` by transaction bytes (no multicast).
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const void* tmap, int x, int y, int z,
                                            int w, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(w), "r"(tc::smem_u32(bar))
      : "memory");
}

// This call's tag from the previous call's (a bijection of 64-bit words:
// an odd-multiplier affine step followed by an xor-shift).
__device__ __forceinline__ uint64_t next_tag(uint64_t g) {
  const uint64_t t = g * 0xD1342543DE82EF95ull + 0x2545F4914F6CDD1Dull;
  return t ^ (t >> 29);
}

__host__ __device__ inline int imin(int a, int b) { return a < b ? a : b; }

// Balanced range of n items (n a multiple of gran) for CTA c of P.
__host__ __device__ inline void fz_range(int n, int gran, int c, int P, int& lo, int& hi) {
  const int nu = n / gran;
  lo = (int)((int64_t)nu * c / P) * gran;
  hi = (int)((int64_t)nu * (c + 1) / P) * gran;
}

// The CTA's units in issue order: phase 1 (router rows, the shared-gate row
// on the last CTA, shared gate/up), then phase 3 (shared down, routed
// gate/up), then phase 4 (routed down).  Returns the count; n1, n3 the
// counts of phases 1 and 3.
__host__ __device__ inline int fz_units(const FusedArgs& a, int c, int P, FzUnit* T, int cap,
                                        int* n1, int* n3) {
  int u = 0;
  auto add = [&](int r0, int n, int kind, int k) {
    if (T && u < cap) {
      T[u].r0 = r0;
      T[u].n = (int16_t)n;
      T[u].kind = (int8_t)kind;
      T[u].k = (int8_t)k;
    }
    ++u;
  };
  auto ranged = [&](int n_items, int kind, int k, int lo_hi_of) {
    int lo, hi;
    fz_range(n_items, a.kind[lo_hi_of].gran, c, P, lo, hi);
    const int rb = a.kind[kind].RB;
    for (int r = lo; r < hi; r += rb) add(r, imin(rb, hi - r), kind, k);
  };
  if (a.route_from_router) ranged(a.E, FZ_ROUTER, 0, FZ_ROUTER);
  if (a.has_shared) {
    if (c == P - 1) add(0, 1, FZ_SGATE, 0);
    ranged(a.Ish, FZ_SHGU, 0, FZ_SHGU);
  }
  *n1 = u;
  if (a.has_shared) ranged(a.H, FZ_SHDN, 0, FZ_DN);
  {
    int lo, hi;
    fz_range(a.K * a.I, a.kind[FZ_GU].gran, c, P, lo, hi);
    for (int q = lo; q < hi;) {
      const int k = q / a.I, i = q % a.I;
      const int n = imin(a.kind[FZ_GU].RB, imin(hi - q, a.I - i));
      add(i, n, FZ_GU, k);
      q += n;
    }
  }
  *n3 = u - *n1;
  for (int k = 0; k < a.K; ++k) ranged(a.H, FZ_DN, k, FZ_DN);
  return u;
}

// Tile row m of a unit: whether it holds a weight row, in which box and at
// which box row.  Gate/up units: gate box rows in tile rows 0..7, up box rows
// in 8..15; the others: box 0 rows in tile rows 0..15.
__host__ __device__ inline bool tile_row(const FzUnit& u, int m, int& box, int& r) {
  if (u.kind == FZ_SHGU || u.kind == FZ_GU) {
    box = m >> 3;
    r = m & 7;
  } else {
    box = 0;
    r = m;
  }
  return r < u.n;
}

__host__ __device__ inline const moeq_qtensor& unit_tensor(const FusedArgs& a, const FzUnit& u,
                                                           int box) {
  switch (u.kind) {
    case FZ_ROUTER: return a.router;
    case FZ_SGATE: return a.sgate;
    case FZ_SHGU: return box ? a.sh_up : a.sh_gate;
    case FZ_SHDN: return a.sh_down;
    case FZ_GU: return box ? a.up : a.gate;
    default: return a.down;
  }
}

__host__ __device__ inline int unit_map(const FzUnit& u, int box) {
  switch (u.kind) {
    case FZ_ROUTER: return FZM_ROUTER;
    case FZ_SGATE: return FZM_SGATE;
    case FZ_SHGU: return box ? FZM_SHU : FZM_SHG;
    case FZ_SHDN: return FZM_SHD;
    case FZ_GU: return box ? FZM_U : FZM_G;
    default: return FZM_D;
  }
}

// ------------------------------------------------------------------ input tables
// Value order inside a 32-value block: MMA index kappa = 4q + j (q: the
// quarter a lane's register holds, j: its byte) -> position of the value.
template <int BITS>
__host__ __device__ constexpr int kappa_pos(int q, int j) {
  return BITS == 8 ? 4 * q + j
       : BITS == 4 ? (q < 4 ? 8 * q + 2 * j : 8 * (q - 4) + 2 * j + 1)
                   : (q < 4 ? q + 4 * j : 16 + (q - 4) + 4 * j);
}

// Table of a vector of len values: per 32-value block 3 limb columns x 8
// quarter words (96 bytes), then per group of 64 values (xs, xs * sum X).
// One lane per 32-value block; the two lanes of a group (aligned,
// consecutive) share its scale.
template <bool F32>
__device__ __forceinline__ void load_block(const void* src, int64_t off, bool on, float (&xv)[32]) {
  if (!on) {
#pragma unroll
    for (int i = 0; i < 32; ++i) xv[i] = 0.0f;
    return;
  }
  if (F32) {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(src) + off);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 q = __ldcg(p + i);
      xv[4 * i] = q.x;
      xv[4 * i + 1] = q.y;
      xv[4 * i + 2] = q.z;
      xv[4 * i + 3] = q.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(src) + off);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 q = p[i];
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        xv[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
        xv[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
      }
    }
  }
}

// Block fixed point of a lane's 32 values, the scale shared with the other
// lane of its 64-value group (all lanes of the warp call): X = rint(x * 2^k),
// |X| < 2^22, returned as its three signed byte limbs in natural value order
// (L[l][i / 4] byte i % 4 = limb l of value i).
__device__ __forceinline__ void quantize_block(const float (&xv)[32], uint32_t (&L)[3][8],
                                               float& down, int& tot) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(xv[i]));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  // m < 2^e; scale so that |X| < 2^22 (three signed limbs hold it)
  const int e = (int)((__float_as_uint(m) >> 23) & 0xFFu) - 126;
  int k = m > 0.0f ? 22 - e : 0;
  k = max(-120, min(k, 120));
  const float up = __uint_as_float((uint32_t)(127 + k) << 23);
  down = __uint_as_float((uint32_t)(127 - k) << 23);
  tot = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    uint32_t w0 = 0, w1 = 0, w2 = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int x = __float2int_rn(xv[4 * w + j] * up);
      x = max(-(1 << 22) + 1, min(x, (1 << 22) - 1));
      tot += x;
      const int l0 = ((x + 128) & 255) - 128;
      const int x1 = (x - l0) >> 8;
      const int l1 = ((x1 + 128) & 255) - 128;
      const int l2 = (x1 - l1) >> 8;
      w0 |= (uint32_t)(l0 & 255) << (8 * j);
      w1 |= (uint32_t)(l1 & 255) << (8 * j);
      w2 |= (uint32_t)(l2 & 255) << (8 * j);
    }
    L[0][w] = w0;
    L[1][w] = w1;
    L[2][w] = w2;
  }
  tot += __shfl_xor_sync(0xffffffffu, tot, 1);
}

// Quarter word q of one limb in the value order of BITS (see kappa_pos)
// from the limb's 8 natural-order words.
template <int BITS>
__device__ __forceinline__ uint32_t quarter_word(const uint32_t (&n)[8], int q) {
  if (BITS == 8) return n[q];
  if (BITS == 4) {
    // q < 4: values 8q + 0,2,4,6; q >= 4: values 8(q-4) + 1,3,5,7
    const int p = q & 3;
    return __byte_perm(n[2 * p], n[2 * p + 1], q < 4 ? 0x6420 : 0x7531);
  }
  // q < 4: values q, q+4, q+8, q+12; q >= 4: the same + 16 (byte q & 3 of
  // four consecutive words)
  const int p = q & 3, b = (q >> 2) * 4;
  const uint32_t sel_lo = (uint32_t)(p | ((p + 4) << 4));
  const uint32_t lo = __byte_perm(n[b], n[b + 1], sel_lo);
  const uint32_t hi = __byte_perm(n[b + 2], n[b + 3], sel_lo);
  return __byte_perm(lo, hi, 0x5410);
}

// Writes block blk of a table at tv (nblk blocks) in the value order of BITS.
template <int BITS>
__device__ __forceinline__ void emit_block(uint8_t* tv, int blk, int nblk, const uint32_t (&L)[3][8],
                                           float down, int tot) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint32_t* wa = reinterpret_cast<uint32_t*>(tv + blk * 96) + q;
    wa[0] = quarter_word<BITS>(L[0], q);
    wa[8] = quarter_word<BITS>(L[1], q);
    wa[16] = quarter_word<BITS>(L[2], q);
  }
  if ((blk & 1) == 0)
    *reinterpret_cast<float2*>(tv + nblk * 96 + (blk >> 1) * 8) = make_float2(down, (float)tot * down);
}

// Tables of n_vec vectors (vector v: src + v * len, table v at
// t + v * tab_bytes) in up to three value orders from one pass over the
// input (B2, B3 = 0: unused).
template <bool F32, int B1, int B2 = 0, int B3 = 0>
__device__ void build_tabs(const void* src, int len, int n_vec, int tab_bytes, uint8_t* t1,
                           uint8_t* t2, uint8_t* t3, int tid, int nthr) {
  const int nblk = len / 32;
  const int total = n_vec * nblk;
  for (int base = tid & ~31; base < total; base += nthr) {
    const int task = base + (tid & 31);
    const bool on = task < total;
    const int v = on ? task / nblk : 0, blk = on ? task % nblk : 0;
    float xv[32];
    load_block<F32>(src, (int64_t)v * len + blk * 32, on, xv);
    uint32_t L[3][8];
    float down;
    int tot;
    quantize_block(xv, L, down, tot);
    if (on) {
      const int off = v * tab_bytes;
      emit_block<B1>(t1 + off, blk, nblk, L, down, tot);
      if constexpr (B2 != 0) emit_block<B2>(t2 + off, blk, nblk, L, down, tot);
      if constexpr (B3 != 0) emit_block<B3>(t3 + off, blk, nblk, L, down, tot);
    }
  }
}

// ------------------------------------------------------------------ one unit
// A fragment of the tile rows at rg, rg8 for 32-value block kb (slab stride
// ss bytes, slab of sbytes).
template <int BITS>
__device__ __forceinline__ void load_a(const uint8_t* rg, const uint8_t* rg8, int kb, int ss,
                                       int sshift, int tig, uint32_t (&a)[4]) {
  constexpr int KBB = BITS * 4;  // bytes of a 32-value block
  const int byte = kb * KBB;
  const int off = (byte >> sshift) * ss + (byte & ((1 << sshift) - 1));
  if (BITS == 4) {
    const uint32_t w0 = *reinterpret_cast<const uint32_t*>(rg + off + tig * 4);
    const uint32_t w1 = *reinterpret_cast<const uint32_t*>(rg8 + off + tig * 4);
    a[0] = w0 & 0x0F0F0F0Fu;
    a[2] = (w0 >> 4) & 0x0F0F0F0Fu;
    a[1] = w1 & 0x0F0F0F0Fu;
    a[3] = (w1 >> 4) & 0x0F0F0F0Fu;
  } else if (BITS == 8) {
    a[0] = *reinterpret_cast<const uint32_t*>(rg + off + tig * 4);
    a[2] = *reinterpret_cast<const uint32_t*>(rg + off + 16 + tig * 4);
    a[1] = *reinterpret_cast<const uint32_t*>(rg8 + off + tig * 4);
    a[3] = *reinterpret_cast<const uint32_t*>(rg8 + off + 16 + tig * 4);
  } else {
    const uint2 w0 = *reinterpret_cast<const uint2*>(rg + off);
    const uint2 w1 = *reinterpret_cast<const uint2*>(rg8 + off);
    a[0] = (w0.x >> (2 * tig)) & 0x03030303u;
    a[2] = (w0.y >> (2 * tig)) & 0x03030303u;
    a[1] = (w1.x >> (2 * tig)) & 0x03030303u;
    a[3] = (w1.y >> (2 * tig)) & 0x03030303u;
  }
}

// This warp's share (groups [gb, ge), at most 8) of the unit in stage st
// against table tab: returns, on lane (g, tig 0), the partial value of tile
// row g and, on lane (g, tig 1), that of tile row g + 8.  Groups go in two
// batches of four with independent accumulators, so that their loads and
// MMAs overlap; the limbs of a row meet in one lane after two exchanges
// between lanes tig 0 and 1.  Out of line: one copy of the loop per bit
// width.
template <int BITS>
__device__ __noinline__ float unit_part(const uint8_t* st, FzUnit u, const FzKind* gp,
                                        const uint8_t* tab, int nblk_tab, int gb, int ge,
                                        int lane) {
  const FzKind g = *gp;
  const int gid = lane >> 2, tig = lane & 3;
  // tile rows without a weight row read box 0 row 0 (results unused)
  int b0, r0, b8, r8;
  if (!tile_row(u, gid, b0, r0)) b0 = r0 = 0;
  if (!tile_row(u, gid + 8, b8, r8)) b8 = r8 = 0;
  const int rstride = g.slab_bytes + 16;
  const int ss = g.RB * rstride;  // bytes from one slab to the next
  const int sshift = __ffs(g.slab_bytes) - 1;
  const uint8_t* rg = st + b0 * g.box_stride + r0 * rstride;
  const uint8_t* rg8 = st + b8 * g.box_stride + r8 * rstride;
  // this lane's row (tig 0: tile row g, tig 1: g + 8) of the scale/bias boxes
  const int bm = (tig & 1) ? b8 : b0, rm = (tig & 1) ? r8 : r0;
  const uint8_t* sbase = st + g.nbox * g.box_stride + bm * 2 * g.sb_stride + rm * (g.gpr + 8) * 2;
  const uint16_t* srow = reinterpret_cast<const uint16_t*>(sbase);
  const uint16_t* brow = reinterpret_cast<const uint16_t*>(sbase + g.sb_stride);
  const float2* xsv = reinterpret_cast<const float2*>(tab + nblk_tab * 96);
  const uint32_t* tw = reinterpret_cast<const uint32_t*>(tab) + gid * 8 + tig;
  float acc = 0.0f;
  for (int h = 0; h < 2; ++h) {
    if (gb + 4 * h >= ge) break;
    int d[4][4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      d[q][0] = d[q][1] = d[q][2] = d[q][3] = 0;
      const int grp = gb + 4 * h + q;
      if (grp < ge) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int kb = grp * 2 + j;
          uint32_t a[4];
          load_a<BITS>(rg, rg8, kb, ss, sshift, tig, a);
          uint32_t bl = 0, bh = 0;
          if (gid < 3) {
            bl = tw[kb * 24];
            bh = tw[kb * 24 + 4];
          }
          imma(d[q], a, bl, bh);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int grp = gb + 4 * h + q;
      // columns 0, 1, 2 hold limbs 0, 1, 2; lane tig 0 owns row g, tig 1 row g + 8
      const int x1 = __shfl_xor_sync(0xffffffffu, tig == 0 ? d[q][2] : d[q][0], 1);
      const int y1 = __shfl_xor_sync(0xffffffffu, d[q][3], 1);
      if (tig < 2 && grp < ge) {
        const int l0 = tig == 0 ? d[q][0] : x1;
        const int l1 = tig == 0 ? d[q][1] : y1;
        const int l2 = tig == 0 ? x1 : d[q][2];
        const float2 xs = xsv[grp];  // (scale, scale * sum X)
        const float f = fmaf(65536.0f, (float)l2, fmaf(256.0f, (float)l1, (float)l0));
        acc += fmaf(bf16_bits_to_float(srow[grp]), xs.x * f, bf16_bits_to_float(brow[grp]) * xs.y);
      }
    }
  }
  return acc;
}

__device__ __forceinline__ float silu_mul(float g, float u) {
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

// ------------------------------------------------------------------ shared memory
struct FzSmem {
  const FusedArgs* a;
  uint8_t* base;    // the dynamic shared memory
  uint32_t ring;    // its shared-memory address of the ring (copy destinations)
  FzUnit* units;
  float* red;       // [2][FZ_CW][16] partial row values
  float* dpart;     // [K + 1][drows_max]
  uint64_t* full;   // [FZ_NS]
  uint64_t* empty;  // [FZ_NS]
  uint64_t* rbar;   // the routing is known (the producer arrives once)
  int* misc;        // [0] dead, [1] units, [2] n1, [3] n3
  int32_t* idx;     // [kFusedMaxK]
  float* w;         // [kFusedMaxK]
  float* sigma;
};

__device__ __forceinline__ FzSmem fz_smem(uint8_t* sm, const FusedArgs& p) {
  FzSmem s;
  s.a = reinterpret_cast<const FusedArgs*>(sm + p.off_args);
  s.base = sm;
  s.ring = tc::smem_u32(sm) + p.off_ring;
  s.units = reinterpret_cast<FzUnit*>(sm + p.off_units);
  s.red = reinterpret_cast<float*>(sm + p.off_red);
  s.dpart = reinterpret_cast<float*>(sm + p.off_dpart);
  s.full = reinterpret_cast<uint64_t*>(sm + p.off_bar);
  s.empty = s.full + FZ_NS;
  s.rbar = s.empty + FZ_NS;
  s.misc = reinterpret_cast<int*>(s.rbar + 1);
  s.idx = s.misc + 4;
  s.w = reinterpret_cast<float*>(s.idx + kFusedMaxK);
  s.sigma = s.w + kFusedMaxK;
  return s;
}

// Wait for an mbarrier phase, sleeping in hardware (up to 1 ms per try),
// for at most about two seconds; gives up early once the CTA is dead.
__device__ __forceinline__ bool fz_wait(uint64_t* bar, uint32_t parity, int* status, const int* dead) {
  const uint32_t addr = tc::smem_u32(bar);
  for (int i = 0; i < 2000; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(addr), "r"(parity), "r"(1000000u)
        : "memory");
    if (ok) return true;
    if (ld_vol(dead)) return false;
  }
  set_status(status, MOEQ_ERR_TIMEOUT);
  return false;
}

// Warp-wide bounded wait until flags[0..n) all equal tag (then an acquire
// fence); false on timeout (status set) or when the CTA is dead.
__device__ __forceinline__ bool wait_all_flags(const uint64_t* flags, int n, uint64_t tag,
                                               int* status, const int* dead) {
  const int lane = threadIdx.x & 31;
  const uint64_t t0 = tc::globaltimer_ns();
  for (;;) {
    bool ok = true;
    for (int i = lane; i < n; i += 32) ok = ok && ld_relaxed_u64(flags + i) == tag;
    if (__all_sync(0xffffffffu, ok)) break;
    bool give_up = ld_vol(dead) != 0;
    if (!give_up && tc::globaltimer_ns() - t0 > 2000000000ull) {
      set_status(status, MOEQ_ERR_TIMEOUT);
      give_up = true;
    }
    if (__any_sync(0xffffffffu, give_up)) return false;
  }
  fence_acq_rel_gpu();
  return true;
}

__device__ __forceinline__ int64_t unit_expert(const FzSmem& S, const FzUnit& u) {
  return (u.kind == FZ_GU || u.kind == FZ_DN) ? S.idx[u.k] : 0;
}

// ------------------------------------------------------------------ producer
// Fills the stage of unit `seq` (lane 0: one tensor-map copy per box) after
// the stage's previous unit was used.
__device__ __forceinline__ bool issue_unit(const FzSmem& S, const FzMaps& M, int seq) {
  const FusedArgs& a = *S.a;
  const int lane = threadIdx.x & 31;
  const int stage = seq % FZ_NS;
  bool ok = true;
  if (seq >= FZ_NS) ok = fz_wait(&S.empty[stage], (uint32_t)((seq / FZ_NS - 1) & 1), a.status, S.misc);
  if (lane == 0) {
    if (!ok) {
      mark_dead(S.misc);
    } else {
      const FzUnit u = S.units[seq];
      const FzKind& g = a.kind[u.kind];
      const uint32_t st = S.ring + (uint32_t)stage * a.stage_bytes;
      const int e = (int)unit_expert(S, u);
      tc::mbar_arrive_expect_tx(&S.full[stage],
                                (uint32_t)(g.nbox * (g.box_bytes + 2 * g.sb_bytes)));
      const uint32_t sbb = st + (uint32_t)(g.nbox * g.box_stride);
      for (int b = 0; b < g.nbox; ++b) {
        const int mi = 3 * unit_map(u, b);
        tma_load_4d(st + (uint32_t)(b * g.box_stride), &M.tm[mi], 0, u.r0, 0, e, &S.full[stage]);
        tc::tma_load_3d(sbb + (uint32_t)(2 * b * g.sb_stride), &M.tm[mi + 1], 0, u.r0, e,
                        &S.full[stage]);
        tc::tma_load_3d(sbb + (uint32_t)((2 * b + 1) * g.sb_stride), &M.tm[mi + 2], 0, u.r0, e,
                        &S.full[stage]);
      }
    }
  }
  __syncwarp();
  return ok;
}

// L2 prefetch of the rows and scale/bias runs of units [from, to).
__device__ __forceinline__ void prefetch_units(const FzSmem& S, int from, int to) {
  const FusedArgs& a = *S.a;
  const int lane = threadIdx.x & 31;
  for (int q = from + (lane >> 1); q < to; q += 16) {
    const FzUnit u = S.units[q];
    const FzKind& g = a.kind[u.kind];
    const int box = lane & 1;
    if (box >= g.nbox) continue;
    const moeq_qtensor& t = unit_tensor(a, u, box);
    const int64_t e = unit_expert(S, u);
    tc::prefetch_l2(reinterpret_cast<const uint8_t*>(t.w + e * t.expert_stride_w) +
                        (int64_t)u.r0 * g.row_bytes,
                    (uint32_t)(u.n * g.row_bytes));
    const uint32_t sbn = (uint32_t)(u.n * g.gpr * 2);
    const int64_t so = (e * t.expert_stride_sb + (int64_t)u.r0 * g.gpr) * 2;
    if ((sbn & 15) == 0 && (so & 15) == 0) {
      tc::prefetch_l2(reinterpret_cast<const uint8_t*>(t.scales) + so, sbn);
      tc::prefetch_l2(reinterpret_cast<const uint8_t*>(t.biases) + so, sbn);
    }
  }
}

// The routing selection over the logit buffer into the CTA's routing slots
// (out of line: the early warm-up run and the real selection execute the
// same code).
__device__ __noinline__ void route_select(const FusedArgs& a, const FzSmem& S) {
  const float* lg = a.logits;
  if (a.E <= 32) route_token_regs<1>(lg, a.E, a.K, a.renorm, a.router_scale, S.idx, S.w);
  else if (a.E <= 64) route_token_regs<2>(lg, a.E, a.K, a.renorm, a.router_scale, S.idx, S.w);
  else if (a.E <= 128) route_token_regs<4>(lg, a.E, a.K, a.renorm, a.router_scale, S.idx, S.w);
  else if (a.E <= 256) route_token_regs<8>(lg, a.E, a.K, a.renorm, a.router_scale, S.idx, S.w);
  else if (a.E <= 512) route_token_regs<16>(lg, a.E, a.K, a.renorm, a.router_scale, S.idx, S.w);
  else route_token_regs<32>(lg, a.E, a.K, a.renorm, a.router_scale, S.idx, S.w);
}

// ------------------------------------------------------------------ compute side
// Groups of the unit's rows this warp takes.
__device__ __forceinline__ void warp_groups(const FzKind& g, int warp, int& gb, int& ge) {
  gb = warp * g.gpr / FZ_CW;
  ge = (warp + 1) * g.gpr / FZ_CW;
}

template <int BR, int BS, int BE>
__device__ __forceinline__ void run_unit(const FzSmem& S, int seq, int dlo, int warp, int lane,
                                         int& rbuf) {
  const FusedArgs& a = *S.a;
  const int stage = seq % FZ_NS;
  if (!fz_wait(&S.full[stage], (uint32_t)((seq / FZ_NS) & 1), a.status, S.misc) && lane == 0)
    mark_dead(S.misc);
  const FzUnit u = S.units[seq];
  const FzKind& g = a.kind[u.kind];
  const uint8_t* st = S.base + a.off_ring + stage * a.stage_bytes;
  int gb, ge;
  warp_groups(g, warp, gb, ge);
  float v = 0.0f;
  if (!ld_vol(S.misc)) {
    // the unit's input table and the bit width of its codes
    const uint8_t* tab;
    int nblk, bits;
    switch (u.kind) {
      case FZ_ROUTER:
      case FZ_SGATE: tab = S.base + a.off_xR; nblk = a.H / 32; bits = BR; break;
      case FZ_SHGU: tab = S.base + a.off_xS; nblk = a.H / 32; bits = BS; break;
      case FZ_SHDN: tab = S.base + a.off_hS; nblk = a.Ish / 32; bits = BS; break;
      case FZ_GU: tab = S.base + a.off_xE; nblk = a.H / 32; bits = BE; break;
      default: tab = S.base + a.off_hl + u.k * a.tab_h1; nblk = a.I / 32; bits = BE; break;
    }
    if (bits == BR) v = unit_part<BR>(st, u, &g, tab, nblk, gb, ge, lane);
    else if constexpr (BE != BR) {
      if (bits == BE) v = unit_part<BE>(st, u, &g, tab, nblk, gb, ge, lane);
      else if constexpr (BS != 0 && BS != BE && BS != BR) v = unit_part<BS>(st, u, &g, tab, nblk, gb, ge, lane);
    } else if constexpr (BS != 0 && BS != BE) {
      v = unit_part<BS>(st, u, &g, tab, nblk, gb, ge, lane);
    }
  }
  float* red = S.red + rbuf * FZ_CW * 16;
  if ((lane & 3) < 2) red[warp * 16 + (lane >> 2) + 8 * (lane & 1)] = v;
  tc::named_sync(FZ_BAR_C, FZ_CT);
  const int t = threadIdx.x;
  if (t < 16 && t < u.n && !ld_vol(S.misc)) {
    float v = 0.0f;
    for (int q = 0; q < FZ_CW; ++q) v += red[q * 16 + t];
    if (u.kind == FZ_SHGU || u.kind == FZ_GU) {
      float w8 = 0.0f;
      for (int q = 0; q < FZ_CW; ++q) w8 += red[q * 16 + t + 8];
      const float hv = silu_mul(v, w8);
      if (u.kind == FZ_GU) a.h[(int64_t)u.k * a.I + u.r0 + t] = hv;
      else a.hsh[u.r0 + t] = hv;
    } else if (u.kind == FZ_ROUTER) {
      a.logits[u.r0 + t] = v;
    } else if (u.kind == FZ_SGATE) {
      a.logits[a.E] = v;
    } else {
      const int slot = u.kind == FZ_SHDN ? a.K : u.k;
      S.dpart[slot * a.drows_max + (u.r0 - dlo) + t] = v;
    }
  }
  if (t == 0) tc::mbar_arrive(&S.empty[stage]);
  rbuf ^= 1;
}

// Units [j0, j1) in order.
template <int BR, int BS, int BE>
__device__ __forceinline__ void run_units(const FzSmem& S, int j0, int j1, int dlo, int warp,
                                          int lane, int& rbuf) {
  for (int j = j0; j < j1; ++j) run_unit<BR, BS, BE>(S, j, dlo, warp, lane, rbuf);
}

template <int BR, int BS, int BE>
__global__ void __maxnreg__(96) k_fused_decode(const __grid_constant__ FusedArgs p,
                                                const __grid_constant__ FzMaps maps) {
  extern __shared__ __align__(128) uint8_t fsm[];
  const FzSmem S = fz_smem(fsm, p);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x, P = gridDim.x;
  int* dead = S.misc;

  // the arguments in shared memory (one coalesced pass over parameter space)
  {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(&p);
    uint32_t* dst = reinterpret_cast<uint32_t*>(fsm + p.off_args);
    for (int i = threadIdx.x; i < (int)(sizeof(FusedArgs) / 4); i += FZ_THREADS) dst[i] = src[i];
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < FZ_NS; ++i) {
      tc::mbar_init(&S.full[i], 1);
      tc::mbar_init(&S.empty[i], 1);
    }
    tc::mbar_init(S.rbar, 1);
    tc::fence_mbar_init();
  }
  __syncthreads();
  const FusedArgs& a = *S.a;
  if (threadIdx.x == 0) {
    int n1, n3;
    const int nu = fz_units(a, c, P, S.units, FZ_UMAX, &n1, &n3);
    S.misc[0] = nu > FZ_UMAX ? 1 : 0;
    S.misc[1] = imin(nu, FZ_UMAX);
    S.misc[2] = n1;
    S.misc[3] = n3;
    if (nu > FZ_UMAX) set_status(a.status, MOEQ_ERR_INVALID_ARG);
  }
  __syncthreads();
  const int nu = S.misc[1], n1 = S.misc[2], n3 = S.misc[3];
  const bool phase1 = a.route_from_router || a.has_shared;
  int dlo, dhi;
  fz_range(a.H, a.dgran, c, P, dlo, dhi);

  if (warp == FZ_PROD) {
    // ------------------------------------------------------------ producer
    // routing-independent weights first, before the dependency wait; a
    // shared down unit is issued early only into a stage whose previous
    // unit is consumed before the routing
    const int n_sdn = a.has_shared ? (dhi - dlo + a.kind[FZ_SHDN].RB - 1) / a.kind[FZ_SHDN].RB : 0;
    const int n_pre = n1 + n_sdn;
    if (n_pre > FZ_NS) prefetch_units(S, FZ_NS, n_pre);
    int seq = 0;
    for (; seq < n_pre && seq < FZ_NS; ++seq)
      if (!issue_unit(S, maps, seq)) break;
    tc::grid_dep_wait();
    tc::grid_dep_launch();
    // (every tag computation reads word 0 before CTA 0 rewrites it at its end)
    const uint64_t tag = next_tag(*a.gen);
    for (; seq < n_pre && seq - FZ_NS < n1 && !ld_vol(dead); ++seq)
      if (!issue_unit(S, maps, seq)) break;
    // While the first flags are outstanding, run the top-K once on whatever
    // the logit buffer holds (results discarded: the real routing below
    // overwrites them), so that its code is in the instruction cache when
    // the routing is on the critical path.
    if (a.route_from_router && phase1) route_select(a, S);
    // routing: every CTA's logits, shared gate logit and shared hidden values are out
    bool ok = !ld_vol(dead);
    if (ok && phase1) ok = wait_all_flags(a.flag1, P, tag, a.status, dead);
    if (ok) {
      if (a.route_from_router) {
        route_select(a, S);
      } else if (lane < a.K) {
        int e = a.idx_in[lane];
        if (e < 0 || e >= a.E) {
          set_status(a.status, MOEQ_ERR_INVALID_ARG);
          e = 0;
        }
        S.idx[lane] = e;
        S.w[lane] = a.w_in[lane];
      }
      if (lane == 0 && a.has_shared) *S.sigma = 1.0f / (1.0f + expf(-a.logits[a.E]));
      __syncwarp();
      if (c == 0 && lane < a.K) {
        if (a.idx_out) a.idx_out[lane] = S.idx[lane];
        if (a.w_out) a.w_out[lane] = S.w[lane];
      }
    } else if (lane == 0) {
      mark_dead(dead);
    }
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(S.rbar);
    if (ok) {
      // the routed bytes into L2 in stream order, then through the ring
      prefetch_units(S, seq, nu);
      for (; seq < nu; ++seq)
        if (!issue_unit(S, maps, seq)) break;
    }
    // every stage's last fill has landed before the CTA exits (bounded, and
    // regardless of whether the CTA gave up on its work)
    const int alive = 0;
    for (int st = 0; st < FZ_NS && st < seq; ++st) {
      const int last = st + ((seq - 1 - st) / FZ_NS) * FZ_NS;
      fz_wait(&S.full[st], (uint32_t)((last / FZ_NS) & 1), a.status, &alive);
    }
    return;
  }

  // ---------------------------------------------------------------- compute warps
  const int t = threadIdx.x;
  int rbuf = 0;
  tc::grid_dep_wait();
  tc::grid_dep_launch();
  const uint64_t tag = next_tag(*a.gen);
  // the token as tables, one per value order in use
  {
    constexpr bool sep_s = BS != 0 && BS != BE;
    if (phase1) {
      if constexpr (sep_s) build_tabs<false, BR, BE, BS>(a.x, a.H, 1, 0, S.base + a.off_xR,
                                                         S.base + a.off_xE, S.base + a.off_xS, t, FZ_CT);
      else build_tabs<false, BR, BE>(a.x, a.H, 1, 0, S.base + a.off_xR, S.base + a.off_xE,
                                     nullptr, t, FZ_CT);
    } else {
      build_tabs<false, BE>(a.x, a.H, 1, 0, S.base + a.off_xE, nullptr, nullptr, t, FZ_CT);
    }
  }
  tc::named_sync(FZ_BAR_C, FZ_CT);

  // phase 1: router rows, shared gate row, shared gate/up (scale/bias of the
  // next unit only when it does not need the routing)
  run_units<BR, BS, BE>(S, 0, n1, dlo, warp, lane, rbuf);
  tc::named_sync(FZ_BAR_C, FZ_CT);
  if (phase1 && t == 0) {
    __threadfence();
    st_release_u64(a.flag1 + c, tag);
  }
  // routing known: the producer passed the first flag barrier
  if (!fz_wait(S.rbar, 0, a.status, dead) && t == 0) mark_dead(dead);
  fence_acq_rel_gpu();
  if constexpr (BS != 0) {
    if (a.has_shared && !ld_vol(dead))
      build_tabs<true, BS>(a.hsh, a.Ish, 1, 0, S.base + a.off_hS, nullptr, nullptr, t, FZ_CT);
  }
  tc::named_sync(FZ_BAR_C, FZ_CT);

  // phase 3: shared down rows, routed gate/up + SwiGLU
  run_units<BR, BS, BE>(S, n1, n1 + n3, dlo, warp, lane, rbuf);
  tc::named_sync(FZ_BAR_C, FZ_CT);
  if (t == 0) {
    __threadfence();
    st_release_u64(a.flag2 + c, tag);
  }
  if (warp == 0 && !wait_all_flags(a.flag2, P, tag, a.status, dead) && lane == 0) mark_dead(dead);
  tc::named_sync(FZ_BAR_C, FZ_CT);
  fence_acq_rel_gpu();
  if (!ld_vol(dead))
    build_tabs<true, BE>(a.h, a.I, a.K, a.tab_h1, S.base + a.off_hl, nullptr, nullptr, t, FZ_CT);
  tc::named_sync(FZ_BAR_C, FZ_CT);

  // phase 4: routed down rows, then this CTA's rows of y
  run_units<BR, BS, BE>(S, n1 + n3, nu, dlo, warp, lane, rbuf);
  tc::named_sync(FZ_BAR_C, FZ_CT);
  if (!ld_vol(dead)) {
    const float sg = a.has_shared ? *S.sigma : 0.0f;
    for (int r = t; r < dhi - dlo; r += FZ_CT) {
      float acc = a.has_shared ? sg * S.dpart[a.K * a.drows_max + r] : 0.0f;
      for (int k = 0; k < a.K; ++k) acc = fmaf(S.w[k], S.dpart[k * a.drows_max + r], acc);
      if (a.residual) acc += a.residual[dlo + r];
      a.y[dlo + r] = acc;
    }
  }
  // the next call's tag derives from this one (every CTA has read the old
  // value: CTA 0 got here only after every flag of this call was raised)
  if (c == 0 && t == 0) *a.gen = tag;
}

// Raises the kernel's dynamic shared-memory limit to a.smem_bytes on the
// current device (once per size) and checks that one CTA of FZ_THREADS fits
// on an SM: the register file is split over four sub-partitions, so a block
// of 17 warps is charged for 20.
template <int BR, int BS, int BE>
cudaError_t fz_prepare(const FusedArgs& a) {
  auto kern = k_fused_decode<BR, BS, BE>;
  static std::atomic<int> attr_set[kMaxDevices];
  int dev;
  if (!current_device(dev)) return cudaErrorInvalidDevice;
  cudaError_t e;
  if (attr_set[dev].load(std::memory_order_acquire) >= a.smem_bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, a.smem_bytes);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, FZ_THREADS, a.smem_bytes);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorLaunchOutOfResources;
  int cur = attr_set[dev].load();
  while (cur < a.smem_bytes && !attr_set[dev].compare_exchange_weak(cur, a.smem_bytes)) {
  }
  return cudaSuccess;
}

template <int BR, int BS, int BE>
cudaError_t launch_fz(const FusedArgs& a, const FzMaps& m, int grid, cudaStream_t st) {
  auto kern = k_fused_decode<BR, BS, BE>;
  cudaError_t e = fz_prepare<BR, BS, BE>(a);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(FZ_THREADS);
  cfg.dynamicSmemBytes = a.smem_bytes;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, m);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (null if
// the driver does not provide it).
PFN_cuTensorMapEncodeTiled_v12000 fz_encode_fn() {
  static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
  PFN_cuTensorMapEncodeTiled_v12000 f = fn.load(std::memory_order_acquire);
  if (!f) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
      fn.store(f, std::memory_order_release);
    }
  }
  return f;
}

// Unit geometry of a tensor: rows of row_bytes cut into slabs of up to 128
// bytes (a power of two dividing the row, at least one 32-value block).
bool kind_geom(FzKind& k, const moeq_qtensor& t, int RB, int nbox, int gran) {
  k.row_bytes = t.in_dim * t.bits / 8;
  k.gpr = t.in_dim / t.group_size;
  k.RB = RB;
  k.nbox = nbox;
  k.gran = gran;
  int sb = 128;
  while (sb > t.bits * 4 && (k.row_bytes % sb)) sb >>= 1;
  if (k.row_bytes % sb || sb < t.bits * 4 || sb < 16) return false;
  k.slab_bytes = sb;
  k.S = k.row_bytes / sb;
  k.box_bytes = k.S * RB * (sb + 16);
  k.box_stride = (k.box_bytes + 127) & ~127;
  k.sb_bytes = RB * (k.gpr + 8) * 2;
  k.sb_stride = (k.sb_bytes + 127) & ~127;
  // scale/bias rows: whole 16-byte runs
  return k.S <= 256 && k.gpr % 8 == 0 && k.gpr + 8 <= 256;
}

// 4-D map (slab words, row, slab, matrix) of a code tensor with a box of
// (slab + 4 words, RB rows, all slabs, 1 matrix).
bool code_map(CUtensorMap* m, const moeq_qtensor& t, const FzKind& k, int n_mat) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = fz_encode_fn();
  if (!fn || ((uintptr_t)t.w & 15)) return false;
  const int64_t mat_bytes = n_mat > 1 ? t.expert_stride_w * 4 : (int64_t)t.out_dim * k.row_bytes;
  if ((mat_bytes & 15) || mat_bytes <= 0) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)(k.slab_bytes / 4), (cuuint64_t)t.out_dim,
                              (cuuint64_t)k.S, (cuuint64_t)n_mat};
  const cuuint64_t strides[3] = {(cuuint64_t)k.row_bytes, (cuuint64_t)k.slab_bytes,
                                 (cuuint64_t)mat_bytes};
  const cuuint32_t box[4] = {(cuuint32_t)(k.slab_bytes / 4 + 4), (cuuint32_t)k.RB,
                             (cuuint32_t)k.S, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<uint32_t*>(t.w), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map (entry, row, matrix) of a scale or bias array with a box of
// (gpr + 8 entries, RB rows, 1 matrix).
bool sb_map(CUtensorMap* m, const uint16_t* p, const moeq_qtensor& t, const FzKind& k, int n_mat) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = fz_encode_fn();
  if (!fn || ((uintptr_t)p & 15)) return false;
  const int64_t mat_bytes =
      n_mat > 1 ? t.expert_stride_sb * 2 : (int64_t)t.out_dim * k.gpr * 2;
  if ((mat_bytes & 15) || mat_bytes <= 0) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)k.gpr, (cuuint64_t)t.out_dim, (cuuint64_t)n_mat};
  const cuuint64_t strides[2] = {(cuuint64_t)k.gpr * 2, (cuuint64_t)mat_bytes};
  const cuuint32_t box[3] = {(cuuint32_t)(k.gpr + 8), (cuuint32_t)k.RB, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<uint16_t*>(p), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Code, scale and bias maps of tensor id.
bool tensor_maps(FzMaps& maps, int id, const moeq_qtensor& t, const FzKind& k, int n_mat) {
  return code_map(&maps.tm[3 * id], t, k, n_mat) && sb_map(&maps.tm[3 * id + 1], t.scales, t, k, n_mat) &&
         sb_map(&maps.tm[3 * id + 2], t.biases, t, k, n_mat);
}

int tab_bytes(int len) { return ((len / 32) * 96 + (len / FZ_G) * 8 + 15) & ~15; }

bool fz_fits(const FusedArgs& a);

}  // namespace

// Geometry, tensor maps, shared-memory layout and applicability of the
// one-launch decode for this layer (M = 1).  Fills the shape part of `a`.
bool fused_decode_plan(const moeq_layer* L, int grid, bool route_from_router, FusedArgs& a,
                       FzMaps& maps) {
  const int H = L->hidden, I = L->inter, E = L->n_experts, K = L->top_k;
  if (K > kFusedMaxK || E > 1024 || grid < 1 || grid > kFusedMaxGrid) return false;
  const moeq_qtensor &R = L->router, &Gt = L->gate, &D = L->down;
  const int BR = R.bits, BE = Gt.bits;
  if (BR != 8 || D.bits != BE || L->up.bits != BE) return false;
  if (!(BE == 4 || BE == 2 || BE == 8)) return false;
  int BS = 0;
  const int Ish = L->has_shared ? L->sh_gate.out_dim : 0;
  if (L->has_shared) {
    BS = L->sh_gate.bits;
    if (L->sh_down.bits != BS || L->sh_up.bits != BS) return false;
    if (BS != 4 && BS != BE) return false;
    if (L->sh_expert_gate.bits != BR) return false;
  }
  // every tensor: affine, groups of 64, whole 32-value blocks, at most 8
  // groups per compute warp
  const moeq_qtensor* all[8] = {&R, &Gt, &L->up, &D, &L->sh_gate, &L->sh_up, &L->sh_down,
                                &L->sh_expert_gate};
  const int n_all = L->has_shared ? 8 : 4;
  for (int i = 0; i < n_all; ++i) {
    const moeq_qtensor& t = *all[i];
    if (t.format != MOEQ_FMT_AFFINE) return false;  // bf16 scale and bias per group only
    if (t.group_size != FZ_G || t.in_dim % FZ_G || t.in_dim / FZ_G > 8 * FZ_CW) return false;
  }
  memset(&a, 0, sizeof(a));
  memset(&maps, 0, sizeof(maps));
  a.H = H;
  a.I = I;
  a.E = E;
  a.K = K;
  a.Ish = Ish;
  a.renorm = L->renorm;
  a.router_scale = L->router_scale;
  a.has_shared = L->has_shared;
  a.route_from_router = route_from_router ? 1 : 0;
  a.router = R;
  a.gate = Gt;
  a.up = L->up;
  a.down = D;
  if (L->has_shared) {
    a.sgate = L->sh_expert_gate;
    a.sh_gate = L->sh_gate;
    a.sh_up = L->sh_up;
    a.sh_down = L->sh_down;
  }
  // units: router 4 rows, gate/up 4 indices (two boxes), down 8 rows; the
  // CTA ranges are whole units
  if (E % 4 || I % 8 || H % 8 || (L->has_shared && Ish % 8)) return false;
  bool ok = kind_geom(a.kind[FZ_ROUTER], R, 4, 1, 4) && kind_geom(a.kind[FZ_GU], Gt, 8, 2, 8) &&
            kind_geom(a.kind[FZ_DN], D, 8, 1, 8);
  FzKind up_k;
  ok = ok && kind_geom(up_k, L->up, 8, 2, 8) && up_k.box_bytes == a.kind[FZ_GU].box_bytes;
  if (L->has_shared) {
    FzKind shu_k;
    ok = ok && kind_geom(a.kind[FZ_SGATE], L->sh_expert_gate, 4, 1, 4) &&
         kind_geom(a.kind[FZ_SHGU], L->sh_gate, 8, 2, 8) &&
         kind_geom(shu_k, L->sh_up, 8, 2, 8) && shu_k.box_bytes == a.kind[FZ_SHGU].box_bytes &&
         kind_geom(a.kind[FZ_SHDN], L->sh_down, 8, 1, 8);
  }
  if (!ok) return false;
  a.dgran = 8;
  // tensor maps (one per code tensor)
  ok = tensor_maps(maps, FZM_ROUTER, R, a.kind[FZ_ROUTER], 1) &&
       tensor_maps(maps, FZM_G, Gt, a.kind[FZ_GU], E) &&
       tensor_maps(maps, FZM_U, L->up, a.kind[FZ_GU], E) &&
       tensor_maps(maps, FZM_D, D, a.kind[FZ_DN], E);
  if (L->has_shared)
    ok = ok && tensor_maps(maps, FZM_SGATE, L->sh_expert_gate, a.kind[FZ_SGATE], 1) &&
         tensor_maps(maps, FZM_SHG, L->sh_gate, a.kind[FZ_SHGU], 1) &&
         tensor_maps(maps, FZM_SHU, L->sh_up, a.kind[FZ_SHGU], 1) &&
         tensor_maps(maps, FZM_SHD, L->sh_down, a.kind[FZ_SHDN], 1);
  if (!ok) return false;
  // stage: the largest unit
  int stage = 0;
  for (int k = 0; k < 6; ++k) {
    if (!L->has_shared && (k == FZ_SGATE || k == FZ_SHGU || k == FZ_SHDN)) continue;
    stage = std::max(stage, a.kind[k].nbox * (a.kind[k].box_stride + 2 * a.kind[k].sb_stride));
  }
  a.stage_bytes = (stage + 127) & ~127;
  // units per CTA
  int max_units = 0, max_drows = 0;
  for (int c = 0; c < grid; ++c) {
    int n1, n3;
    max_units = std::max(max_units, fz_units(a, c, grid, nullptr, 0, &n1, &n3));
    int lo, hi;
    fz_range(H, a.dgran, c, grid, lo, hi);
    max_drows = std::max(max_drows, hi - lo);
  }
  if (max_units > FZ_UMAX) return false;
  a.drows_max = max_drows;
  // input tables
  a.tab_x8 = tab_bytes(H);
  a.tab_xe = tab_bytes(H);
  a.tab_xs = L->has_shared ? tab_bytes(H) : 0;
  a.tab_hs = L->has_shared ? tab_bytes(Ish) : 0;
  a.tab_h1 = tab_bytes(I);
  size_t off = 0;
  auto take = [&](size_t b) {
    const size_t o = off;
    off += (b + 127) & ~(size_t)127;
    return (int32_t)o;
  };
  a.off_ring = take((size_t)FZ_NS * a.stage_bytes);
  // the routed hidden tables reuse the router's token table (phase 4 only)
  a.off_xR = take(std::max((size_t)a.tab_x8, (size_t)K * a.tab_h1));
  a.off_hl = a.off_xR;
  a.off_xE = take((size_t)a.tab_xe);
  a.off_xS = (L->has_shared && BS != BE) ? take((size_t)a.tab_xs) : a.off_xE;
  a.off_hS = L->has_shared ? take((size_t)a.tab_hs) : a.off_xE;
  a.off_units = take((size_t)FZ_UMAX * sizeof(FzUnit));
  a.off_red = take((size_t)2 * FZ_CW * 16 * 4);
  a.off_dpart = take((size_t)(K + 1) * max_drows * 4);
  a.off_args = take(sizeof(FusedArgs));
  a.off_bar = take((2 * FZ_NS + 1) * 8 + (4 + 2 * kFusedMaxK + 1) * 4 + 16);
  a.smem_bytes = (int32_t)off;
  if (off > FZ_SMEM_MAX) return false;
  a.bits[0] = BR;
  a.bits[1] = BS;
  a.bits[2] = BE;
  // one CTA per SM must fit (shared memory and registers)
  return fz_fits(a);
}

int fused_decode_threads() { return FZ_THREADS; }

namespace {
bool fz_fits(const FusedArgs& a) {
  const int BS = a.bits[1], BE = a.bits[2];
  cudaError_t e;
  if (BS == 0) e = BE == 4 ? fz_prepare<8, 0, 4>(a) : BE == 2 ? fz_prepare<8, 0, 2>(a) : fz_prepare<8, 0, 8>(a);
  else if (BE == 4) e = fz_prepare<8, 4, 4>(a);
  else if (BE == 2) e = BS == 4 ? fz_prepare<8, 4, 2>(a) : fz_prepare<8, 2, 2>(a);
  else e = BS == 4 ? fz_prepare<8, 4, 8>(a) : fz_prepare<8, 8, 8>(a);
  if (e != cudaSuccess) cudaGetLastError();  // a refusal here is not sticky
  return e == cudaSuccess;
}
}  // namespace

cudaError_t launch_fused_decode(const FusedArgs& a, const FzMaps& m, int grid, cudaStream_t st) {
  const int BS = a.bits[1], BE = a.bits[2];
  if (BS == 0) {
    if (BE == 4) return launch_fz<8, 0, 4>(a, m, grid, st);
    if (BE == 2) return launch_fz<8, 0, 2>(a, m, grid, st);
    return launch_fz<8, 0, 8>(a, m, grid, st);
  }
  if (BE == 4) return launch_fz<8, 4, 4>(a, m, grid, st);
  if (BE == 2) return BS == 4 ? launch_fz<8, 4, 2>(a, m, grid, st) : launch_fz<8, 2, 2>(a, m, grid, st);
  return BS == 4 ? launch_fz<8, 4, 8>(a, m, grid, st) : launch_fz<8, 8, 8>(a, m, grid, st);
}

}  // namespace moeq
