// Decode path kernels: split-K quantised GEMV (router, gate/up + SwiGLU,
// down), top-K routing with the grouped work plan, and the weighted combine.
#include "gemv.cuh"
#include "kernels.h"
#include "route.cuh"
#include "tc.cuh"

namespace moeq {

GemvShape gemv_shape(int in_dim, int bits, int nmat, int G) {
  GemvShape sh;
  const int cpr = in_dim / chunk_values(bits);
  sh.S = (cpr + 31) / 32;
  sh.J = sh.S >= 8 ? 1 : 8 / sh.S;
  // fewer row subsets when a unit would not fit one stage
  const int64_t row = (int64_t)in_dim * bits / 8 + 4 * (in_dim / G);
  while (sh.J > 1 && (int64_t)nmat * sh.J * (8 / nmat) * row > 44 * 1024) sh.J >>= 1;
  sh.RU = sh.J * (8 / nmat);
  return sh;
}

bool gemv_fits(int in_dim, int bits, int nmat, int G) {
  const GemvShape sh = gemv_shape(in_dim, bits, nmat, G);
  const int64_t row = (int64_t)in_dim * bits / 8 + 4 * (in_dim / G);
  return sh.S <= 8 && (int64_t)nmat * sh.RU * row <= 44 * 1024;
}

int gemv_units(int out_dim, const GemvShape& sh) { return (out_dim + sh.RU - 1) / sh.RU; }

size_t gemv_xslice_words(int H, int bits) {
  if (bits != 2 && bits != 4 && bits != 8) return 0;
  const int vpc = chunk_values(bits);
  const int S = (H / vpc + 31) / 32;
  const int slw = 2 * (vpc / 4) + 2 * (bits == 2 ? 2 : 1);  // 2 limbs, block scales and sums
  return (size_t)S * slw * 32;
}

// One slice (32 chunks) of a token row in the gate/up launch's format, by
// one warp, into the table (word-major, as slice_load reads it).
template <int B>
__device__ __forceinline__ void xslice_one(const uint16_t* row, int H, int sl, uint32_t* out,
                                           int lane) {
  const int ch = sl * 32 + lane;
  SliceVec<B, 2> sv;
  build_slice<B, 2, SrcBF16>(row, ch, ch < H / Chunk<B>::VPC, sv);
  slice_store<B, 2>(out, sv, lane);
}

// The helper warp's share of the token slice table: task t = (token, slice)
// for t = blockIdx.x, blockIdx.x + gridDim.x, ...
__device__ __noinline__ void build_xslices(const TokenSlices& ts) {
  const int lane = threadIdx.x & 31;
  const int tasks = ts.M * ts.S;
  for (int t = blockIdx.x; t < tasks; t += gridDim.x) {
    const uint16_t* row = static_cast<const uint16_t*>(ts.x) + (int64_t)(t / ts.S) * ts.H;
    const int sl = t % ts.S;
    if (ts.bits == 2)
      xslice_one<2>(row, ts.H, sl, ts.table + (size_t)t * (2 * 16 + 4) * 32, lane);
    else if (ts.bits == 4)
      xslice_one<4>(row, ts.H, sl, ts.table + (size_t)t * (2 * 8 + 2) * 32, lane);
    else if (ts.bits == 8)
      xslice_one<8>(row, ts.H, sl, ts.table + (size_t)t * (2 * 4 + 2) * 32, lane);
  }
}

// ============================================================== staged GEMV kernel
// Persistent CTAs (one per SM).  Warp 16 is the producer: it reads the work
// description of up to 32 of its CTA's units at once (one unit per lane),
// then per unit (RU consecutive rows of NMAT matrices of one segment) lane
// 0 issues bulk copies of the contiguous packed rows and, when 16-byte
// aligned, of their bf16 scale and bias runs into a 4-stage shared-memory
// ring (otherwise the lanes copy those entry by entry); the unit's
// input/output vector references follow by cp.async.  Warp 17 issues the
// L2 prefetches.  A gate/up launch with a small step computes the step's
// routing and work lists itself in every CTA (the plan), lists the shared
// expert first and pre-issues its first unit before the dependency wait;
// the down launch's producer may start on the plan's published-lists flag.  Warps 0-15 form two consumer groups that take
// alternate units, so one group computes while the other waits for its
// stage.  In a group, warps 0..S*J-1 consume: warp (slice s, subset j)
// keeps its 32-chunk slice of the input vector in registers as fixed-point
// limbs, takes RU/J rows of each matrix from the stage (one 16-byte chunk
// per lane per row), reduces the eight row partials of each lane with the
// transposing butterfly, and the S slices are summed in fixed order through
// a double-buffered shared-memory exchange guarded by mbarriers (every wait
// bounded).
constexpr int GV_CW = 8;                  // consumer warps per group
constexpr int GV_GROUPS = 2;              // consumer groups, alternating units
constexpr int GV_PRODUCER = GV_GROUPS * GV_CW;  // producer warp
constexpr int GV_HELPER = GV_PRODUCER + 1;      // L2-prefetch warp
constexpr int GV_THREADS = (GV_PRODUCER + 2) * 32;
constexpr int GV_STAGES = 4;
constexpr int GV_STAGE_BYTES = 44 * 1024;
constexpr int GV_VMAX = 64;               // vector references staged per unit
constexpr int GV_UB_CAP = 2064;           // segment start units cached in shared memory

// What the consumers need to know about the unit in a stage.
struct GvMeta {
  int32_t r0, nrows, n_vec, vec_mode;
  const void* src_base;
  int64_t src_stride;
  float* dst_base;
  int64_t dst_stride;
  const VecRef* vecs;
};

struct GvSmem {
  static constexpr int META_STRIDE = 64;
  static constexpr int STAGE_OFF = 0;
  static constexpr int META_OFF = GV_STAGES * GV_STAGE_BYTES;
  static constexpr int VEC_OFF = META_OFF + GV_STAGES * META_STRIDE;
  static constexpr int UB_OFF = VEC_OFF + GV_STAGES * GV_VMAX * 16;
  static constexpr int BAR_OFF = UB_OFF + GV_UB_CAP * 4;
  static constexpr int N_BARS = 2 * GV_STAGES + 8 * GV_GROUPS;
  static constexpr int RED_OFF = BAR_OFF + N_BARS * 8;
  // the CTA's own plan (gate/up launch that computes it): segments, vector
  // references, counts, experts; then the fused combine's flags
  static constexpr int PSEG_OFF = RED_OFF + GV_GROUPS * 2 * GV_CW * 8 * 4;
  static constexpr int PVEC_OFF = PSEG_OFF + (((kFusedMaxPairs + 1) * (int)sizeof(Seg) + 15) & ~15);
  static constexpr int PCNT_OFF = PVEC_OFF + kFusedMaxPairs * 16;
  static constexpr int PEXP_OFF = PCNT_OFF + 8 * 4;
  static constexpr int FLAG_OFF = PEXP_OFF + kFusedMaxPairs * 4;
  // one input slice per consumer group, shared by its warps when they all
  // hold the same chunk (a single slice: S = 1)
  static constexpr int SL_OFF = (FLAG_OFF + GV_GROUPS * 4 + 15) & ~15;
  static constexpr int SL_WORDS = 64 * 32;
  static constexpr int BYTES = SL_OFF + GV_GROUPS * SL_WORDS * 4;
  static constexpr int RING_BYTES = GV_STAGES * GV_STAGE_BYTES;
};
static_assert(sizeof(GvMeta) <= GvSmem::META_STRIDE, "GvMeta exceeds its slot");
static_assert(GvSmem::BYTES <= 227 * 1024, "GEMV shared memory exceeds the per-CTA limit");
static_assert(kFusedMaxPairs + 1 <= GV_UB_CAP, "a fused plan's segment starts fit the cache");
static_assert(GvSmem::PSEG_OFF % 16 == 0 && GvSmem::PVEC_OFF % 16 == 0, "plan region alignment");

int gemv_threads() { return GV_THREADS; }
// A plan computed inside a gate/up launch keeps its scratch in stages 1..3
// of the ring: stage 0 may already be receiving the shared expert's unit.
int gemv_plan_scratch_cap() { return GvSmem::RING_BYTES - GV_STAGE_BYTES; }
static_assert(sizeof(VecRef) == 16, "VecRef is copied in 16-byte pieces");

// Last segment whose first unit is <= unit; p[i * stride] is segment i's
// first unit.
__device__ __forceinline__ int find_seg(const int32_t* p, int stride, int n, int unit) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p[(int64_t)mid * stride] <= unit) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// The prefetch ranges into L2 in 32 KB pieces; piece g of the concatenated
// ranges is issued by CTA g % gridDim.x (lane (g / gridDim.x) % 32 of the
// calling warp), so every SM's copy engine takes a share.
__device__ __forceinline__ void prefetch_ranges(const PrefetchRange* pf, int n) {
  constexpr int64_t PIECE = 32 * 1024;
  const int lane = threadIdx.x & 31;
  int64_t g0 = 0;
  for (int i = 0; i < n; ++i) {
    const int64_t pieces = (pf[i].bytes + PIECE - 1) / PIECE;
    int64_t g = g0 + ((blockIdx.x - g0 % gridDim.x) + gridDim.x) % gridDim.x;
    for (int64_t j = 0; g < g0 + pieces; g += gridDim.x, ++j) {
      if ((int)(j % 32) != lane) continue;
      const int64_t off = (g - g0) * PIECE;
      const int64_t len = min(PIECE, pf[i].bytes - off) & ~(int64_t)15;
      if (len > 0) tc::prefetch_l2((const uint8_t*)pf[i].p + off, (uint32_t)len);
    }
    g0 += pieces;
  }
}

// Matrix 0 (codes, scales, biases) of every listed segment into L2, spread
// over the CTAs the same way.
__device__ __forceinline__ void prefetch_segs(const Seg* segs, int n) {
  constexpr int64_t PIECE = 32 * 1024;
  const int lane = threadIdx.x & 31;
  int64_t g0 = 0;
  for (int i = 0; i < n; ++i) {
    const Seg& sg = segs[i];
    const int64_t gr = (int64_t)sg.out_dim * (sg.in_dim / sg.G);
    const void* p[3] = {sg.w[0], sg.s[0], sg.b[0]};
    const int64_t bytes[3] = {(int64_t)sg.out_dim * sg.in_dim * sg.bits / 8, gr * 2, gr * 2};
    for (int k = 0; k < 3; ++k) {
      const int64_t pieces = (bytes[k] + PIECE - 1) / PIECE;
      // first global index >= g0 owned by this CTA, then every gridDim.x
      int64_t g = g0 + ((blockIdx.x - g0 % gridDim.x) + gridDim.x) % gridDim.x;
      for (int64_t j = 0; g < g0 + pieces; g += gridDim.x, ++j) {
        if ((int)(j % 32) != lane) continue;
        const int64_t off = (g - g0) * PIECE;
        const int64_t len = min(PIECE, bytes[k] - off) & ~(int64_t)15;
        if (len > 0 && ((uintptr_t)p[k] & 15) == 0)
          tc::prefetch_l2((const uint8_t*)p[k] + off, (uint32_t)len);
      }
      g0 += pieces;
    }
  }
}

// Down projections (codes, scales, biases) of the listed experts and of
// the shared expert into L2, spread over the CTAs in 32 KB pieces.
__device__ __forceinline__ void prefetch_down(const DecodePlanArgs& p, const int32_t* ent,
                                              int n_ent) {
  constexpr int64_t PIECE = 32 * 1024;
  const int lane = threadIdx.x & 31;
  const int n_src = n_ent + (p.has_shared ? 1 : 0);
  int64_t g0 = 0;
  for (int i = 0; i < n_src; ++i) {
    const bool sh = i >= n_ent;
    const moeq_qtensor& t = sh ? p.sh_down : p.down;
    const int64_t e = sh ? 0 : ent[i];
    const int64_t gr = (int64_t)t.out_dim * (t.in_dim / t.group_size);
    const bool mx = t.format == MOEQ_FMT_MXFP4;
    const void* ptr[3] = {t.w + e * t.expert_stride_w, scale_at(t, e * t.expert_stride_sb),
                          mx ? nullptr : t.biases + e * t.expert_stride_sb};
    const int64_t bytes[3] = {(int64_t)t.out_dim * t.in_dim * t.bits / 8, gr * (mx ? 1 : 2),
                              mx ? 0 : gr * 2};
    for (int k = 0; k < 3; ++k) {
      const int64_t pieces = (bytes[k] + PIECE - 1) / PIECE;
      int64_t g = g0 + ((blockIdx.x - g0 % gridDim.x) + gridDim.x) % gridDim.x;
      for (int64_t j = 0; g < g0 + pieces; g += gridDim.x, ++j) {
        if ((int)(j % 32) != lane) continue;
        const int64_t off = (g - g0) * PIECE;
        const int64_t len = min(PIECE, bytes[k] - off) & ~(int64_t)15;
        if (len > 0 && ((uintptr_t)ptr[k] & 15) == 0)
          tc::prefetch_l2((const uint8_t*)ptr[k] + off, (uint32_t)len);
      }
      g0 += pieces;
    }
  }
}

__device__ __forceinline__ void plan_cta(const DecodePlanArgs& a, uint8_t* sm, int R,
                                         const PlanSinks& o);

// y[m][r] = sum_k w[m][k] d[m*K + k][r] (+ sigma[m] d[M*K + m][r]) (+ residual[m][r])
// for rows [r0, r0 + nrows), k in order; the same operations as k_combine.
// The d rows come from other CTAs of this launch: read through L2.
__device__ __forceinline__ void combine_rows(const CombineArgs& c, int r0, int nrows, int t,
                                             int nt) {
  const int total = c.M * nrows;
  for (int i = t; i < total; i += nt) {
    const int m = i / nrows;
    const int r = r0 + i % nrows;
    float acc = 0.0f;
    for (int k = 0; k < c.K; ++k)
      acc = fmaf(c.w[m * c.K + k], __ldcg(c.d + ((int64_t)m * c.K + k) * c.H + r), acc);
    if (c.has_shared)
      acc = fmaf(c.sigma[m], __ldcg(c.d + ((int64_t)c.M * c.K + m) * c.H + r), acc);
    if (c.residual) acc += c.residual[(int64_t)m * c.H + r];
    c.y[(int64_t)m * c.H + r] = acc;
  }
}

template <typename T>
__device__ __forceinline__ T shfl_ptr(T p, int src) {
  return reinterpret_cast<T>(__shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(p), src));
}

// Bounded wait (lane 0 polls, about two seconds) until *p == 1; the warp
// gets the outcome.  On timeout sets MOEQ_ERR_TIMEOUT.
__device__ __forceinline__ bool wait_flag(const int32_t* p, int* status) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) {
    const uint64_t t0 = tc::globaltimer_ns();
    int v;
    for (;;) {
      asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
      if (v == 1) break;
      __nanosleep(128);
      if (tc::globaltimer_ns() - t0 > 2000000000ull) {
        set_status(status, MOEQ_ERR_TIMEOUT);
        ok = false;
        break;
      }
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok;
}

// One unit of work as the producer issues it.
struct GvUnit {
  int r0, nrows, n_vec, vec_mode;
  const uint32_t* w[2];
  const uint16_t* s[2];
  const uint16_t* b[2];
  const void* src_base;
  int64_t src_stride;
  float* dst_base;
  int64_t dst_stride;
  const VecRef* vecs;
};

// Fills stage s with unit u (every producer lane calls; lane 0 writes the
// stage's description and issues the bulk copies): packed rows, then the
// scale/bias rows -- contiguous runs of nrows * gpr entries, bulk-copied
// when 16-byte aligned, else copied entry by entry -- and the unit's vector
// references when they live in global memory.
// (MX: one exponent byte per group in the scale rows, no bias rows.)
template <int NMAT, bool MX = false>
__device__ __forceinline__ void gv_issue(uint8_t* gsm, uint32_t sbase, uint64_t* full, uint32_t s,
                                         const GvUnit& u, int row_bytes, int gpr, int RU) {
  constexpr int ES = MX ? 1 : 2;  // bytes per scale entry
  const int lane = threadIdx.x & 31;
  const int codes_bytes = NMAT * RU * row_bytes;
  const int sb_bytes = RU * gpr * ES;
  const uint32_t st = sbase + s * GV_STAGE_BYTES;
  const int sb_n = u.nrows * gpr;
  auto srow = [&](int m) {
    return reinterpret_cast<const uint8_t*>(u.s[m]) + (int64_t)u.r0 * gpr * ES;
  };
  bool sb_bulk = ((sb_n * ES) & 15) == 0 && ((codes_bytes | sb_bytes) & 15) == 0;
#pragma unroll
  for (int m = 0; m < NMAT; ++m)
    sb_bulk = sb_bulk && ((((uintptr_t)srow(m)) |
                           (MX ? 0 : (uintptr_t)(u.b[m] + (int64_t)u.r0 * gpr))) & 15) == 0;
  if (lane == 0) {
    GvMeta* mt = reinterpret_cast<GvMeta*>(gsm + GvSmem::META_OFF + s * GvSmem::META_STRIDE);
    mt->r0 = u.r0;
    mt->nrows = u.nrows;
    mt->n_vec = u.n_vec;
    mt->vec_mode = u.vec_mode;
    mt->src_base = u.src_base;
    mt->src_stride = u.src_stride;
    mt->dst_base = u.dst_base;
    mt->dst_stride = u.dst_stride;
    mt->vecs = u.vecs;
    tc::mbar_arrive_expect_tx(
        &full[s], (uint32_t)(NMAT * u.nrows * row_bytes +
                             (sb_bulk ? (MX ? 1 : 2) * NMAT * sb_n * ES : 0)));
#pragma unroll
    for (int m = 0; m < NMAT; ++m) {
      tc::bulk_g2s(st + m * RU * row_bytes,
                   reinterpret_cast<const uint8_t*>(u.w[m]) + (int64_t)u.r0 * row_bytes,
                   (uint32_t)(u.nrows * row_bytes), &full[s]);
      if (sb_bulk) {
        tc::bulk_g2s(st + codes_bytes + m * sb_bytes, srow(m), (uint32_t)(sb_n * ES), &full[s]);
        if (!MX)
          tc::bulk_g2s(st + codes_bytes + (NMAT + m) * sb_bytes, u.b[m] + (int64_t)u.r0 * gpr,
                       (uint32_t)(sb_n * 2), &full[s]);
      }
    }
  }
  if (!sb_bulk && MX) {
#pragma unroll
    for (int m = 0; m < NMAT; ++m) {
      const uint8_t* s0 = srow(m);
      uint8_t* sd = gsm + s * GV_STAGE_BYTES + codes_bytes + m * sb_bytes;
      for (int e = lane; e < sb_n; e += 32) sd[e] = s0[e];
    }
  } else if (!sb_bulk) {
#pragma unroll
    for (int m = 0; m < NMAT; ++m) {
      const uint16_t* s0 = u.s[m] + (int64_t)u.r0 * gpr;
      const uint16_t* b0 = u.b[m] + (int64_t)u.r0 * gpr;
      uint16_t* sd =
          reinterpret_cast<uint16_t*>(gsm + s * GV_STAGE_BYTES + codes_bytes + m * sb_bytes);
      uint16_t* bd = reinterpret_cast<uint16_t*>(gsm + s * GV_STAGE_BYTES + codes_bytes +
                                                 (NMAT + m) * sb_bytes);
      for (int e = lane; e < sb_n; e += 32) {
        sd[e] = s0[e];
        bd[e] = b0[e];
      }
    }
  }
  if (u.vec_mode == 1 && u.n_vec <= GV_VMAX && !__isShared(u.vecs)) {
    const uint32_t vd = sbase + GvSmem::VEC_OFF + s * GV_VMAX * 16;
    for (int v = lane; v < u.n_vec; v += 32) tc::cp_async16(vd + 16 * v, u.vecs + v, 16);
  }
  if (sb_bulk) {
    tc::cp_async_arrive_noinc(&full[s]);
  } else {
    // plain shared-memory stores above: released by an ordinary arrive
    tc::cp_async_wait_all();
    tc::mbar_arrive(&full[s]);
  }
}

// MX: the segments' tensors are MX FP4 (4-bit E2M1 codes translated to
// q' = 2 e2m1 + 12 after the split, s = 2^(e - 128), b = -12 s per group).
template <int BITS, int NL, int NMAT, int SRC, int EPI, bool MX = false>
__global__ void __launch_bounds__(GV_THREADS, 1) k_gemv(const __grid_constant__ GemvArgs a) {
  static_assert(!MX || BITS == 4, "MX FP4 codes are 4-bit");
  constexpr int VPC = Chunk<BITS>::VPC;
  constexpr int NC = Chunk<BITS>::NC;
  constexpr int NB = SliceVec<BITS, NL>::NB;
  constexpr int RPW = 8 / NMAT;  // rows per warp per matrix and unit
  using SrcT = typename std::conditional<SRC == SRC_BF16, SrcBF16, SrcF32>::type;
  extern __shared__ __align__(128) uint8_t gsm[];
  VecRef* svec = reinterpret_cast<VecRef*>(gsm + GvSmem::VEC_OFF);
  int32_t* ub = reinterpret_cast<int32_t*>(gsm + GvSmem::UB_OFF);
  uint64_t* full = reinterpret_cast<uint64_t*>(gsm + GvSmem::BAR_OFF);
  uint64_t* empty = full + GV_STAGES;
  uint64_t* red_full = empty + GV_STAGES;           // [group][2]: slices 1..S-1 -> slice 0
  uint64_t* red_empty = red_full + 2 * GV_GROUPS;   // [group][2]: slice 0 -> slices 1..S-1
  uint64_t* slot_full = red_empty + 2 * GV_GROUPS;  // [group][2]: built slice -> group
  uint64_t* slot_empty = slot_full + 2 * GV_GROUPS; // [group][2]: group read it -> builder
  float* red = reinterpret_cast<float*>(gsm + GvSmem::RED_OFF);  // [group][2][GV_CW][8]
  const uint32_t sbase = tc::smem_u32(gsm);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.slices, J = a.subsets, RU = a.rows_per_unit;
  const int W = S * J;
  if (threadIdx.x == 0) {
    for (int i = 0; i < GV_STAGES; ++i) {
      tc::mbar_init(&full[i], 1 + 32);
      tc::mbar_init(&empty[i], GV_CW * 32);
    }
    for (int i = 0; i < 2 * GV_GROUPS; ++i) {
      tc::mbar_init(&red_full[i], (uint32_t)((S > 1 ? S - 1 : 1) * J * 8));
      tc::mbar_init(&red_empty[i], (uint32_t)(J * 8));
      tc::mbar_init(&slot_full[i], 32u);
      tc::mbar_init(&slot_empty[i], (uint32_t)((W > 1 ? W - 1 : 1) * 32));
    }
    tc::fence_mbar_init();
  }
  // fixed segments (router, qmv): no earlier kernel writes them or the
  // weights, so the producer starts streaming before the preceding kernel
  // ends; everyone else waits for it (input vectors, segment lists)
  const bool static_segs = !a.dyn_segs && !a.fused_plan;
  if (static_segs)
    for (int i = threadIdx.x; i < a.n_segs; i += blockDim.x) ub[i] = a.segs[i].unit_begin;
  __syncthreads();
  // ranges known before the preceding kernel ends (the shared expert's
  // weights) go to L2 while it finishes; the other warps do not wait for it
  if (warp == GV_HELPER && a.n_pf) prefetch_ranges(a.pf, a.n_pf);
  const int row_bytes = a.in_dim * BITS / 8;
  const int gpr = a.in_dim / a.G;
  const int cpr = a.in_dim / VPC;
  // stage layout: codes [NMAT][RU][row_bytes], scales [NMAT][RU*gpr], biases [NMAT][RU*gpr]
  const int codes_bytes = NMAT * RU * row_bytes;
  const int sb_bytes = RU * gpr * (MX ? 1 : 2);
  int* status = a.status;
  // a step planned in this launch lists the shared expert first; its
  // weights do not depend on the routing, so the producer puts this CTA's
  // first unit of it into stage 0 before the preceding kernel ends
  int preissued = 0;
  if constexpr (NMAT == 2) {
    const DecodePlanArgs& pl = a.plan;
    if (a.fused_plan && pl.has_shared && warp == GV_PRODUCER &&
        (int)blockIdx.x < pl.units_per_seg_gu_sh) {
      // the shared segment's unit blockIdx.x, mapped as the producer maps it
      const int nvc = seg_vchunks(pl.M, pl.sh_vpu_gu);
      const int rbi = (int)blockIdx.x / nvc;
      const int v0 = ((int)blockIdx.x - rbi * nvc) * pl.sh_vpu_gu;
      GvUnit gu;
      gu.r0 = rbi * RU;
      gu.nrows = min(RU, pl.sh_gate.out_dim - gu.r0);
      gu.n_vec = nvc > 1 ? min(pl.sh_vpu_gu, pl.M - v0) : pl.M;
      gu.vec_mode = 0;
      gu.w[0] = pl.sh_gate.w;
      gu.s[0] = pl.sh_gate.scales;
      gu.b[0] = pl.sh_gate.biases;
      gu.w[1] = pl.sh_up.w;
      gu.s[1] = pl.sh_up.scales;
      gu.b[1] = pl.sh_up.biases;
      gu.src_base = pl.x + (int64_t)v0 * pl.H;
      gu.src_stride = pl.H;
      gu.dst_base = pl.h + (int64_t)pl.M * pl.K * pl.I + (int64_t)v0 * pl.sh_gate.out_dim;
      gu.dst_stride = pl.sh_gate.out_dim;
      gu.vecs = nullptr;
      gv_issue<2, MX>(gsm, sbase, full, 0, gu, row_bytes, gpr, RU);
      preissued = 1;
    }
  }
  // the down launch's producer may start on the plan's flag (below)
  const bool early = a.flag_wait != nullptr;
  if (!((static_segs || early) && warp == GV_PRODUCER)) tc::grid_dep_wait();
  tc::grid_dep_launch();
  if (a.flag_reset && blockIdx.x == 0 && threadIdx.x == 0) *a.flag_reset = 0;

  // consumer geometry, and the input slice a consumer warp holds (built
  // early from token 0's row by the warps the fused plan leaves idle)
  const int grp = warp / GV_CW, cw = warp % GV_CW;
  const bool on_w = cw < W;
  const int sl = cw % S, j = cw / S;
  const int ch = sl * 32 + lane;
  const bool lane_on = on_w && ch < cpr;
  SliceVec<BITS, NL> sv;
  const void* cur_src = nullptr;
  // words of one lane's slice; token 0's slices, built by group 1 during a
  // fused plan, shared through shared memory when all S of them fit
  constexpr int SLW = NL * Chunk<BITS>::NC + 2 * SliceVec<BITS, NL>::NB;
  uint32_t* const sl_base = reinterpret_cast<uint32_t*>(gsm + GvSmem::SL_OFF);
  bool x_shared = false;

  const Seg* segs;
  int n_segs, total_units;
  bool timed_out_p = false;
  int32_t* pcnt = reinterpret_cast<int32_t*>(gsm + GvSmem::PCNT_OFF);
  int32_t* pexp = reinterpret_cast<int32_t*>(gsm + GvSmem::PEXP_OFF);
  if (static_segs) {
    segs = a.segs;
    n_segs = a.n_segs;
    total_units = a.total_units;
  } else {
    bool planned = false;
    if constexpr (NMAT == 2) {
      if (a.fused_plan) {
        // this CTA's copy of the step's plan, in shared memory; CTA 0 also
        // writes the routing, the down lists and zeroed combine counters
        Seg* psegs = reinterpret_cast<Seg*>(gsm + GvSmem::PSEG_OFF);
        PlanSinks o;
        memset(&o, 0, sizeof(o));
        o.segs_gu = psegs;
        o.count_gu = pcnt;
        o.vecs_gu = reinterpret_cast<VecRef*>(gsm + GvSmem::PVEC_OFF);
        o.experts = pexp;
        o.n_experts = pcnt + 4;
        o.ub_gu = ub;  // at most kFusedMaxPairs + 1 segments: within GV_UB_CAP
        if (blockIdx.x == 0) {
          o.idx = a.plan.idx_out;
          o.w = a.plan.w_out;
          o.sigma = a.plan.sigma;
          o.segs_dn = a.plan.segs_dn;
          o.count_dn = a.plan.count_dn;
          o.vecs_dn = a.plan.vecs_dn;
          o.ctr = a.plan.ctr;
          o.n_ctr = a.plan.n_ctr;
        }
        // the scratch of the plan lives in stages 1..3 of the (still unused)
        // ring; stage 0 may be receiving the shared expert's unit
        o.shared_first = a.plan.has_shared;
        const int pr = plan_route_warps(a.plan.M, a.plan.E, GV_THREADS / 32);
        // consumer warps the plan does not use build their slice of token
        // 0's row now (the first vector of the shared expert's units, and
        // of every unit when M = 1); the others build it after the plan
        // (not with a single slice, S = 1: there the group's warps share one
        // build, which needs every warp of the group to take the same path)
        if (S > 1 && warp >= max(pr, 4 * a.plan.M) && warp < GV_PRODUCER && on_w) {
          build_slice<BITS, NL, SrcT>(a.plan.x, ch, lane_on, sv);
          cur_src = a.plan.x;
        }
        // when the whole of group 1 is idle during the plan, its first
        // subset's warps leave their slices for the routing warps, which
        // copy them after the plan instead of loading the row themselves
        x_shared = S > 1 && S * SLW <= 2 * GvSmem::SL_WORDS / 32 && GV_CW >= max(pr, 4 * a.plan.M);
        if (x_shared && grp == 1 && j == 0 && on_w)
          slice_store<BITS, NL>(sl_base + sl * SLW * 32, sv, lane);
        plan_cta(a.plan, gsm + GV_STAGE_BYTES, pr, o);
        if (a.flag_set && blockIdx.x == 0 && threadIdx.x == 0) {
          // CTA 0's lists (written before plan_cta's final barrier) are
          // visible GPU-wide before the flag
          __threadfence();
          atomicExch(a.flag_set, 1);
        }
        segs = psegs;
        n_segs = pcnt[0];
        total_units = pcnt[1];
        planned = true;
      }
    }
    if (!planned) {
      if (early && warp == GV_PRODUCER) {
        // wait (bounded) until the plan's down lists are published
        if (!wait_flag(a.flag_wait, status)) timed_out_p = true;
      }
      segs = a.dyn_segs;
      n_segs = timed_out_p ? 0 : a.dyn_count[0];
      total_units = timed_out_p ? 0 : a.dyn_count[1];
    }
    if (planned) {
      // the plan wrote the segment starts; its final barrier published them
    } else if (early) {
      // the producer does not join: the others cache the segment starts
      if (warp != GV_PRODUCER) {
        if (n_segs <= GV_UB_CAP)
          for (int i = threadIdx.x; i < n_segs; i += GV_PRODUCER * 32) ub[i] = segs[i].unit_begin;
        // warps 0..15 and 17 (the helper is warp 17: its 32 threads count)
        tc::named_sync(1, (GV_THREADS - 32));
      }
    } else {
      if (n_segs <= GV_UB_CAP)
        for (int i = threadIdx.x; i < n_segs; i += blockDim.x) ub[i] = segs[i].unit_begin;
      __syncthreads();
    }
  }
  const bool ub_cached = n_segs <= GV_UB_CAP && !(early && warp == GV_PRODUCER);


  if (warp == GV_HELPER) {
    // ------------------------------------------------------------ L2 prefetch
    if (a.fused_plan) prefetch_down(a.plan, pexp, pcnt[4]);
    else if (a.pf_segs) prefetch_segs(a.pf_segs, a.pf_count[0]);
    // the router launch: the token slice table of the gate/up launch
    if constexpr (NMAT == 1 && SRC == SRC_BF16 && !MX)
      if (a.xsl.table) build_xslices(a.xsl);
  } else if (warp == GV_PRODUCER) {
    // ------------------------------------------------------------ producer
    uint32_t it = preissued;
    bool dead = false;
    for (int base = blockIdx.x + preissued * gridDim.x; base < total_units && !dead;
         base += 32 * gridDim.x) {
      // lane u describes unit base + u * gridDim.x
      const int mine = base + lane * gridDim.x;
      int r0 = 0, nrows = 0, n_vec = 0, vec_mode = 0;
      const uint32_t* w[2] = {nullptr, nullptr};
      const uint16_t* sp[2] = {nullptr, nullptr};
      const uint16_t* bp[2] = {nullptr, nullptr};
      const void* src_base = nullptr;
      float* dst_base = nullptr;
      int64_t src_stride = 0, dst_stride = 0;
      const VecRef* vecs = nullptr;
      if (mine < total_units) {
        const int si = ub_cached ? find_seg(ub, 1, n_segs, mine)
                                 : find_seg(&segs[0].unit_begin, (int)(sizeof(Seg) / 4), n_segs,
                                            mine);
        const Seg& sg = segs[si];
        const int u0 = ub_cached ? ub[si] : sg.unit_begin;
        // a segment split by vectors: units (row block, run of vpu vectors)
        const int nvc = seg_vchunks(sg.n_vec, sg.vpu);
        const int rbi = (mine - u0) / nvc;
        const int v0 = (mine - u0 - rbi * nvc) * sg.vpu;  // 0 when nvc == 1
        r0 = rbi * RU;
        nrows = min(RU, sg.out_dim - r0);
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          w[m] = sg.w[m];
          sp[m] = sg.s[m];
          bp[m] = sg.b[m];
        }
        n_vec = nvc > 1 ? min(sg.vpu, sg.n_vec - v0) : sg.n_vec;
        vec_mode = sg.vec_mode;
        src_base = sg.src_base;
        src_stride = sg.src_stride;
        dst_base = sg.dst_base;
        dst_stride = sg.dst_stride;
        vecs = sg.vecs;
        if (v0 > 0) {
          if (vec_mode == 0) {
            src_base = static_cast<const char*>(src_base) +
                       (int64_t)v0 * src_stride * (SRC == SRC_BF16 ? 2 : 4);
            dst_base += (int64_t)v0 * dst_stride;
          } else {
            vecs += v0;
          }
        }
      }
      const int nb = min(32, (total_units - base + (int)gridDim.x - 1) / (int)gridDim.x);
      for (int u = 0; u < nb; ++u, ++it) {
        const uint32_t s = it % GV_STAGES, ph = (it / GV_STAGES) & 1u;
        if (!tc::mbar_wait(&empty[s], ph ^ 1u, status)) {
          dead = true;
          break;
        }
        GvUnit gu;
        gu.r0 = __shfl_sync(0xffffffffu, r0, u);
        gu.nrows = __shfl_sync(0xffffffffu, nrows, u);
        gu.n_vec = __shfl_sync(0xffffffffu, n_vec, u);
        gu.vec_mode = __shfl_sync(0xffffffffu, vec_mode, u);
        gu.vecs = shfl_ptr(vecs, u);
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          gu.w[m] = shfl_ptr(w[m], u);
          gu.s[m] = shfl_ptr(sp[m], u);
          gu.b[m] = shfl_ptr(bp[m], u);
        }
        gu.src_base = shfl_ptr(src_base, u);
        gu.dst_base = shfl_ptr(dst_base, u);
        gu.src_stride = __shfl_sync(0xffffffffu, src_stride, u);
        gu.dst_stride = __shfl_sync(0xffffffffu, dst_stride, u);
        gv_issue<NMAT, MX>(gsm, sbase, full, s, gu, row_bytes, gpr, RU);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    // group grp takes every GV_GROUPS-th unit of the CTA (stages grp, grp + GV_GROUPS, ...)
    int gi[2];
#pragma unroll
    for (int pb = 0; pb < 2; ++pb) gi[pb] = (ch * VPC + (pb < NB ? pb : 0) * kXBlock) / a.G;
    // an input row's slice: copied from the table an earlier launch built
    // (token rows: the router launch; hidden rows: the slice launch before
    // the down launch), else converted here
    auto vec_slice = [&](const void* src) {
      constexpr bool kTable = !MX && NL == 2 && !stream_bits(BITS) &&
                              ((NMAT == 2 && SRC == SRC_BF16) || (NMAT == 1 && SRC == SRC_F32));
      if constexpr (kTable) {
        if (a.xsl.table) {
          using T = typename std::conditional<SRC == SRC_BF16, uint16_t, float>::type;
          const int64_t off = static_cast<const T*>(src) - static_cast<const T*>(a.xsl.x);
          if (off >= 0 && off % a.xsl.H == 0 && off / a.xsl.H < a.xsl.M) {
            const int64_t m = off / a.xsl.H;
            slice_load<BITS, NL>(a.xsl.table + (m * a.xsl.S + sl) * SLW * 32, sv, lane);
            return;
          }
        }
      }
      build_slice<BITS, NL, SrcT>(src, ch, lane_on, sv);
    };
    // With a single slice (S = 1) every warp of the group holds the same
    // chunk: warp 0 of the group converts each new vector and hands the
    // slice to the others through a double-buffered slot (full: warp 0's
    // 32 lanes arrive; empty: the other warps' lanes arrive after copying;
    // every wait bounded).  Build b uses buffer b & 1.
    const bool share_build =
        !a.xsl.table && S == 1 && W > 1 && 2 * SLW * 32 <= GvSmem::SL_WORDS;
    uint32_t* const sl_grp = sl_base + grp * GvSmem::SL_WORDS;
    uint32_t nbuild = 0;
    bool slot_timeout = false;
    auto group_build = [&](const void* src) {
      const uint32_t b = nbuild++, buf = b & 1u;
      uint32_t* slot = sl_grp + buf * SLW * 32;
      if (cw == 0) {
        if (b >= 2 && !slot_timeout)
          slot_timeout = !tc::mbar_wait(&slot_empty[grp * 2 + buf], ((b >> 1) + 1u) & 1u, status);
        vec_slice(src);
        slice_store<BITS, NL>(slot, sv, lane);
        __syncwarp();
        tc::mbar_arrive(&slot_full[grp * 2 + buf]);
      } else {
        if (!slot_timeout)
          slot_timeout = !tc::mbar_wait(&slot_full[grp * 2 + buf], (b >> 1) & 1u, status);
        slice_load<BITS, NL>(slot, sv, lane);
        __syncwarp();
        tc::mbar_arrive(&slot_empty[grp * 2 + buf]);
      }
    };
    // the first vector's slice is built while the first stage streams in
    if (on_w) {
      const int u0 = blockIdx.x + grp * gridDim.x;
      if (u0 < total_units) {
        const int si = ub_cached ? find_seg(ub, 1, n_segs, u0)
                                 : find_seg(&segs[0].unit_begin, (int)(sizeof(Seg) / 4), n_segs,
                                            u0);
        const Seg& sg = segs[si];
        if (sg.n_vec > 0) {
          const int nvc = seg_vchunks(sg.n_vec, sg.vpu);
          const int lu = u0 - (ub_cached ? ub[si] : sg.unit_begin);
          const int v0 = (lu - (lu / nvc) * nvc) * sg.vpu;  // 0 when nvc == 1
          const void* src0 =
              sg.vec_mode == 0
                  ? static_cast<const void*>(static_cast<const char*>(sg.src_base) +
                                             (int64_t)v0 * sg.src_stride *
                                                 (SRC == SRC_BF16 ? 2 : 4))
                  : sg.vecs[v0].src;
          if (src0 != cur_src) {
            if (x_shared && src0 == (const void*)a.plan.x) {
              slice_load<BITS, NL>(sl_base + sl * SLW * 32, sv, lane);
            } else if (share_build) {
              group_build(src0);
            } else {
              vec_slice(src0);
            }
            cur_src = src0;
          }
        }
      }
    }
    // After a wait that ran out, every later wait is skipped and no vector
    // is processed; all waits are bounded, so the CTA always ends.
    bool timed_out = false;
    uint32_t it = grp, rc = 0;
    for (int unit = blockIdx.x + grp * gridDim.x; unit < total_units;
         unit += GV_GROUPS * gridDim.x, it += GV_GROUPS) {
      const uint32_t s = it % GV_STAGES, ph = (it / GV_STAGES) & 1u;
      if (!timed_out) timed_out = !tc::mbar_wait(&full[s], ph, status);
      const GvMeta* mp = reinterpret_cast<const GvMeta*>(gsm + GvSmem::META_OFF +
                                                         s * GvSmem::META_STRIDE);
      const int n_vec = timed_out ? 0 : mp->n_vec;
      const int r0 = timed_out ? 0 : mp->r0, nrows = timed_out ? 0 : mp->nrows;
      const uint32_t st = sbase + s * GV_STAGE_BYTES;
      if (on_w && n_vec > 0) {
        const int vec_mode = mp->vec_mode;
        const VecRef* vl = (vec_mode == 1 && n_vec <= GV_VMAX && !__isShared(mp->vecs))
                               ? svec + s * GV_VMAX
                               : mp->vecs;
        for (int v = 0; v < n_vec && !timed_out; ++v) {
          const void* src;
          float* dst;
          if (vec_mode == 0) {
            src = (SRC == SRC_BF16)
                      ? (const void*)((const uint16_t*)mp->src_base + (int64_t)v * mp->src_stride)
                      : (const void*)((const float*)mp->src_base + (int64_t)v * mp->src_stride);
            dst = mp->dst_base + (int64_t)v * mp->dst_stride;
          } else {
            src = vl[v].src;
            dst = vl[v].dst;
          }
          if (src != cur_src) {
            if (share_build) group_build(src);
            else vec_slice(src);
            cur_src = src;
          }
          float acc[8];
#pragma unroll
          for (int m = 0; m < NMAT; ++m)
#pragma unroll
            for (int i = 0; i < RPW; ++i) {
              const int row = j * RPW + i;
              const bool ok = lane_on && row < nrows;
              uint4 wv = make_uint4(0, 0, 0, 0);
              constexpr bool STREAM = stream_bits(BITS);  // cross-word packed codes
              uint32_t ws3[STREAM ? Chunk<BITS>::BYTES / 4 : 1] = {};
              float s2[2] = {0.f, 0.f}, b2[2] = {0.f, 0.f};
              if (ok) {
                const uint32_t ca = st + (m * RU + row) * row_bytes + ch * Chunk<BITS>::BYTES;
                if constexpr (BITS == 3 || BITS == 5) {  // 4-byte aligned runs
#pragma unroll
                  for (int q = 0; q < Chunk<BITS>::BYTES / 4; ++q) ws3[q] = lds32_gv(ca + 4 * q);
                } else if constexpr (BITS == 6) {  // 8-byte aligned runs
#pragma unroll
                  for (int q = 0; q < 3; ++q) {
                    const uint2 v = lds64_gv(ca + 8 * q);
                    ws3[2 * q] = v.x;
                    ws3[2 * q + 1] = v.y;
                  }
                } else {
                  wv = gq_lds128(ca);
                }
                if (MX) {
                  // one group per 32-value chunk: s = 2^(e - 128), b = -12 s
                  const uint32_t e = lds_u8(st + codes_bytes + m * sb_bytes + row * gpr + gi[0]);
                  s2[0] = 0.5f * mx_scale(e);
                  b2[0] = -12.0f * s2[0];
                } else {
                  const uint32_t sd = st + codes_bytes + m * sb_bytes + row * gpr * 2;
                  const uint32_t bd = st + codes_bytes + (NMAT + m) * sb_bytes + row * gpr * 2;
#pragma unroll
                  for (int pb = 0; pb < NB; ++pb) {
                    s2[pb] = bf16_bits_to_float(lds_u16(sd + gi[pb] * 2));
                    b2[pb] = bf16_bits_to_float(lds_u16(bd + gi[pb] * 2));
                  }
                }
              }
              uint32_t c[NC];
              if constexpr (STREAM) Chunk<BITS>::split_stream(ws3, c);
              else Chunk<BITS>::split(wv, c);
              if (MX) {
#pragma unroll
                for (int k = 0; k < NC; ++k) c[k] = mx_q8(c[k]);
              }
              acc[m * RPW + i] = chunk_contrib<BITS, NL>(c, sv, s2, b2);
            }
          float tot = transpose_reduce<8>(acc);  // lane l: value l % 8
          if (S > 1) {
            // slices 1..S-1 hand their partials to slice 0, which adds them
            // in slice order
            const uint32_t buf = rc & 1u, rph = (rc >> 1) & 1u;
            ++rc;
            float* rb = red + (grp * 2 + buf) * GV_CW * 8;
            uint64_t* rf = &red_full[grp * 2 + buf];
            uint64_t* re = &red_empty[grp * 2 + buf];
            if (sl != 0) {
              if (!tc::mbar_wait(re, rph ^ 1u, status)) timed_out = true;
              if (lane < 8) {
                rb[cw * 8 + lane] = tot;
                tc::mbar_arrive(rf);
              }
            } else {
              if (!tc::mbar_wait(rf, rph, status)) timed_out = true;
              if (lane < 8) {
                float t = tot;
                for (int q = 1; q < S; ++q) t += rb[(j * S + q) * 8 + lane];
                tot = t;
                tc::mbar_arrive(re);
              }
            }
          }
          if (EPI == EPI_SWIGLU) {
            // values 0..3: gate rows, 4..7: up rows of the same four rows
            const float u = __shfl_sync(0xffffffffu, tot, (lane + RPW) & 31);
            const int row = j * RPW + lane;
            if (sl == 0 && lane < RPW && row < nrows)
              dst[r0 + row] = __fdividef(tot, 1.0f + __expf(-tot)) * u;
          } else {
            const int row = j * RPW + lane;
            if (sl == 0 && lane < 8 && row < nrows) {
              dst[r0 + row] = tot;
              // visible GPU-wide before the row block is counted as done
              if (a.fuse_combine) __threadfence();
            }
          }
        }
      }
      tc::mbar_arrive(&empty[s]);
      if (NMAT == 1 && EPI == EPI_PLAIN && a.fuse_combine) {
        // the group's stores of this unit are done; the CTA that brings the
        // row block's count to the number of segments sums the block
        tc::named_sync(2 + grp, GV_CW * 32);
        int* flag = reinterpret_cast<int*>(gsm + GvSmem::FLAG_OFF) + grp;
        if (cw == 0 && lane == 0) {
          int last = 0;
          if (n_vec > 0) {
            // every segment covers every row block: one unit each, the
            // shared one sh_units (split by tokens)
            const int target = n_segs + (a.comb.has_shared ? a.comb.sh_units - 1 : 0);
            last = atomicAdd(&a.comb.ctr[r0 / RU], 1) == target - 1;
            if (last) __threadfence();
          }
          *flag = last;
        }
        tc::named_sync(2 + grp, GV_CW * 32);
        if (*flag) combine_rows(a.comb, r0, nrows, cw * 32 + lane, GV_CW * 32);
      }
    }
  }
}

template <int BITS, int NL, int NMAT, int SRC, int EPI, bool MX = false>
static cudaError_t launch_one(const GemvArgs& a, int grid, cudaStream_t st) {
  auto kern = k_gemv<BITS, NL, NMAT, SRC, EPI, MX>;
  // the shared-memory opt-in is per device
  static std::atomic<bool> attr[kMaxDevices];
  int dev;
  if (!current_device(dev)) return cudaErrorInvalidDevice;
  if (!attr[dev].load(std::memory_order_acquire)) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GvSmem::BYTES);
    if (e != cudaSuccess) return e;
    attr[dev].store(true, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(GV_THREADS);
  cfg.dynamicSmemBytes = GvSmem::BYTES;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

// Slices of fp32 rows (the hidden rows of a decode step) in the down
// launch's format, one warp per (row, slice).
template <int B>
__global__ void __launch_bounds__(128) k_hslices(const TokenSlices ts) {
  constexpr int SLW = 2 * Chunk<B>::NC + 2 * SliceVec<B, 2>::NB;
  // the down launch may be scheduled at once (its producer starts on the
  // plan's flag); the rows are read after the gate/up launches end
  tc::grid_dep_launch();
  tc::grid_dep_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (t >= ts.M * ts.S) return;
  const int sl = t % ts.S, ch = sl * 32 + lane;
  const float* row = static_cast<const float*>(ts.x) + (int64_t)(t / ts.S) * ts.H;
  SliceVec<B, 2> sv;
  build_slice<B, 2, SrcF32>(row, ch, ch < ts.H / Chunk<B>::VPC, sv);
  slice_store<B, 2>(ts.table + (size_t)t * SLW * 32, sv, lane);
}

cudaError_t launch_hslices(const TokenSlices& ts, cudaStream_t st) {
  const int tasks = ts.M * ts.S;
  if (!ts.table || tasks <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((tasks + 3) / 4);
  cfg.blockDim = dim3(128);
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  if (ts.bits == 2) return cudaLaunchKernelEx(&cfg, k_hslices<2>, ts);
  if (ts.bits == 4) return cudaLaunchKernelEx(&cfg, k_hslices<4>, ts);
  if (ts.bits == 8) return cudaLaunchKernelEx(&cfg, k_hslices<8>, ts);
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemv(int bits, int nl, int nmat, int src, const GemvArgs& a, int grid,
                        cudaStream_t st) {
  if (grid <= 0) return cudaSuccess;
  if (stream_bits(bits)) {  // cross-word packed codes
    if (nmat == 2 && nl == 2 && src == SRC_BF16)
      return bits == 3 ? launch_one<3, 2, 2, SRC_BF16, EPI_SWIGLU>(a, grid, st)
           : bits == 5 ? launch_one<5, 2, 2, SRC_BF16, EPI_SWIGLU>(a, grid, st)
                       : launch_one<6, 2, 2, SRC_BF16, EPI_SWIGLU>(a, grid, st);
    if (nmat == 1 && nl == 3 && src == SRC_BF16)
      return bits == 3 ? launch_one<3, 3, 1, SRC_BF16, EPI_PLAIN>(a, grid, st)
           : bits == 5 ? launch_one<5, 3, 1, SRC_BF16, EPI_PLAIN>(a, grid, st)
                       : launch_one<6, 3, 1, SRC_BF16, EPI_PLAIN>(a, grid, st);
    if (nmat == 1 && nl == 2 && src == SRC_F32)
      return bits == 3 ? launch_one<3, 2, 1, SRC_F32, EPI_PLAIN>(a, grid, st)
           : bits == 5 ? launch_one<5, 2, 1, SRC_F32, EPI_PLAIN>(a, grid, st)
                       : launch_one<6, 2, 1, SRC_F32, EPI_PLAIN>(a, grid, st);
    return cudaErrorInvalidValue;
  }
  if (a.fmt == MOEQ_FMT_MXFP4) {  // 4-bit E2M1 experts (and qmv)
    if (bits != 4) return cudaErrorInvalidValue;
    if (nmat == 2 && nl == 2 && src == SRC_BF16)
      return launch_one<4, 2, 2, SRC_BF16, EPI_SWIGLU, true>(a, grid, st);
    if (nmat == 1 && nl == 3 && src == SRC_BF16)
      return launch_one<4, 3, 1, SRC_BF16, EPI_PLAIN, true>(a, grid, st);
    if (nmat == 1 && nl == 2 && src == SRC_F32)
      return launch_one<4, 2, 1, SRC_F32, EPI_PLAIN, true>(a, grid, st);
    return cudaErrorInvalidValue;
  }
  // instantiated forms: router / qmv (3 limbs, bf16 tokens), gate/up + SwiGLU
  // (2 limbs, bf16 tokens), down (2 limbs, fp32 hidden rows)
  if (nmat == 2 && nl == 2 && src == SRC_BF16) {
    if (bits == 8) return launch_one<8, 2, 2, SRC_BF16, EPI_SWIGLU>(a, grid, st);
    if (bits == 4) return launch_one<4, 2, 2, SRC_BF16, EPI_SWIGLU>(a, grid, st);
    return launch_one<2, 2, 2, SRC_BF16, EPI_SWIGLU>(a, grid, st);
  }
  if (nmat == 1 && nl == 3 && src == SRC_BF16) {
    if (bits == 8) return launch_one<8, 3, 1, SRC_BF16, EPI_PLAIN>(a, grid, st);
    if (bits == 4) return launch_one<4, 3, 1, SRC_BF16, EPI_PLAIN>(a, grid, st);
    return launch_one<2, 3, 1, SRC_BF16, EPI_PLAIN>(a, grid, st);
  }
  if (nmat == 1 && nl == 2 && src == SRC_F32) {
    if (bits == 8) return launch_one<8, 2, 1, SRC_F32, EPI_PLAIN>(a, grid, st);
    if (bits == 4) return launch_one<4, 2, 1, SRC_F32, EPI_PLAIN>(a, grid, st);
    return launch_one<2, 2, 1, SRC_F32, EPI_PLAIN>(a, grid, st);
  }
  return cudaErrorInvalidValue;
}

// ============================================================== top-K routing
// One warp per token; each warp stages its token's logits in shared memory.
__global__ void __launch_bounds__(256) k_route_topk(const float* __restrict__ logits, int M, int E,
                                                    int K, int renorm, float scale,
                                                    int32_t* __restrict__ idx,
                                                    float* __restrict__ w) {
  extern __shared__ __align__(16) uint8_t rsm[];
  const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int words = (E + 31) >> 5;
  const int wbytes = ((words * 4 + 15) & ~15) + E * 4;
  uint32_t* taken = reinterpret_cast<uint32_t*>(rsm + warp * wbytes);
  float* row = reinterpret_cast<float*>(rsm + warp * wbytes + ((words * 4 + 15) & ~15));
  const int t = blockIdx.x * nw + warp;
  if (t >= M) return;
  route_token_warp(logits + (int64_t)t * E, E, K, renorm, scale, idx + (int64_t)t * K,
                   w + (int64_t)t * K, row, taken);
}

// Warps per routing CTA so that the staged rows fit 48 KB.
int route_warps_per_cta(int E) {
  const int wbytes = (((E + 31) / 32 * 4 + 15) & ~15) + E * 4;
  int w = (48 * 1024) / wbytes;
  return w < 1 ? 1 : (w > 8 ? 8 : w);
}

cudaError_t launch_route_topk(const float* logits, int M, int E, int K, int renorm, float scale,
                              int32_t* idx, float* w, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  const int warps = route_warps_per_cta(E);
  const int grid = (M + warps - 1) / warps;
  const size_t smem = (size_t)warps * ((((E + 31) / 32 * 4 + 15) & ~15) + (size_t)E * 4);
  k_route_topk<<<grid, warps * 32, smem, st>>>(logits, M, E, K, renorm, scale, idx, w);
  return cudaGetLastError();
}

// ============================================================== decode plan
__host__ __device__ int plan_route_warps(int M, int E, int nwarps) {
  int r = kPlanStageBytes / (E * 4);
  if (r < 1) r = 1;
  if (r > nwarps) r = nwarps;
  if (r > M) r = M;
  return r;
}

// Scratch of one CTA's plan: routing results, sort keys and the staged
// logit rows of R routing warps.
struct PlanScratch {
  int32_t* sidx;      // [n] routed experts
  float* sw;          // [n] routed weights
  float* ssig;        // [M] shared-expert gate values
  int32_t* key;       // [n] expert of pair
  int32_t* sorted;    // [n] pairs sorted by (expert, pair)
  int32_t* head;      // [n] 1 at the first pair of an expert
  int32_t* entry_of;  // [n] entry index of sorted position
  uint32_t* taken;    // [R][words] routing bitmaps
  float* rows;        // [R][E] staged logits (16-byte aligned)
  int32_t* cidx;      // [M][4][K] candidates of the parts of a token
  float* cval;        // [M][4][K]
  float* pmax;        // [M][4] largest value of each part
  float* psum;        // [M][4] sum of exp(v - part maximum)
};

__host__ __device__ size_t plan_scratch_bytes(int M, int K, int E, int R) {
  const size_t n = (size_t)M * K;
  size_t b = (7 * n + (size_t)M) * 4 + (size_t)R * ((E + 31) / 32) * 4;
  b = (b + 15) & ~(size_t)15;
  return b + (size_t)R * E * 4 + (size_t)M * 4 * K * 8 + (size_t)M * 4 * 8;
}

__device__ __forceinline__ PlanScratch plan_scratch(uint8_t* sm, int M, int K, int E, int R) {
  const int n = M * K;
  PlanScratch p;
  p.sidx = reinterpret_cast<int32_t*>(sm);
  p.sw = reinterpret_cast<float*>(p.sidx + n);
  p.ssig = p.sw + n;
  p.key = reinterpret_cast<int32_t*>(p.ssig + M);
  p.sorted = p.key + n;
  p.head = p.sorted + n;
  p.entry_of = p.head + n;
  p.taken = reinterpret_cast<uint32_t*>(p.entry_of + n);
  size_t off = (size_t)(7 * n + M) * 4 + (size_t)R * ((E + 31) / 32) * 4;
  off = (off + 15) & ~(size_t)15;
  p.rows = reinterpret_cast<float*>(sm + off);
  p.cidx = reinterpret_cast<int32_t*>(p.rows + (size_t)R * E);
  p.cval = reinterpret_cast<float*>(p.cidx + (size_t)M * 4 * K);
  p.pmax = p.cval + (size_t)M * 4 * K;
  p.psum = p.pmax + (size_t)M * 4;
  return p;
}

// Vector references of the pair at sorted position i (pair p).
__device__ __forceinline__ void write_pair_lists(const DecodePlanArgs& a, const PlanSinks& o, int i,
                                                 int p) {
  const int t = p / a.K;
  if (o.vecs_gu) {
    o.vecs_gu[i].src = a.x + (int64_t)t * a.H;
    o.vecs_gu[i].dst = a.h + (int64_t)p * a.I;
  }
  if (o.vecs_dn) {
    o.vecs_dn[i].src = a.h + (int64_t)p * a.I;
    o.vecs_dn[i].dst = a.d + (int64_t)p * a.H;
  }
}

// Gate/up and down segments of entry u: expert e, its `cnt` pairs starting
// at sorted position i.
__device__ __forceinline__ void write_expert_segs(const DecodePlanArgs& a, const PlanSinks& o, int i,
                                                  int u, int e, int cnt) {
  if (o.experts) o.experts[u] = e;
  if (o.segs_gu) {
    // shared expert first: the routed entries follow it
    const int gi = o.shared_first ? u + 1 : u;
    const int gu0 = o.shared_first ? a.units_per_seg_gu_sh : 0;
    Seg g;
    g.w[0] = a.gate.w + (int64_t)e * a.gate.expert_stride_w;
    g.s[0] = scale_at(a.gate, (int64_t)e * a.gate.expert_stride_sb);
    g.b[0] = a.gate.biases + (int64_t)e * a.gate.expert_stride_sb;
    g.w[1] = a.up.w + (int64_t)e * a.up.expert_stride_w;
    g.s[1] = scale_at(a.up, (int64_t)e * a.up.expert_stride_sb);
    g.b[1] = a.up.biases + (int64_t)e * a.up.expert_stride_sb;
    g.out_dim = a.I;
    g.in_dim = a.H;
    g.G = a.gate.group_size;
    g.bits = a.gate.bits;
    g.n_vec = cnt;
    g.unit_begin = gu0 + u * a.units_per_seg_gu;
    g.vec_mode = 1;
    g.vpu = 0;
    g.src_base = nullptr;
    g.src_stride = 0;
    g.dst_base = nullptr;
    g.dst_stride = 0;
    g.vecs = o.vecs_gu + i;
    o.segs_gu[gi] = g;
    if (o.ub_gu) o.ub_gu[gi] = g.unit_begin;
  }
  if (o.segs_dn) {
    Seg dn;
    dn.w[0] = dn.w[1] = a.down.w + (int64_t)e * a.down.expert_stride_w;
    dn.s[0] = dn.s[1] = scale_at(a.down, (int64_t)e * a.down.expert_stride_sb);
    dn.b[0] = dn.b[1] = a.down.biases + (int64_t)e * a.down.expert_stride_sb;
    dn.out_dim = a.H;
    dn.in_dim = a.I;
    dn.G = a.down.group_size;
    dn.bits = a.down.bits;
    dn.n_vec = cnt;
    dn.unit_begin = u * a.units_per_seg_dn;
    dn.vec_mode = 1;
    dn.vpu = 0;
    dn.src_base = nullptr;
    dn.src_stride = 0;
    dn.dst_base = nullptr;
    dn.dst_stride = 0;
    dn.vecs = o.vecs_dn + i;
    o.segs_dn[u] = dn;
  }
}

// Computes the routing and the grouped work plan of a decode step in one
// CTA (every thread of the CTA calls it; it synchronises the CTA):
//   1. routes the M tokens (or takes the given routing) and the
//      shared-expert gate;
//   2. sorts the M*K (token, slot) pairs by expert (stable);
//   3. lists one gate/up segment and one down segment per distinct expert,
//      then the shared expert's segments, with the (input, output) vector
//      references of every pair in sorted order.
// Each output group of `o` is written only if its pointer is non-null.
__device__ __forceinline__ void plan_cta(const DecodePlanArgs& a, uint8_t* sm, int R,
                                         const PlanSinks& o) {
  const int M = a.M, K = a.K, n = M * K;
  const int tid = threadIdx.x, warp = tid >> 5, nthr = blockDim.x;
  const int words = (a.E + 31) >> 5;
  const PlanScratch ps = plan_scratch(sm, M, K, a.E, R);

  // 1. routing: for few tokens and many experts, four warps per token each
  //    select candidates from a quarter of the experts and one merges them;
  //    otherwise R warps, one token each at a time
  const int WT = (a.logits && a.E >= 256 && M <= 8 && M * 4 <= (nthr >> 5)) ? 4 : 1;
  // the shared expert's gate, by the CTA's last warp (idle in a GEMV
  // launch's plan) while the others route
  if (a.has_shared && a.sg_logit && warp == (nthr >> 5) - 1)
    for (int t = tid & 31; t < M; t += 32) ps.ssig[t] = 1.0f / (1.0f + expf(-a.sg_logit[t]));
  if (WT > 1) {
    if (warp < M * WT) {
      const int t = warp / WT, part = warp % WT;
      int32_t* cidx = ps.cidx + t * 4 * K;
      float* cval = ps.cval + t * 4 * K;
      route_part(a.logits + (int64_t)t * a.E, a.E, K, a.router_scale, part, WT, cidx + part * K,
                 cval + part * K, ps.pmax + t * 4 + part, ps.psum + t * 4 + part);
      tc::named_sync(4 + t, WT * 32);
      if (part == 0)
        route_merge_parts(cidx, cval, WT * K, K, a.renorm, ps.pmax + t * 4, ps.psum + t * 4, WT,
                          ps.sidx + t * K, ps.sw + t * K);
    }
  } else if (a.logits) {
    if (warp < R)
      for (int t = warp; t < M; t += R)
        route_token_warp(a.logits + (int64_t)t * a.E, a.E, K, a.renorm, a.router_scale,
                         ps.sidx + t * K, ps.sw + t * K, ps.rows + (int64_t)warp * a.E,
                         ps.taken + warp * words);
  } else {
    for (int p = tid; p < n; p += nthr) {
      ps.sidx[p] = a.idx_in[p];
      ps.sw[p] = a.w_in[p];
    }
  }
  __syncthreads();
  if (o.sigma && a.has_shared && a.sg_logit)
    for (int t = tid; t < M; t += nthr) o.sigma[t] = ps.ssig[t];
  for (int i = tid; i < o.n_ctr; i += nthr) o.ctr[i] = 0;

  // 2.-3. (the entry count is known to thread 0 afterwards)
  int n_entries = 0;
  if (n <= 32) {
    // warp 0 alone: rank of (expert, pair) by shuffles, runs of equal
    // experts by a ballot of their first positions
    if (warp == 0) {
      const int lane = tid;
      int e = lane < n ? ps.sidx[lane] : 0;
      if (lane < n && o.idx) {
        o.idx[lane] = e;
        o.w[lane] = ps.sw[lane];
      }
      if (lane < n && (e < 0 || e >= a.E)) {
        set_status(a.status, MOEQ_ERR_INVALID_ARG);
        e = 0;
      }
      int rank = 0;
      for (int q = 0; q < n; ++q) {
        const int eq = __shfl_sync(0xffffffffu, e, q);
        rank += (eq < e) || (eq == e && q < lane);
      }
      if (lane < n) ps.sorted[rank] = lane;
      __syncwarp();
      const int sp = lane < n ? ps.sorted[lane] : 0;  // pair at sorted position `lane`
      const int se = __shfl_sync(0xffffffffu, e, sp);
      const int prev = __shfl_up_sync(0xffffffffu, se, 1);
      const bool head = lane < n && (lane == 0 || se != prev);
      const uint32_t hb = __ballot_sync(0xffffffffu, head);
      const uint32_t upto = lane == 31 ? 0xffffffffu : ((2u << lane) - 1u);
      const uint32_t later = hb & ~upto;
      if (lane < n) write_pair_lists(a, o, lane, sp);
      if (head)
        write_expert_segs(a, o, lane, __popc(hb & upto) - 1, se,
                          (later ? __ffs(later) - 1 : n) - lane);
      n_entries = __popc(hb);
    }
  } else {
    // stable sort of pairs by expert: rank of (expert, pair)
    for (int p = tid; p < n; p += nthr) {
      int e = ps.sidx[p];
      if (o.idx) {
        o.idx[p] = e;
        o.w[p] = ps.sw[p];
      }
      if (e < 0 || e >= a.E) {
        set_status(a.status, MOEQ_ERR_INVALID_ARG);
        e = 0;
      }
      ps.key[p] = e;
    }
    __syncthreads();
    for (int p = tid; p < n; p += nthr) {
      const int e = ps.key[p];
      int rank = 0;
      for (int q = 0; q < n; ++q) {
        const int f = ps.key[q];
        rank += (f < e) || (f == e && q < p);
      }
      ps.sorted[rank] = p;
    }
    __syncthreads();
    for (int i = tid; i < n; i += nthr)
      ps.head[i] = (i == 0) || (ps.key[ps.sorted[i]] != ps.key[ps.sorted[i - 1]]);
    __syncthreads();
    // entry index = inclusive prefix count of heads - 1 (scan by warp 0)
    if (warp == 0) {
      int run = 0;
      for (int base = 0; base < n; base += 32) {
        const int i = base + (tid & 31);
        int h = (i < n) ? ps.head[i] : 0;
        int incl = h;
#pragma unroll
        for (int sft = 1; sft < 32; sft <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, sft);
          if ((tid & 31) >= sft) incl += y;
        }
        if (i < n) ps.entry_of[i] = run + incl - 1;
        run += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
    __syncthreads();
    n_entries = n > 0 ? ps.entry_of[n - 1] + 1 : 0;
    for (int i = tid; i < n; i += nthr) {
      const int p = ps.sorted[i];
      write_pair_lists(a, o, i, p);
      if (ps.head[i]) {
        int cnt = 1;
        while (i + cnt < n && !ps.head[i + cnt]) ++cnt;
        write_expert_segs(a, o, i, ps.entry_of[i], ps.key[p], cnt);
      }
    }
  }
  if (tid == 0) {
    int nseg_gu = n_entries, nseg_dn = n_entries;
    int units_gu = n_entries * a.units_per_seg_gu, units_dn = n_entries * a.units_per_seg_dn;
    int sep_gu[2] = {0, 0}, sep_dn[2] = {0, 0};
    if (a.has_shared) {
      // the shared expert: all M tokens, strided rows after the M*K pair rows;
      // same format as the routed experts: appended to the routed list;
      // otherwise stored at index n (one past the largest routed list) for
      // a launch of its own
      const bool same_gu = a.shared_same_gu != 0;
      const bool same_dn = a.shared_same_dn != 0;
      if (o.segs_gu) {
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
        g.bits = a.sh_gate.bits;
        g.n_vec = M;
        g.vec_mode = 0;
        g.vpu = a.sh_vpu_gu;
        g.src_base = a.x;
        g.src_stride = a.H;
        g.dst_base = a.h + (int64_t)n * a.I;
        g.dst_stride = a.sh_gate.out_dim;
        g.vecs = nullptr;
        if (o.shared_first) {
          g.unit_begin = 0;
          o.segs_gu[0] = g;
          if (o.ub_gu) o.ub_gu[0] = 0;
        } else {
          g.unit_begin = same_gu ? units_gu : 0;
          o.segs_gu[same_gu ? n_entries : n] = g;
          if (o.ub_gu && same_gu) o.ub_gu[n_entries] = g.unit_begin;
        }
      }
      if (o.segs_dn) {
        Seg dn;
        dn.w[0] = dn.w[1] = a.sh_down.w;
        dn.s[0] = dn.s[1] = a.sh_down.scales;
        dn.b[0] = dn.b[1] = a.sh_down.biases;
        dn.out_dim = a.H;
        dn.in_dim = a.sh_down.in_dim;
        dn.G = a.sh_down.group_size;
        dn.bits = a.sh_down.bits;
        dn.n_vec = M;
        dn.vec_mode = 0;
        dn.vpu = a.sh_vpu_dn;
        dn.src_base = a.h + (int64_t)n * a.I;
        dn.src_stride = a.sh_gate.out_dim;
        dn.dst_base = a.d + (int64_t)n * a.H;
        dn.dst_stride = a.H;
        dn.vecs = nullptr;
        dn.unit_begin = same_dn ? units_dn : 0;
        o.segs_dn[same_dn ? n_entries : n] = dn;
      }
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
    if (o.count_gu) {
      o.count_gu[0] = nseg_gu;
      o.count_gu[1] = units_gu;
      o.count_gu[2] = sep_gu[0];
      o.count_gu[3] = sep_gu[1];
    }
    if (o.count_dn) {
      o.count_dn[0] = nseg_dn;
      o.count_dn[1] = units_dn;
      o.count_dn[2] = sep_dn[0];
      o.count_dn[3] = sep_dn[1];
    }
    if (o.n_experts) *o.n_experts = n_entries;
  }
  __syncthreads();
}

// The plan as a kernel of its own (one CTA), writing every list to global
// memory for the GEMV launches that follow.
constexpr int kPlanThreads = 256;
__global__ void __launch_bounds__(kPlanThreads) k_decode_plan(const __grid_constant__ DecodePlanArgs a) {
  extern __shared__ __align__(16) uint8_t psm[];
  tc::grid_dep_wait();
  tc::grid_dep_launch();
  PlanSinks o;
  memset(&o, 0, sizeof(o));
  o.idx = a.idx_out;
  o.w = a.w_out;
  o.sigma = a.sigma;
  o.segs_gu = a.segs_gu;
  o.count_gu = a.count_gu;
  o.vecs_gu = a.vecs_gu;
  o.segs_dn = a.segs_dn;
  o.count_dn = a.count_dn;
  o.vecs_dn = a.vecs_dn;
  o.ctr = a.ctr;
  o.n_ctr = a.n_ctr;
  plan_cta(a, psm, plan_route_warps(a.M, a.E, kPlanThreads / 32), o);
}

cudaError_t launch_decode_plan(const DecodePlanArgs& a, cudaStream_t st) {
  const int R = plan_route_warps(a.M, a.E, kPlanThreads / 32);
  const size_t smem = plan_scratch_bytes(a.M, a.K, a.E, R);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_decode_plan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kPlanThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_decode_plan, a);
}

// ============================================================== wait self test
// Warp 0 waits on an mbarrier phase that never completes, warp 1 on a flag
// that stays 0; both waits are the bounded ones the kernels above use.
__device__ int32_t g_never_set = 0;

__global__ void __launch_bounds__(64) k_wait_probe(int* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    tc::mbar_wait(&bar, 0, status);
  } else {
    wait_flag(&g_never_set, status);
  }
}

cudaError_t launch_wait_probe(int* status, cudaStream_t st) {
  k_wait_probe<<<1, 64, 0, st>>>(status);
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
