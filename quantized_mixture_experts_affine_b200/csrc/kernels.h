// Host-side launchers shared between the C ABI (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moeq.h"

namespace moeq {

// Argument checks shared by the layer entry points (api.cu): the layer, M,
// the mode, and the x / y / residual pointers, before any workspace check.
moeq_status forward_arg_check(const moeq_layer* L, const uint16_t* x, int32_t M, float* y,
                              const float* residual, int32_t mode);

// Diagnostics (api.cu): launch counter and the optional profiling events.
void count_launches(int n);
cudaError_t profile_mark(bool start, cudaStream_t st);

// ------------------------------------------------------------------ GEMV segments
// One vector of a segment: its source row and its output row.
struct VecRef {
  const void* src;  // bf16 row (x) or fp32 row (h), in_dim values
  float* dst;       // fp32 output row, out_dim values
};

// A run of rows of one or two matrices (gate and up) multiplied with a set
// of vectors.  Vectors are either strided (src_base + i*src_stride) or an
// explicit VecRef list.
struct Seg {
  const uint32_t* w[2];
  const uint16_t* s[2];
  const uint16_t* b[2];
  int32_t out_dim;
  int32_t in_dim;
  int32_t G;
  int32_t bits;
  int32_t n_vec;
  int32_t unit_begin;  // first work unit of this segment
  int32_t vec_mode;    // 0 strided, 1 list
  int32_t vpu;         // vectors per work unit (0: all n_vec in one unit)
  const void* src_base;
  int64_t src_stride;  // elements
  float* dst_base;
  int64_t dst_stride;  // elements
  const VecRef* vecs;
};

constexpr int kInlineSegs = 4;
constexpr int kMaxPrefetch = 10;

// A global range to pull into L2 at kernel start (16-byte aligned).
struct PrefetchRange {
  const void* p;
  int64_t bytes;
};

struct DecodePlanArgs {
  const float* logits;      // [M][E] fp32, or null when idx/w are given
  const float* sg_logit;    // [M] shared-gate logit, or null
  const int32_t* idx_in;    // [M][K] when logits == null
  const float* w_in;
  int32_t M, E, K, renorm;
  float router_scale;
  int32_t* idx_out;         // [M][K]
  float* w_out;             // [M][K]
  const uint16_t* x;        // [M][H] bf16
  int32_t H, I;
  int32_t has_shared;
  moeq_qtensor gate, up, down, sh_gate, sh_up, sh_down;
  float* h;                 // [(M*K + M)][I] fp32 hidden rows (pairs, then shared rows)
  float* d;                 // [(M*K + M)][H] fp32 down rows
  float* sigma;             // [M] sigmoid gate values
  Seg* segs_gu;             // gate/up segments
  int32_t* count_gu;        // [4]: segs, units; separate shared list: segs, units
  Seg* segs_dn;             // down segments
  int32_t* count_dn;        // [4]
  VecRef* vecs_gu;          // [(M*K + M)]
  VecRef* vecs_dn;
  int32_t* ctr;             // [n_ctr] per-row-block counters of the fused combine, zeroed
  int32_t n_ctr;
  int32_t units_per_seg_gu; // computed on the host from the shapes
  int32_t units_per_seg_dn;
  int32_t units_per_seg_gu_sh;  // row blocks x vector splits of the shared gate/up
  int32_t units_per_seg_dn_sh;  // row blocks x vector splits of the shared down
  int32_t shared_same_gu;   // 1: the shared gate/up segment joins the routed launch
  int32_t shared_same_dn;   // 1: the shared down segment joins the routed launch
  int32_t sh_vpu_gu;        // tokens per unit of the shared gate/up segment (0: all M)
  int32_t sh_vpu_dn;        // tokens per unit of the shared down segment (0: all M)
  int* status;
};

// Where a CTA's plan goes (each group written only when its pointer is set).
struct PlanSinks {
  int32_t* idx;
  float* w;
  float* sigma;
  Seg* segs_gu;
  int32_t* count_gu;
  VecRef* vecs_gu;
  Seg* segs_dn;
  int32_t* count_dn;
  VecRef* vecs_dn;
  int32_t* ctr;             // set to zero
  int32_t n_ctr;
  int32_t* experts;         // [entries] expert of each entry
  int32_t* n_experts;
  // gate/up list with the shared expert first (segment 0, units from 0) and
  // the routed entries after it
  int32_t shared_first;
  // first unit of every gate/up segment (a GEMV's cached segment starts)
  int32_t* ub_gu;
};

// Staged logits of the plan's routing warps: at most this many bytes.
constexpr int kPlanStageBytes = 64 * 1024;
// Largest M*K whose plan the gate/up GEMV computes itself (in every CTA).
constexpr int kFusedMaxPairs = 64;
__host__ __device__ int plan_route_warps(int M, int E, int nwarps);
// Units per row block of a segment whose n_vec vectors are split into runs
// of vpu (vpu = 0: one unit takes them all).
__host__ __device__ inline int seg_vchunks(int n_vec, int vpu) {
  return (vpu > 0 && vpu < n_vec) ? (n_vec + vpu - 1) / vpu : 1;
}
__host__ __device__ size_t plan_scratch_bytes(int M, int K, int E, int R);

// The weighted combine done by the down GEMV: the CTA that completes the
// last segment of a row block writes y for those rows.
struct CombineArgs {
  const float* w;           // [M][K] routed weights
  const float* sigma;       // [M] shared-expert gate values
  const float* residual;    // [M][H] or null
  float* y;                 // [M][H]
  const float* d;           // [(M*K + M)][H] down rows
  int32_t* ctr;             // [row blocks], zero on entry
  int32_t M, K, H, has_shared;
  int32_t sh_units;         // units per row block of the shared segment (>= 1)
};

// Input rows of a GEMV launch in its fixed-point format (2 limbs, `bits`-bit
// chunks), [row][slice][word][lane], as slice_load reads them: the token
// rows (bf16) for the gate/up launch, the hidden rows (fp32) for the down
// launch.
struct TokenSlices {
  uint32_t* table;          // null: unused
  const void* x;            // the rows they were built from, [M][H]
  int32_t M, H, bits, S;    // S: 32-chunk slices per row
};

struct GemvArgs {
  Seg segs[kInlineSegs];    // used when dyn_segs == nullptr
  int32_t n_segs;
  int32_t total_units;      // used when dyn_segs == nullptr
  const Seg* dyn_segs;      // device list written by the decode plan
  const int32_t* dyn_count; // [0] = number of segments, [1] = total units
  // shape shared by every segment of the launch
  int32_t in_dim;
  int32_t G;
  int32_t fmt;              // MOEQ_FMT_* of every segment's tensors
  int32_t slices;           // S: 32-chunk slices per row
  int32_t subsets;          // J: row subsets (warps = S * J)
  int32_t rows_per_unit;    // RU = J * (8 / NMAT)
  PrefetchRange pf[kMaxPrefetch];
  int32_t n_pf;
  // segments (device list) whose matrix 0 is pulled into L2 at kernel start,
  // spread over all CTAs (the down projections, from the gate/up launch)
  const Seg* pf_segs;
  const int32_t* pf_count;
  int* status;
  // gate/up launch: every CTA computes the step's plan itself (M*K <= kFusedMaxPairs)
  int32_t fused_plan;
  DecodePlanArgs plan;
  // down launch: weighted combine by the last CTA of each row block
  int32_t fuse_combine;
  CombineArgs comb;
  // the step's "down lists published" flag: the router launch sets it to 0
  // after its dependency wait, the gate/up launch that plans the step sets
  // it to 1 once CTA 0 has written the down lists, and the down launch's
  // producer starts on it instead of on the dependency wait (null: unused)
  int32_t* flag_reset;
  int32_t* flag_set;
  const int32_t* flag_wait;
  // the step's token slices (router launch: writes them; gate/up launch:
  // copies a token's slice instead of converting its row again)
  TokenSlices xsl;
};

enum GemvEpi { EPI_PLAIN = 0, EPI_SWIGLU = 1 };
enum GemvSrc { SRC_BF16 = 0, SRC_F32 = 1 };

// Work shape of the staged GEMV for rows of `in_dim` codes at `bits`.
struct GemvShape {
  int S;   // slices of 32 chunks per row
  int J;   // row subsets
  int RU;  // rows per unit
};
GemvShape gemv_shape(int in_dim, int bits, int nmat, int G);
bool gemv_fits(int in_dim, int bits, int nmat, int G);
int gemv_threads();     // threads of a GEMV CTA
int gemv_plan_scratch_cap();  // bytes a plan computed inside a GEMV launch may use
int gemv_units(int out_dim, const GemvShape& sh);
// Words of one token's slices in the gate/up launch's format (2 limbs) for
// rows of H codes at `bits` (0: no table for this width).
size_t gemv_xslice_words(int H, int bits);
// Slices of the M fp32 rows of ts.x (stride ts.H) into ts.table, after the
// preceding launch (the gate/up launches that wrote the rows).
cudaError_t launch_hslices(const TokenSlices& ts, cudaStream_t st);

// Launch with programmatic dependent launch (the kernel waits for its
// predecessor's results before reading them).
cudaError_t launch_gemv(int bits, int nl, int nmat, int src, const GemvArgs& a, int grid,
                        cudaStream_t st);

// ------------------------------------------------------------------ routing
int route_warps_per_cta(int E);  // warps of a routing CTA (staged logits fit 48 KB)
cudaError_t launch_route_topk(const float* logits, int M, int E, int K, int renorm, float scale,
                              int32_t* idx, float* w, cudaStream_t st);

// Decode plan: top-K for M tokens, then the grouped work lists for the
// gate/up and down GEMVs (one segment per distinct expert, plus the shared
// expert), written into `plan` (device workspace).

cudaError_t launch_decode_plan(const DecodePlanArgs& a, cudaStream_t st);

// ------------------------------------------------------------------ one-launch decode (M = 1)
constexpr int kFusedMaxK = 8;       // top-K of the one-launch decode
constexpr int kFusedMaxGrid = 256;  // CTAs (flags per array in the workspace)

// Unit kinds of the one-launch decode, in issue order within a CTA.
enum FzKindId { FZ_ROUTER = 0, FZ_SGATE = 1, FZ_SHGU = 2, FZ_SHDN = 3, FZ_GU = 4, FZ_DN = 5 };
// Tensors of the one-launch decode; each has a code map, a scale map and a
// bias map (map index = 3 * tensor + 0, 1, 2).
enum FzMapId { FZM_ROUTER = 0, FZM_SGATE, FZM_SHG, FZM_SHU, FZM_SHD, FZM_G, FZM_U, FZM_D, FZM_N };

// Geometry of one unit kind.  A unit holds nbox boxes of RB rows (gate/up:
// a gate box and an up box of RB intermediate indices); a row's codes are
// cut into S slabs of slab_bytes, stored at a padded stride of slab_bytes +
// 16 per (slab, row): box = [S][RB][slab_bytes + 16], box_bytes long,
// placed box_stride bytes apart (a multiple of 128: tensor copies land on
// 128-byte aligned shared memory).
// A box's scale (bias) rows follow the code boxes: [RB][gpr + 8] bf16 each
// (the 8 padding entries read as zeros), sb_bytes long, sb_stride apart.
struct FzKind {
  int32_t row_bytes, gpr, RB, S, slab_bytes, box_bytes, box_stride, nbox, gran;
  int32_t sb_bytes, sb_stride;
};

struct FzMaps {
  CUtensorMap tm[3 * FZM_N];
};

struct FusedArgs {
  moeq_qtensor router, sgate, gate, up, down, sh_gate, sh_up, sh_down;
  int32_t H, I, Ish, E, K, renorm, has_shared, route_from_router;
  float router_scale;
  const uint16_t* x;        // [H] bf16
  const int32_t* idx_in;    // [K] when the routing is given
  const float* w_in;
  const float* residual;    // [H] or null
  float* y;                 // [H]
  int32_t* idx_out;         // [K] or null
  float* w_out;
  uint64_t* gen;            // previous call's tag (workspace word 0)
  uint64_t* flag1;          // [grid] router logits / shared hidden values published
  uint64_t* flag2;          // [grid] routed hidden values published
  float* logits;            // [E + 1]: router logits, then the shared gate logit
  float* hsh;               // [Ish] shared hidden values
  float* h;                 // [K][I] routed hidden values
  int* status;
  FzKind kind[6];
  int32_t dgran, drows_max, stage_bytes;
  int32_t tab_x8, tab_xe, tab_xs, tab_hs, tab_h1;  // bytes of each input table (tab_h1: one expert)
  int32_t off_args, off_ring, off_xR, off_xE, off_xS, off_hS, off_hl, off_units, off_red,
      off_dpart, off_bar, smem_bytes;
  int32_t bits[3];          // router, shared (0: none), routed experts
};

// Shape part of the arguments, the code tensor maps and the shared-memory
// layout for `grid` CTAs; false when the layer's formats or sizes are
// outside what the one-launch decode handles (the multi-launch path runs
// instead).
bool fused_decode_plan(const moeq_layer* L, int grid, bool route_from_router, FusedArgs& a,
                       FzMaps& m);
int fused_decode_threads();
cudaError_t launch_fused_decode(const FusedArgs& a, const FzMaps& m, int grid, cudaStream_t st);

// ------------------------------------------------------------------ single-token decode
// Three lean launches for M = 1 (k_single.cu): router rows, then top-K with
// the gate/up rows and SwiGLU, then the down rows with the combine.  Each
// CTA bulk-copies whole row blocks of every matrix it reads into shared
// memory at once; blocks that do not depend on the preceding launch are
// issued before its dependency wait.
constexpr int kS1MaxK = 16;

struct S1Args {
  int32_t H, I, Ish, E, K, has_shared, renorm;
  float router_scale;
  moeq_qtensor router, sg, gate, up, down, sh_gate, sh_up, sh_down;
  // row blocks: a matrix's rows split over a grid in units of q rows (the
  // smallest count whose scales fill whole 16-byte runs)
  int32_t qR, qG, qGs, qD;
  int32_t gridR, gridG, gridD;
  int32_t r_rows_max, g_sh_max, g_rt_max, d_rows_max;  // largest block of a CTA
  int32_t nsR, nsG, nsD;                               // input slices per lane
  uint32_t smem_R, smem_G, smem_D;                     // dynamic shared memory
  // G: warps per row pair (routed, shared layout); byte offsets of the
  // routed and shared input slices, the partial sums and the row blocks
  int32_t g_sgc_r, g_sgc_s;
  uint32_t g_sl_r, g_sl_s, g_red, g_blk;
  // D: bytes of one hidden vector's slices; byte offset of the row blocks
  uint32_t d_set_bytes, d_blk;
  const uint16_t* x;      // [H] bf16
  const float* residual;  // [H] or null
  float* y;               // [H]
  float* logits;          // [E]
  float* sg_logit;        // [1]
  const int32_t* idx_in;  // [K] the caller's routing, or null: the router's
  const float* w_in;      // [K]
  int32_t* idx;           // [K] routing out (the experts the launches use)
  float* w;               // [K]
  float* sigma;           // [1]
  float* h;               // [K*I + Ish] hidden rows (routed, then shared)
  int* status;
};

// Shape part of the arguments for this layer on `sms` SMs; false when the
// layer's formats or sizes are outside what the three launches take (the
// general decode path runs it then).
bool single_decode_plan(const moeq_layer* L, int sms, S1Args& a);
cudaError_t launch_single_router(const S1Args& a, cudaStream_t st);
cudaError_t launch_single_gateup(const S1Args& a, cudaStream_t st);
cudaError_t launch_single_down(const S1Args& a, cudaStream_t st);

// Codes and/or fp32 weights of one matrix.
cudaError_t launch_dequant(const moeq_qtensor& t, int expert, uint8_t* q_out, float* w_out,
                           cudaStream_t st);

// y[t] = sum_k w[t][k] * d[t*K + k] + sigma[t] * d[M*K + t] + residual[t]
// Failure-path self test: bounded waits that run out (MOEQ_ERR_TIMEOUT).
cudaError_t launch_wait_probe(int* status, cudaStream_t st);

cudaError_t launch_combine(const float* d, const float* w, const float* sigma, int has_shared,
                           const float* residual, float* y, int M, int K, int H, cudaStream_t st);

}  // namespace moeq
