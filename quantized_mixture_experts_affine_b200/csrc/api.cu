// C ABI of libmoeq.so (include/moeq.h): argument checks, workspace layout
// and the launch sequences of the decode and prefill paths.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "moeq.h"
#include "prefill.h"

#define MOEQ_API extern "C" __attribute__((visibility("default")))

using namespace moeq;

// ------------------------------------------------------------------ device status word
__device__ int g_moeq_status;

static int* status_ptr() {
  static std::mutex mu;
  static int* ptrs[kMaxDevices] = {nullptr};
  int dev;
  if (!current_device(dev)) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_moeq_status) != cudaSuccess) return nullptr;
    ptrs[dev] = (int*)p;
  }
  return ptrs[dev];
}

// ------------------------------------------------------------------ diagnostics
static std::atomic<uint64_t> g_launches{0};
static thread_local cudaEvent_t t_prof_start = nullptr, t_prof_stop = nullptr;

namespace moeq {
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
cudaError_t profile_mark(bool start, cudaStream_t st) {
  cudaEvent_t e = start ? t_prof_start : t_prof_stop;
  if (!e) return cudaSuccess;
  // inside a stream capture a plain record only orders the capture; the
  // external flag makes it a timestamp node of the graph
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t err = cudaStreamIsCapturing(st, &cs);
  if (err != cudaSuccess) return err;
  if (cs == cudaStreamCaptureStatusActive)
    return cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
  return cudaEventRecord(e, st);
}
}  // namespace moeq

// ------------------------------------------------------------------ checks
static bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// Shape/format checks of one tensor.  n_mats: experts addressable (>= 1).
static bool is_mx(const moeq_qtensor& t) { return t.format == MOEQ_FMT_MXFP4; }

static moeq_status check_tensor(const moeq_qtensor* t, int64_t n_mats) {
  if (!t) return MOEQ_ERR_INVALID_ARG;
  if (t->format != MOEQ_FMT_AFFINE && t->format != MOEQ_FMT_MXFP4) return MOEQ_ERR_UNSUPPORTED;
  const bool mx = is_mx(*t);
  if (!t->w || !t->scales || (!mx && !t->biases)) return MOEQ_ERR_INVALID_ARG;
  if (t->out_dim <= 0 || t->in_dim <= 0 || n_mats <= 0) return MOEQ_ERR_INVALID_ARG;
  if (t->bits < 2 || t->bits > 8 || t->bits == 7)
    return MOEQ_ERR_UNSUPPORTED;
  if (t->group_size != 32 && t->group_size != 64 && t->group_size != 128)
    return MOEQ_ERR_UNSUPPORTED;
  if (mx && (t->bits != 4 || t->group_size != 32)) return MOEQ_ERR_UNSUPPORTED;
  const int vpc = chunk_values(t->bits);  // codes per chunk (16 bytes; 3, 5, 6 bits: 32 codes)
  if (t->in_dim % t->group_size || t->in_dim % vpc) return MOEQ_ERR_ALIGNMENT;
  // rows of whole 16-byte runs (3 and 5 bits: in_dim % 128, 6 bits: % 64)
  if (((int64_t)t->in_dim * t->bits / 8) % 16) return MOEQ_ERR_ALIGNMENT;
  if (!aligned(t->w, 16) || (!mx && (!aligned(t->scales, 2) || !aligned(t->biases, 2))))
    return MOEQ_ERR_ALIGNMENT;
  const int64_t words = (int64_t)t->out_dim * t->in_dim * t->bits / 32;
  const int64_t groups = (int64_t)t->out_dim * (t->in_dim / t->group_size);
  if (n_mats > 1) {
    if (t->expert_stride_w < words || t->expert_stride_sb < groups) return MOEQ_ERR_INVALID_ARG;
    if ((t->expert_stride_w * 4) % 16) return MOEQ_ERR_ALIGNMENT;
  }
  return MOEQ_OK;
}

// Decode GEMV limit: a row is cut into at most 8 slices of 512 bytes.
static int slices_of(const moeq_qtensor& t) {
  const int cpr = t.in_dim / chunk_values(t.bits);
  return (cpr + 31) / 32;
}

static moeq_status check_layer(const moeq_layer* L) {
  if (!L) return MOEQ_ERR_INVALID_ARG;
  const int H = L->hidden, I = L->inter, E = L->n_experts, K = L->top_k;
  if (H <= 0 || I <= 0 || E <= 0 || K <= 0) return MOEQ_ERR_INVALID_ARG;
  if (K > E) return MOEQ_ERR_INVALID_ARG;
  if (K > kMaxK || E > kMaxE) return MOEQ_ERR_UNSUPPORTED;
  moeq_status s;
  if ((s = check_tensor(&L->router, 1)) != MOEQ_OK) return s;
  if ((s = check_tensor(&L->gate, E)) != MOEQ_OK) return s;
  if ((s = check_tensor(&L->up, E)) != MOEQ_OK) return s;
  if ((s = check_tensor(&L->down, E)) != MOEQ_OK) return s;
  if (L->router.out_dim != E || L->router.in_dim != H) return MOEQ_ERR_INVALID_ARG;
  if (L->gate.out_dim != I || L->gate.in_dim != H) return MOEQ_ERR_INVALID_ARG;
  if (L->up.out_dim != I || L->up.in_dim != H) return MOEQ_ERR_INVALID_ARG;
  if (L->down.out_dim != H || L->down.in_dim != I) return MOEQ_ERR_INVALID_ARG;
  if (L->gate.bits != L->up.bits || L->gate.group_size != L->up.group_size ||
      L->gate.format != L->up.format)
    return MOEQ_ERR_UNSUPPORTED;
  // MX FP4 is an expert-weight format: the router stays affine
  if (is_mx(L->router)) return MOEQ_ERR_UNSUPPORTED;
  if (L->has_shared != 0 && L->has_shared != 1) return MOEQ_ERR_INVALID_ARG;
  if (L->has_shared) {
    if ((s = check_tensor(&L->sh_gate, 1)) != MOEQ_OK) return s;
    if ((s = check_tensor(&L->sh_up, 1)) != MOEQ_OK) return s;
    if ((s = check_tensor(&L->sh_down, 1)) != MOEQ_OK) return s;
    if ((s = check_tensor(&L->sh_expert_gate, 1)) != MOEQ_OK) return s;
    const int Is = L->sh_gate.out_dim;
    if (L->sh_gate.in_dim != H || L->sh_up.in_dim != H || L->sh_up.out_dim != Is)
      return MOEQ_ERR_INVALID_ARG;
    if (L->sh_down.out_dim != H || L->sh_down.in_dim != Is) return MOEQ_ERR_INVALID_ARG;
    if (L->sh_expert_gate.out_dim != 1 || L->sh_expert_gate.in_dim != H)
      return MOEQ_ERR_INVALID_ARG;
    if (L->sh_gate.bits != L->sh_up.bits || L->sh_gate.group_size != L->sh_up.group_size ||
        L->sh_gate.format != L->sh_up.format)
      return MOEQ_ERR_UNSUPPORTED;
    if (is_mx(L->sh_expert_gate)) return MOEQ_ERR_UNSUPPORTED;
  }
  return MOEQ_OK;
}

// Decode GEMV limits: rows of at most 4096 bytes of codes and a work unit
// that fits one pipeline stage.  (Scale/bias rows are bulk-copied when
// 16-byte aligned and copied entry by entry otherwise.)
static moeq_status check_gemv_tensor(const moeq_qtensor& t, int nmat) {
  if (slices_of(t) > 8) return MOEQ_ERR_UNSUPPORTED;
  if (!gemv_fits(t.in_dim, t.bits, nmat, t.group_size)) return MOEQ_ERR_UNSUPPORTED;
  return MOEQ_OK;
}

static moeq_status check_decode_shapes(const moeq_layer* L) {
  moeq_status s;
  if ((s = check_gemv_tensor(L->router, 1)) != MOEQ_OK) return s;
  if ((s = check_gemv_tensor(L->gate, 2)) != MOEQ_OK) return s;
  if ((s = check_gemv_tensor(L->down, 1)) != MOEQ_OK) return s;
  if (L->has_shared) {
    if ((s = check_gemv_tensor(L->sh_expert_gate, 1)) != MOEQ_OK) return s;
    if ((s = check_gemv_tensor(L->sh_gate, 2)) != MOEQ_OK) return s;
    if ((s = check_gemv_tensor(L->sh_down, 1)) != MOEQ_OK) return s;
  }
  return MOEQ_OK;
}

// ------------------------------------------------------------------ workspace layout
namespace {
struct Carve {
  size_t off = 0;
  size_t take(size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~(size_t)255;
    return o;
  }
};

struct DecodeWs {
  size_t gen, flag1, flag2, logits, sg_logit, sigma, idx, w, h, d, segs_gu, segs_dn, counts,
      vecs_gu, vecs_dn, ctr, flag, xsl, hsl, total;
};

DecodeWs decode_ws(const moeq_layer* L, int M) {
  const int E = L->n_experts, K = L->top_k, H = L->hidden, I = L->inter;
  const int Is = L->has_shared ? L->sh_gate.out_dim : 0;
  const size_t n = (size_t)M * K;
  Carve c;
  DecodeWs w;
  // one-launch decode: the previous call's tag (word 0) and two flag arrays
  w.gen = c.take(8);
  w.flag1 = c.take((size_t)kFusedMaxGrid * 8);
  w.flag2 = c.take((size_t)kFusedMaxGrid * 8);
  // router logits of M tokens (+ one slot: the shared gate logit of the
  // one-launch decode)
  w.logits = c.take(((size_t)M * E + 1) * 4);
  w.sg_logit = c.take((size_t)M * 4);
  w.sigma = c.take((size_t)M * 4);
  w.idx = c.take(n * 4);
  w.w = c.take(n * 4);
  w.h = c.take((n * I + (size_t)M * Is) * 4);
  w.d = c.take((n + (size_t)M) * H * 4);
  w.segs_gu = c.take((n + 1) * sizeof(Seg));
  w.segs_dn = c.take((n + 1) * sizeof(Seg));
  w.counts = c.take(8 * 4);
  w.vecs_gu = c.take(n * sizeof(VecRef));
  w.vecs_dn = c.take(n * sizeof(VecRef));
  w.ctr = c.take((size_t)H * 4);  // at most one counter per output row
  w.flag = c.take(4);             // "down lists published"
  // the M tokens' slices in the gate/up format (built by the router launch)
  w.xsl = c.take((size_t)M * gemv_xslice_words(H, L->gate.bits) * 4);
  // the hidden rows' slices in the down format (built by a launch of their
  // own; only for steps the gate/up launch plans itself)
  w.hsl = c.take(n <= (size_t)kFusedMaxPairs
                     ? (n + (size_t)M) * gemv_xslice_words(I, L->down.bits) * 4
                     : 0);
  w.total = c.off;
  return w;
}
}  // namespace

// AUTO: the decode path while a call has at most 96 (token, expert) pairs,
// the prefill path beyond.  Measured on B200 (in-graph, per call, decode vs
// prefill): the crossover lies between M*K = 64 and 128 on the 8-bit
// (E 128, K 8: M 8 -> 155 vs 171 us, M 16 -> 275 vs 236 us) and the 2-bit
// bank (E 512, K 4: M 16 -> 387 vs 455 us, M 32 -> 707 vs 626 us), and
// between 128 and 192 on the 4-bit layers; at M 64 prefill is 1.2 to 2.8
// times faster on all four.
constexpr int kAutoDecodePairs = 96;

// (A layer the prefill path cannot take -- 3-, 5- or 6-bit codes -- stays on
// the decode path whenever M allows.)
static int resolve_mode(int mode, int M, const moeq_layer* L) {
  if (mode == MOEQ_MODE_AUTO) {
    if (M <= kMaxDecodeM && (int64_t)M * L->top_k <= kAutoDecodePairs) return MOEQ_MODE_DECODE;
    if (M <= kMaxDecodeM && prefill_workspace_bytes(L, M) == 0) return MOEQ_MODE_DECODE;
    return MOEQ_MODE_PREFILL;
  }
  return mode;
}

// ------------------------------------------------------------------ GEMV helpers
static int units_for(const moeq_qtensor& t, int out_dim, int nmat) {
  return gemv_units(out_dim, gemv_shape(t.in_dim, t.bits, nmat, t.group_size));
}

// CTAs of a persistent launch: one per SM (checked non-zero at entry).
static int grid_cap() { return sm_count(); }

static void set_shape(GemvArgs& a, const moeq_qtensor& t, int nmat) {
  const GemvShape sh = gemv_shape(t.in_dim, t.bits, nmat, t.group_size);
  a.in_dim = t.in_dim;
  a.G = t.group_size;
  a.fmt = t.format;
  a.slices = sh.S;
  a.subsets = sh.J;
  a.rows_per_unit = sh.RU;
}

// Pull a whole tensor (matrix `expert` of a bank) into L2: codes, scales, biases.
static int add_prefetch(GemvArgs& a, const moeq_qtensor& t, int expert) {
  const int64_t words = (int64_t)t.out_dim * t.in_dim * t.bits / 32;
  const int64_t groups = (int64_t)t.out_dim * (t.in_dim / t.group_size);
  const bool mx = is_mx(t);
  const void* p[3] = {t.w + (int64_t)expert * t.expert_stride_w,
                      scale_at(t, (int64_t)expert * t.expert_stride_sb),
                      mx ? nullptr : t.biases + (int64_t)expert * t.expert_stride_sb};
  const int64_t b[3] = {words * 4, groups * (mx ? 1 : 2), mx ? 0 : groups * 2};
  for (int i = 0; i < (mx ? 2 : 3) && a.n_pf < kMaxPrefetch; ++i)
    if (((uintptr_t)p[i] & 15) == 0) a.pf[a.n_pf++] = PrefetchRange{p[i], b[i]};
  return a.n_pf;
}

// x [M][in] (bf16) times one matrix -> y with row stride `ystride`.
static Seg plain_seg(const moeq_qtensor& t, int expert, const void* src, int64_t src_stride,
                     float* dst, int64_t dst_stride, int n_vec, int unit_begin) {
  Seg s;
  memset(&s, 0, sizeof(s));
  const uint32_t* w = t.w + (int64_t)expert * t.expert_stride_w;
  const uint16_t* sc = scale_at(t, (int64_t)expert * t.expert_stride_sb);
  const uint16_t* bi = is_mx(t) ? nullptr : t.biases + (int64_t)expert * t.expert_stride_sb;
  s.w[0] = s.w[1] = w;
  s.s[0] = s.s[1] = sc;
  s.b[0] = s.b[1] = bi;
  s.out_dim = t.out_dim;
  s.in_dim = t.in_dim;
  s.G = t.group_size;
  s.bits = t.bits;
  s.n_vec = n_vec;
  s.unit_begin = unit_begin;
  s.vec_mode = 0;
  s.src_base = src;
  s.src_stride = src_stride;
  s.dst_base = dst;
  s.dst_stride = dst_stride;
  s.vecs = nullptr;
  return s;
}

// Segments of one format (the first segment's tensor gives the shape).
static cudaError_t run_plain(const moeq_qtensor& shape_t, const Seg* segs, int n, int nl,
                             GemvArgs* pf, cudaStream_t st) {
  GemvArgs a;
  if (pf) a = *pf; else memset(&a, 0, sizeof(a));
  set_shape(a, shape_t, 1);
  const GemvShape sh = gemv_shape(shape_t.in_dim, shape_t.bits, 1, shape_t.group_size);
  // Few row blocks and several vectors (the router of a small decode
  // batch): each row block's vectors are split over several units, so that
  // both consumer groups of every CTA get work instead of a few CTAs taking
  // every vector of a block one after another.
  int blocks = 0;
  for (int i = 0; i < n; ++i) blocks += gemv_units(segs[i].out_dim, sh);
  const int want = 2 * grid_cap();
  int vpu = 0;
  if (n > 0 && segs[0].n_vec > 1 && blocks > 0 && blocks < want) {
    const int need = (want + blocks - 1) / blocks;
    const int nvc = need < segs[0].n_vec ? need : segs[0].n_vec;
    vpu = (segs[0].n_vec + nvc - 1) / nvc;
  }
  int units = 0;
  for (int i = 0; i < n; ++i) {
    a.segs[i] = segs[i];
    a.segs[i].unit_begin = units;
    a.segs[i].vpu = vpu;
    units += gemv_units(segs[i].out_dim, sh) * seg_vchunks(segs[i].n_vec, vpu);
  }
  a.n_segs = n;
  a.total_units = units;
  a.status = status_ptr();
  // a launch that carries L2 prefetches gets enough CTAs to spread them
  // (one 32 KB piece per CTA and lane); CTAs without a unit only prefetch
  int64_t pieces = 0;
  for (int i = 0; i < a.n_pf; ++i) pieces += (a.pf[i].bytes + 32 * 1024 - 1) / (32 * 1024);
  int grid = units;
  if (pieces / 8 > grid) grid = (int)(pieces / 8);
  if (grid > grid_cap()) grid = grid_cap();
  return launch_gemv(shape_t.bits, nl, 1, SRC_BF16, a, grid, st);
}

static cudaError_t run_dyn(const moeq_qtensor& shape_t, const Seg* segs, const int32_t* count,
                           int nl, int nmat, int src, int max_units, cudaStream_t st,
                           const Seg* pf_segs = nullptr, const int32_t* pf_count = nullptr,
                           const TokenSlices* xsl = nullptr) {
  GemvArgs a;
  memset(&a, 0, sizeof(a));
  set_shape(a, shape_t, nmat);
  if (xsl) a.xsl = *xsl;
  a.dyn_segs = segs;
  a.dyn_count = count;
  a.pf_segs = pf_segs;
  a.pf_count = pf_count;
  a.status = status_ptr();
  const int grid = max_units < grid_cap() ? max_units : grid_cap();
  return launch_gemv(shape_t.bits, nl, nmat, src, a, grid, st);
}

#define CK(x)                                     \
  do {                                            \
    if ((x) != cudaSuccess) return MOEQ_ERR_CUDA; \
  } while (0)
// one kernel launch through the library
#define LAUNCH(x)          \
  do {                     \
    CK(x);                 \
    count_launches(1);     \
  } while (0)

// ------------------------------------------------------------------ one-launch decode
// Shape part of the one-launch decode's arguments for the last layer seen by
// this host thread (recomputed when the descriptor or grid changes).
struct FusedCache {
  bool valid = false, ok = false;
  moeq_layer L;
  int grid = 0;
  bool from_router = false;
  FusedArgs a;
  FzMaps m;
};
static thread_local FusedCache t_fused;

static bool fused_decode_enabled() {
  const char* e = getenv("MOEQ_FUSED_DECODE");
  return e && e[0] == '1' && e[1] == 0;
}

static const FusedArgs* fused_shape(const moeq_layer* L, int grid, bool from_router) {
  FusedCache& f = t_fused;
  if (!f.valid || f.grid != grid || f.from_router != from_router ||
      memcmp(&f.L, L, sizeof(moeq_layer)) != 0) {
    f.valid = true;
    f.L = *L;
    f.grid = grid;
    f.from_router = from_router;
    f.ok = fused_decode_plan(L, grid, from_router, f.a, f.m);
  }
  return f.ok ? &f.a : nullptr;
}

static moeq_status fused_forward(const FusedArgs& shape, const FzMaps& maps, int grid,
                                 const uint16_t* x,
                                 const int32_t* idx_in, const float* w_in, const float* residual,
                                 float* y, int32_t* idx_out, float* w_out, char* base,
                                 const DecodeWs& lay, cudaStream_t st) {
  FusedArgs a = shape;
  a.x = x;
  a.idx_in = idx_in;
  a.w_in = w_in;
  a.residual = residual;
  a.y = y;
  a.idx_out = idx_out;
  a.w_out = w_out;
  a.gen = (uint64_t*)(base + lay.gen);
  a.flag1 = (uint64_t*)(base + lay.flag1);
  a.flag2 = (uint64_t*)(base + lay.flag2);
  a.logits = (float*)(base + lay.logits);
  a.h = (float*)(base + lay.h);
  a.hsh = a.h + (size_t)a.K * a.I;
  a.status = status_ptr();
  if (!a.status) return MOEQ_ERR_CUDA;
  CK(profile_mark(true, st));
  LAUNCH(launch_fused_decode(a, maps, grid, st));
  CK(profile_mark(false, st));
  return MOEQ_OK;
}

// ------------------------------------------------------------------ single-token decode
// Shape part of the single-token launches' arguments for the last layer
// seen by this host thread.
struct SingleCache {
  bool valid = false, ok = false;
  moeq_layer L;
  int sms = 0;
  S1Args a;
};
static thread_local SingleCache t_single;

// MOEQ_SINGLE_DECODE=0 sends single tokens to the general decode launches.
static bool single_decode_enabled() {
  const char* e = getenv("MOEQ_SINGLE_DECODE");
  return !(e && e[0] == '0' && e[1] == 0);
}

static const S1Args* single_shape(const moeq_layer* L, int sms) {
  SingleCache& c = t_single;
  if (!c.valid || c.sms != sms || memcmp(&c.L, L, sizeof(moeq_layer)) != 0) {
    c.valid = true;
    c.L = *L;
    c.sms = sms;
    c.ok = single_decode_plan(L, sms, c.a);
  }
  return c.ok ? &c.a : nullptr;
}

static moeq_status single_forward(const S1Args& shape, const uint16_t* x, const int32_t* idx_in,
                                  const float* w_in, const float* residual, float* y,
                                  int32_t* idx, float* wts, char* base, const DecodeWs& lay,
                                  cudaStream_t st) {
  S1Args a = shape;
  a.x = x;
  a.idx_in = idx_in;
  a.w_in = w_in;
  a.residual = residual;
  a.y = y;
  a.logits = (float*)(base + lay.logits);
  a.sg_logit = (float*)(base + lay.sg_logit);
  a.idx = idx;
  a.w = wts;
  a.sigma = (float*)(base + lay.sigma);
  a.h = (float*)(base + lay.h);
  a.status = status_ptr();
  if (!a.status) return MOEQ_ERR_CUDA;
  // a given routing needs the router launch only for the shared gate's row
  if (idx_in) a.gridR = 1;
  if (!idx_in || a.has_shared) LAUNCH(launch_single_router(a, st));
  CK(profile_mark(true, st));
  LAUNCH(launch_single_gateup(a, st));
  CK(profile_mark(false, st));
  LAUNCH(launch_single_down(a, st));
  return MOEQ_OK;
}

// ------------------------------------------------------------------ decode path
static moeq_status decode_forward(const moeq_layer* L, const uint16_t* x, int M,
                                  const int32_t* idx_in, const float* w_in, const float* residual,
                                  float* y, int32_t* idx_out, float* w_out, void* ws,
                                  cudaStream_t st) {
  const int E = L->n_experts, K = L->top_k, H = L->hidden, I = L->inter;
  const int n = M * K;
  const DecodeWs lay = decode_ws(L, M);
  char* base = (char*)ws;
  float* logits = (float*)(base + lay.logits);
  float* sg_logit = (float*)(base + lay.sg_logit);
  float* sigma = (float*)(base + lay.sigma);
  int32_t* idx = idx_out ? idx_out : (int32_t*)(base + lay.idx);
  float* wts = w_out ? w_out : (float*)(base + lay.w);
  float* h = (float*)(base + lay.h);
  float* d = (float*)(base + lay.d);
  Seg* segs_gu = (Seg*)(base + lay.segs_gu);
  Seg* segs_dn = (Seg*)(base + lay.segs_dn);
  int32_t* counts = (int32_t*)(base + lay.counts);
  VecRef* vecs_gu = (VecRef*)(base + lay.vecs_gu);
  VecRef* vecs_dn = (VecRef*)(base + lay.vecs_dn);

  // one token: the whole layer in one launch when its formats allow and the
  // caller opted in (MOEQ_FUSED_DECODE=1; measured slower than the three
  // launches below on the 397B-like layer, so not the default)
  if (M == 1 && fused_decode_enabled()) {
    const int grid = grid_cap() < kFusedMaxGrid ? grid_cap() : kFusedMaxGrid;
    if (const FusedArgs* f = fused_shape(L, grid, idx_in == nullptr))
      return fused_forward(*f, t_fused.m, grid, x, idx_in, w_in, residual, y, idx_out, w_out, base,
                           lay, st);
  }
  // one token: three lean launches when the formats allow (k_single.cu)
  if (M == 1 && single_decode_enabled()) {
    if (const S1Args* a = single_shape(L, grid_cap()))
      return single_forward(*a, x, idx_in, w_in, residual, y, idx, wts, base, lay, st);
  }

  // 1. router logits and the shared-expert gate logit (one launch when the
  //    two 8-bit tensors agree in format)
  const moeq_qtensor& R = L->router;
  const moeq_qtensor& SG = L->sh_expert_gate;
  const bool sg_with_router = L->has_shared && SG.bits == R.bits &&
                              SG.group_size == R.group_size && SG.in_dim == R.in_dim;
  // the shared expert's weights do not depend on the routing: pull them into
  // L2 while the router streams
  // small steps plan inside the gate/up launch (fused plan, below); when
  // the router runs too, the down launch's producer starts on the plan's
  // flag instead of on the whole gate/up launch
  const bool sh_same_gu = L->has_shared && L->sh_gate.bits == L->gate.bits &&
                          L->sh_gate.group_size == L->gate.group_size &&
                          L->sh_gate.format == L->gate.format;
  const bool fused_plan =
      n <= kFusedMaxPairs && (!L->has_shared || sh_same_gu) &&
      plan_scratch_bytes(M, K, E, plan_route_warps(M, E, gemv_threads() / 32)) <=
          (size_t)gemv_plan_scratch_cap();
  int32_t* flag = (fused_plan && !idx_in) ? (int32_t*)(base + lay.flag) : nullptr;
  GemvArgs pf;
  memset(&pf, 0, sizeof(pf));
  pf.flag_reset = flag;
  // several tokens and a router launch: it also converts every token row
  // once into the gate/up launch's slice format, which the gate/up
  // consumers copy instead of converting the row for every unit
  TokenSlices xs;
  memset(&xs, 0, sizeof(xs));
  if (M > 1 && !idx_in && L->gate.format == MOEQ_FMT_AFFINE &&
      gemv_xslice_words(H, L->gate.bits) > 0) {
    xs.table = (uint32_t*)(base + lay.xsl);
    xs.x = x;
    xs.M = M;
    xs.H = H;
    xs.bits = L->gate.bits;
    xs.S = gemv_shape(H, L->gate.bits, 2, L->gate.group_size).S;
  }
  pf.xsl = xs;
  if (L->has_shared) {
    add_prefetch(pf, L->sh_gate, 0);
    add_prefetch(pf, L->sh_up, 0);
    add_prefetch(pf, L->sh_down, 0);
  }
  if (!idx_in) {
    Seg segs[2];
    int ns = 0;
    segs[ns++] = plain_seg(R, 0, x, H, logits, E, M, 0);
    if (sg_with_router) segs[ns++] = plain_seg(SG, 0, x, H, sg_logit, 1, M, 0);
    LAUNCH(run_plain(R, segs, ns, 3, &pf, st));
    pf.n_pf = 0;
    pf.flag_reset = nullptr;
    pf.xsl.table = nullptr;
  }
  if (L->has_shared && (idx_in || !sg_with_router)) {
    Seg s = plain_seg(SG, 0, x, H, sg_logit, 1, M, 0);
    LAUNCH(run_plain(SG, &s, 1, 3, &pf, st));
  }

  // 2. routing + grouped plan
  DecodePlanArgs p;
  memset(&p, 0, sizeof(p));
  p.logits = idx_in ? nullptr : logits;
  p.sg_logit = L->has_shared ? sg_logit : nullptr;
  p.idx_in = idx_in;
  p.w_in = w_in;
  p.M = M;
  p.E = E;
  p.K = K;
  p.renorm = L->renorm;
  p.router_scale = L->router_scale;
  p.idx_out = idx;
  p.w_out = wts;
  p.x = x;
  p.H = H;
  p.I = I;
  p.has_shared = L->has_shared;
  p.gate = L->gate;
  p.up = L->up;
  p.down = L->down;
  if (L->has_shared) {
    p.sh_gate = L->sh_gate;
    p.sh_up = L->sh_up;
    p.sh_down = L->sh_down;
  }
  p.h = h;
  p.d = d;
  p.sigma = sigma;
  p.segs_gu = segs_gu;
  p.count_gu = counts;
  p.segs_dn = segs_dn;
  p.count_dn = counts + 4;
  p.vecs_gu = vecs_gu;
  p.vecs_dn = vecs_dn;
  p.units_per_seg_gu = units_for(L->gate, I, 2);
  p.units_per_seg_dn = units_for(L->down, H, 1);
  p.ctr = (int32_t*)(base + lay.ctr);
  p.n_ctr = p.units_per_seg_dn;
  if (L->has_shared) {
    // the shared expert's units hold one token each when there are several:
    // a unit's tokens run one after another on one consumer group, so M of
    // them in one unit make that CTA the step's tail
    p.sh_vpu_gu = M > 1 ? 1 : 0;
    p.sh_vpu_dn = M > 1 ? 1 : 0;
    p.units_per_seg_gu_sh =
        units_for(L->sh_gate, L->sh_gate.out_dim, 2) * seg_vchunks(M, p.sh_vpu_gu);
    p.units_per_seg_dn_sh = units_for(L->sh_down, H, 1) * seg_vchunks(M, p.sh_vpu_dn);
    p.shared_same_gu = (L->sh_gate.bits == L->gate.bits &&
                        L->sh_gate.group_size == L->gate.group_size &&
                        L->sh_gate.format == L->gate.format);
    p.shared_same_dn = (L->sh_down.bits == L->down.bits &&
                        L->sh_down.group_size == L->down.group_size &&
                        L->sh_down.format == L->down.format &&
                        L->sh_down.in_dim == L->down.in_dim);
  }
  p.status = status_ptr();
  // the down launch covers every segment: its CTAs also do the combine
  const bool fuse_combine = !L->has_shared || p.shared_same_dn;
  if (!fused_plan) LAUNCH(launch_decode_plan(p, st));

  // 3. gate/up + SwiGLU, then 4. down, for the routed experts (+ shared)
  const int max_entries = n < E ? n : E;
  const int max_gu = max_entries * p.units_per_seg_gu + (p.shared_same_gu ? p.units_per_seg_gu_sh : 0);
  const int max_dn = max_entries * p.units_per_seg_dn + (p.shared_same_dn ? p.units_per_seg_dn_sh : 0);
  CK(profile_mark(true, st));
  if (fused_plan) {
    // the gate/up launch plans, and pulls the down projections into L2
    GemvArgs a;
    memset(&a, 0, sizeof(a));
    set_shape(a, L->gate, 2);
    a.status = status_ptr();
    a.fused_plan = 1;
    a.plan = p;
    a.flag_set = flag;
    a.xsl = xs;
    const int grid = max_gu < grid_cap() ? max_gu : grid_cap();
    LAUNCH(launch_gemv(L->gate.bits, 2, 2, SRC_BF16, a, grid, st));
  } else {
    // the gate/up launch also pulls the down projections it will feed into L2
    LAUNCH(run_dyn(L->gate, segs_gu, counts, 2, 2, SRC_BF16, max_gu, st, segs_dn, counts + 4,
                   &xs));
  }
  CK(profile_mark(false, st));
  if (L->has_shared && !p.shared_same_gu)
    LAUNCH(run_dyn(L->sh_gate, segs_gu + n, counts + 2, 2, 2, SRC_BF16, p.units_per_seg_gu_sh,
                   st));
  // several tokens planned in the gate/up launch: the hidden rows are
  // converted once into the down launch's slice format (pairs, then the
  // shared expert's rows, all of stride I when they share the launch), which
  // its consumers copy instead of converting a row for every unit.  Larger
  // steps do without (397B-like layer at M = 24: 381.0 against 377.4 us)
  TokenSlices hs;
  memset(&hs, 0, sizeof(hs));
  if (M > 1 && fused_plan && fuse_combine && L->down.format == MOEQ_FMT_AFFINE &&
      gemv_xslice_words(I, L->down.bits) > 0) {
    hs.table = (uint32_t*)(base + lay.hsl);
    hs.x = h;
    hs.M = (int)n + (L->has_shared ? M : 0);
    hs.H = I;
    hs.bits = L->down.bits;
    hs.S = gemv_shape(I, L->down.bits, 1, L->down.group_size).S;
    LAUNCH(launch_hslices(hs, st));
  }
  {
    GemvArgs a;
    memset(&a, 0, sizeof(a));
    set_shape(a, L->down, 1);
    a.xsl = hs;
    a.dyn_segs = segs_dn;
    a.dyn_count = counts + 4;
    a.status = status_ptr();
    a.flag_wait = flag;
    if (fuse_combine) {
      a.fuse_combine = 1;
      a.comb.w = wts;
      a.comb.sigma = sigma;
      a.comb.residual = residual;
      a.comb.y = y;
      a.comb.d = d;
      a.comb.ctr = p.ctr;
      a.comb.M = M;
      a.comb.K = K;
      a.comb.H = H;
      a.comb.has_shared = L->has_shared;
      a.comb.sh_units = seg_vchunks(M, p.sh_vpu_dn);
    }
    const int grid = max_dn < grid_cap() ? max_dn : grid_cap();
    LAUNCH(launch_gemv(L->down.bits, 2, 1, SRC_F32, a, grid, st));
  }
  if (L->has_shared && !p.shared_same_dn)
    LAUNCH(run_dyn(L->sh_down, segs_dn + n, counts + 6, 2, 1, SRC_F32, p.units_per_seg_dn_sh,
                   st));

  // 5. weighted combine in k order (+ shared, + residual), unless the down
  //    launch did it
  if (!fuse_combine)
    LAUNCH(launch_combine(d, wts, sigma, L->has_shared, residual, y, M, K, H, st));
  return MOEQ_OK;
}

// ------------------------------------------------------------------ entry points
MOEQ_API const char* moeq_version(void) { return "moeq 0.1 (sm_100a)"; }

MOEQ_API const char* moeq_status_str(int32_t s) {
  switch (s) {
    case MOEQ_OK: return "ok";
    case MOEQ_ERR_INVALID_ARG: return "invalid argument";
    case MOEQ_ERR_UNSUPPORTED: return "unsupported format or size";
    case MOEQ_ERR_ALIGNMENT: return "misaligned pointer or dimension";
    case MOEQ_ERR_WORKSPACE: return "workspace missing or too small";
    case MOEQ_ERR_CUDA: return "CUDA runtime error";
    case MOEQ_ERR_TIMEOUT: return "device wait timed out";
    case MOEQ_ERR_RANGE: return "operand outside the fp16 range of the prefill tiles";
    default: return "unknown status";
  }
}

MOEQ_API moeq_status moeq_dequant(const moeq_qtensor* t, int32_t expert, uint8_t* q_out,
                                  float* w_out, void* stream) {
  if (!t || (!q_out && !w_out) || expert < 0) return MOEQ_ERR_INVALID_ARG;
  moeq_status s = check_tensor(t, expert + 1);
  if (s != MOEQ_OK) return s;
  if (expert > 0 && (t->expert_stride_w <= 0 || t->expert_stride_sb <= 0))
    return MOEQ_ERR_INVALID_ARG;
  LAUNCH(launch_dequant(*t, expert, q_out, w_out, (cudaStream_t)stream));
  return MOEQ_OK;
}

MOEQ_API moeq_status moeq_qmv(const moeq_qtensor* t, int32_t expert, const uint16_t* x, int32_t M,
                              float* y, void* stream) {
  if (!t || !x || !y || expert < 0 || M <= 0) return MOEQ_ERR_INVALID_ARG;
  if (M > kMaxDecodeM) return MOEQ_ERR_UNSUPPORTED;
  moeq_status s = check_tensor(t, expert + 1);
  if (s != MOEQ_OK) return s;
  if (expert > 0 && (t->expert_stride_w <= 0 || t->expert_stride_sb <= 0))
    return MOEQ_ERR_INVALID_ARG;
  if ((s = check_gemv_tensor(*t, 1)) != MOEQ_OK) return s;
  if (!aligned(x, 16) || ((int64_t)t->in_dim * 2) % 16 || !aligned(y, 4)) return MOEQ_ERR_ALIGNMENT;
  Seg seg = plain_seg(*t, expert, x, t->in_dim, y, t->out_dim, M, 0);
  LAUNCH(run_plain(*t, &seg, 1, 3, nullptr, (cudaStream_t)stream));
  return MOEQ_OK;
}

MOEQ_API moeq_status moeq_route_topk(const float* logits, int32_t M, int32_t E, int32_t K,
                                     int32_t renorm, float router_scale, int32_t* idx, float* w,
                                     void* stream) {
  if (M < 0 || E <= 0 || K <= 0 || K > E) return MOEQ_ERR_INVALID_ARG;
  if (K > kMaxK || E > kMaxE) return MOEQ_ERR_UNSUPPORTED;
  if (M == 0) return MOEQ_OK;
  if (!logits || !idx || !w) return MOEQ_ERR_INVALID_ARG;
  LAUNCH(launch_route_topk(logits, M, E, K, renorm, router_scale, idx, w, (cudaStream_t)stream));
  return MOEQ_OK;
}

MOEQ_API size_t moeq_workspace_bytes(const moeq_layer* L, int32_t M, int32_t mode) {
  if (check_layer(L) != MOEQ_OK || M <= 0) return 0;
  mode = resolve_mode(mode, M, L);
  if (mode == MOEQ_MODE_DECODE) {
    if (M > kMaxDecodeM) return 0;
    return decode_ws(L, M).total;
  }
  if (mode == MOEQ_MODE_PREFILL) return prefill_workspace_bytes(L, M);
  return 0;
}

namespace moeq {
// The argument checks every layer entry point runs before its workspace
// check: the layer, M, the mode, and the token, output and residual pointers.
moeq_status forward_arg_check(const moeq_layer* L, const uint16_t* x, int32_t M, float* y,
                              const float* residual, int32_t mode) {
  moeq_status s = check_layer(L);
  if (s != MOEQ_OK) return s;
  if (M < 0 || !x || !y) return MOEQ_ERR_INVALID_ARG;
  if (mode < MOEQ_MODE_AUTO || mode > MOEQ_MODE_PREFILL) return MOEQ_ERR_INVALID_ARG;
  if (M == 0) return MOEQ_OK;
  if (!aligned(x, 16) || (L->hidden * 2) % 16 || !aligned(y, 16) || L->hidden % 4)
    return MOEQ_ERR_ALIGNMENT;
  if (residual && !aligned(residual, 16)) return MOEQ_ERR_ALIGNMENT;
  return MOEQ_OK;
}
}  // namespace moeq

static moeq_status forward_common(const moeq_layer* L, const uint16_t* x, int32_t M,
                                  const int32_t* idx_in, const float* w_in, const float* residual,
                                  float* y, int32_t* idx_out, float* w_out, void* ws,
                                  size_t ws_bytes, int32_t mode, void* stream,
                                  const NormOut* norm = nullptr) {
  moeq_status s = forward_arg_check(L, x, M, y, residual, mode);
  if (s != MOEQ_OK || M == 0) return s;
  mode = resolve_mode(mode, M, L);
  const size_t need = moeq_workspace_bytes(L, M, mode);
  if (need == 0) return MOEQ_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < need) return MOEQ_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return MOEQ_ERR_ALIGNMENT;
  if (grid_cap() <= 0) return MOEQ_ERR_CUDA;  // no current device to size launches for
  cudaStream_t st = (cudaStream_t)stream;
  if (mode == MOEQ_MODE_DECODE) {
    if (M > kMaxDecodeM) return MOEQ_ERR_UNSUPPORTED;
    if ((s = check_decode_shapes(L)) != MOEQ_OK) return s;
    s = decode_forward(L, x, M, idx_in, w_in, residual, y, idx_out, w_out, ws, st);
    if (s == MOEQ_OK && norm) LAUNCH(launch_rmsnorm_rows(y, M, L->hidden, *norm, st));
    return s;
  }
  return prefill_forward(L, x, M, idx_in, w_in, residual, y, idx_out, w_out, ws, ws_bytes,
                         status_ptr(), st, norm);
}

MOEQ_API moeq_status moeq_expert_ffn(const moeq_layer* L, const uint16_t* x, int32_t M,
                                     const int32_t* idx, const float* w, const float* residual,
                                     float* y, void* ws, size_t ws_bytes, int32_t mode,
                                     void* stream) {
  if (M > 0 && (!idx || !w)) return MOEQ_ERR_INVALID_ARG;
  return forward_common(L, x, M, idx, w, residual, y, nullptr, nullptr, ws, ws_bytes, mode,
                        stream);
}

MOEQ_API moeq_status moeq_layer_forward(const moeq_layer* L, const uint16_t* x, int32_t M,
                                        float* y, const float* residual, int32_t* idx_out,
                                        float* w_out, void* ws, size_t ws_bytes, int32_t mode,
                                        void* stream) {
  return forward_common(L, x, M, nullptr, nullptr, residual, y, idx_out, w_out, ws, ws_bytes,
                        mode, stream);
}

MOEQ_API moeq_status moeq_layer_forward_norm(const moeq_layer* L, const uint16_t* x, int32_t M,
                                             float* y, const float* residual,
                                             const uint16_t* gamma, float eps, uint16_t* y_norm,
                                             int32_t* idx_out, float* w_out, void* ws,
                                             size_t ws_bytes, int32_t mode, void* stream) {
  moeq_status s = forward_arg_check(L, x, M, y, residual, mode);
  if (s != MOEQ_OK || M == 0) return s;
  if (!gamma || !y_norm || !(eps > 0.0f) || !(eps < INFINITY)) return MOEQ_ERR_INVALID_ARG;
  if (!aligned(gamma, 16) || !aligned(y_norm, 16)) return MOEQ_ERR_ALIGNMENT;
  const NormOut n{gamma, eps, y_norm};
  return forward_common(L, x, M, nullptr, nullptr, residual, y, idx_out, w_out, ws, ws_bytes,
                        mode, stream, &n);
}

MOEQ_API moeq_status moeq_set_profile_events(void* start, void* stop) {
  if ((start == nullptr) != (stop == nullptr)) return MOEQ_ERR_INVALID_ARG;
  t_prof_start = (cudaEvent_t)start;
  t_prof_stop = (cudaEvent_t)stop;
  return MOEQ_OK;
}

MOEQ_API uint64_t moeq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

MOEQ_API moeq_status moeq_selftest_wait_timeout(void* stream) {
  int* p = status_ptr();
  if (!p) return MOEQ_ERR_CUDA;
  LAUNCH(launch_wait_probe(p, (cudaStream_t)stream));
  return MOEQ_OK;
}

MOEQ_API moeq_status moeq_device_status(void* stream, int32_t* status_out) {
  if (!status_out) return MOEQ_ERR_INVALID_ARG;
  int* p = status_ptr();
  if (!p) return MOEQ_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  int v = 0;
  CK(cudaMemcpyAsync(&v, p, sizeof(int), cudaMemcpyDeviceToHost, st));
  CK(cudaMemsetAsync(p, 0, sizeof(int), st));
  CK(cudaStreamSynchronize(st));
  *status_out = v;
  return MOEQ_OK;
}
