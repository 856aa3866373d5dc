/*
 * CPU ORACLE for the affine-quantised mixture-of-experts FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load, call,
 * link or execute this file or the library built from it: only the tests,
 * the smoke check and the benchmark's CPU-baseline / reference arm do.  It
 * shares no code, header, table or helper with the CUDA library; it reads
 * only the packed bytes and the bf16 activations it is handed.
 *
 * Plain, slow, obviously correct: every value is dequantised group by group
 * and every sum is accumulated in fp64 (IEEE double), in the order the
 * definitions below state.  Threads (OpenMP) only split independent tokens.
 *
 * Sources (web pages, by title):
 *  [FM-ISSUE] "danveloper/flash-moe" issue thread (roipad.com mirror):
 *             mixed-precision comment -- affine mode, group_size 64,
 *             per-tensor 8-bit overrides for mlp.gate and
 *             mlp.shared_expert_gate, 8 nibbles per uint32 at 4 bits and
 *             4 bytes per uint32 at 8 bits, [512,512] U32 at 4 bits has
 *             in_dim 4096.
 *  [FM-SKILL] "flash-moe-inference" (skillbundle.dev): kernel listing
 *             (matvec_4bit_fma: dequantised value nibble*scale + bias and
 *             its fma(nibble, scale*x, bias*x) factoring; swiglu:
 *             g/(1+exp(-g))*up; moe_combine_residual: combine + residual +
 *             sigmoid gate) and the per-layer pipeline (softmax + topK).
 *  [MB-FIX]   "markbaseengine/MOE_FIX_SUCCESS_EXPERT_WORKS.md", section
 *             "Why This Worked": weights are organised in groups of 64 and
 *             the kernels iterate through the groups.
 *  [MB-ROUTE] "markbaseengine/MOE_ROUTER_WORKS_BREAKTHROUGH.md", section
 *             "Forward Pass Sequence": router projection, router scale,
 *             softmax, top-k, per-expert fused gate/up then down,
 *             accumulation.
 *  [MLX-3856] "Silent numerical corruption in single long forward on
 *             quantized MoE when sequence length % 32 != 0" (ml-explore/mlx
 *             issue 3856): gather_qmm over rows sorted by expert; each row
 *             of the result depends only on its own token.
 *
 * Readings where the pages are silent (each also listed in the design
 * notes): codes are packed low bits first; scales and biases are bf16;
 * ties in top-K go to the lower expert index; the renormalised weights are
 * p_k / sum of the selected p; the sigmoid gate multiplies only the shared
 * expert's output; outputs are fp32 on the device and fp64 here.
 *
 * Parity status: every function below is pinned by the CPU tests (closed
 * forms, brute-force dense products, invariants, special cases); none is
 * "parity unpinned".
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_API __attribute__((visibility("default")))

/* One affine-quantised tensor or bank of tensors (host memory). */
typedef struct {
  const uint32_t* w;      /* packed codes, [mats][out][in*bits/32] */
  const uint16_t* s;      /* bf16 scale bits, [mats][out][in/G] */
  const uint16_t* b;      /* bf16 bias bits,  [mats][out][in/G] */
  int32_t out, in, bits, G;
  int64_t stride_w;       /* words between consecutive matrices */
  int64_t stride_sb;      /* scale/bias entries between matrices */
  int32_t format;         /* 0 affine; 1 MX FP4 (s: uint8 E8M0 exponents, no b) */
} orc_tensor;

typedef struct {
  orc_tensor router, gate, up, down;
  int32_t has_shared;
  orc_tensor sh_gate, sh_up, sh_down, sh_expert_gate;
  int32_t H, I, E, K, renorm;
  double router_scale;
} orc_layer;

static int orc_threads = 0;

ORC_API void oracle_set_threads(int n) { orc_threads = n; }

ORC_API int oracle_get_threads(void) {
  return orc_threads > 0 ? orc_threads : omp_get_max_threads();
}

/* bf16 bits -> value (exact widening). */
static double orc_bf16(uint16_t h) {
  union { float f; uint32_t u; } v;
  v.u = ((uint32_t)h) << 16;
  return (double)v.f;
}

static float orc_bf16f(uint16_t h) {
  union { float f; uint32_t u; } v;
  v.u = ((uint32_t)h) << 16;
  return v.f;
}

/*
 * Code q(r, c) of matrix `mat`: value c of row r.  A 32-bit word holds
 * 32/bits values ([FM-ISSUE]: 8 per word at 4 bits, 4 at 8 bits); value j
 * of a word occupies bits [j*bits, (j+1)*bits) -- low bits first.
 */
static uint32_t orc_code(const orc_tensor* t, int mat, int64_t r, int64_t c) {
  /* value c of a row occupies bits [c*bits, (c+1)*bits) of the row's
   * little-endian stream of u32 words, low bits first; with 3, 5 or 6 bits a
   * value may straddle two words (cross-word packing) */
  const int64_t words_per_row = (int64_t)t->in * t->bits / 32;
  const uint32_t* row = t->w + (int64_t)mat * t->stride_w + r * words_per_row;
  const int64_t bit = c * t->bits;
  const int64_t k = bit / 32;
  const int off = (int)(bit % 32);
  uint64_t v = row[k] >> off;
  if (off + t->bits > 32) v |= (uint64_t)row[k + 1] << (32 - off);
  return (uint32_t)(v & ((1u << t->bits) - 1u));
}

/* Scale and bias of the group holding value c of row r ([MB-FIX]: groups
 * of G consecutive input values within a row). */
static void orc_group(const orc_tensor* t, int mat, int64_t r, int64_t c, double* s, double* b) {
  const int64_t groups = t->in / t->G;
  const int64_t i = (int64_t)mat * t->stride_sb + r * groups + c / t->G;
  *s = orc_bf16(t->s[i]);
  *b = orc_bf16(t->b[i]);
}

/*
 * MX FP4 ([MLX-3856] mode="mxfp4"; element and scale encodings of the OCP
 * Microscaling Formats specification v1.0): a 4-bit E2M1 code q has sign
 * bit 3, exponent bits 2..1 and mantissa bit 0; exponent 0 is subnormal
 * (value m * 2^-1), exponents 1..3 give 2^(e-1) * (1 + m/2).  A group of
 * 32 shares the E8M0 byte x: scale 2^(x - 127); x = 255 is NaN.
 */
static double orc_e2m1(uint32_t q) {
  const int sign = (q >> 3) & 1, e = (q >> 1) & 3, m = q & 1;
  const double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return sign ? -v : v;
}

static double orc_e8m0(const orc_tensor* t, int mat, int64_t r, int64_t c) {
  const int64_t groups = t->in / t->G;
  const uint8_t x = ((const uint8_t*)t->s)[(int64_t)mat * t->stride_sb + r * groups + c / t->G];
  return x == 255 ? NAN : ldexp(1.0, (int)x - 127);
}

/* The weight of value c of row r in fp64 (exact for both formats). */
static double orc_weight(const orc_tensor* t, int mat, int64_t r, int64_t c) {
  if (t->format == 1) return orc_e2m1(orc_code(t, mat, r, c)) * orc_e8m0(t, mat, r, c);
  double s, b;
  orc_group(t, mat, r, c, &s, &b);
  return (double)orc_code(t, mat, r, c) * s + b;
}

/* Unpacked codes, one byte per value, [out][in]. */
ORC_API void oracle_unpack(const orc_tensor* t, int mat, uint8_t* q) {
  for (int64_t r = 0; r < t->out; ++r)
    for (int64_t c = 0; c < t->in; ++c) q[r * t->in + c] = (uint8_t)orc_code(t, mat, r, c);
}

/*
 * Dequantised fp32 weights w = q*scale + bias ([FM-SKILL] "nibble*scale +
 * bias"), formed as ONE correctly rounded fp32 fused multiply-add of the
 * exact operands; that is the value an fp32 device dequantiser must return
 * bit for bit.
 */
ORC_API void oracle_dequant_f32(const orc_tensor* t, int mat, float* wout) {
  if (t->format == 1) {
    /* MX FP4: e2m1 * 2^(x-127) is exact in fp64; one rounding to fp32 */
    for (int64_t r = 0; r < t->out; ++r)
      for (int64_t c = 0; c < t->in; ++c) wout[r * t->in + c] = (float)orc_weight(t, mat, r, c);
    return;
  }
  for (int64_t r = 0; r < t->out; ++r)
    for (int64_t c = 0; c < t->in; ++c) {
      const int64_t groups = t->in / t->G;
      const int64_t i = (int64_t)mat * t->stride_sb + r * groups + c / t->G;
      wout[r * t->in + c] =
          fmaf((float)orc_code(t, mat, r, c), orc_bf16f(t->s[i]), orc_bf16f(t->b[i]));
    }
}

/*
 * y[r] = sum over groups g of sum over c in g of (q(r,c)*s(r,g) + b(r,g)) * x[c],
 * all in fp64, group by group ([MB-FIX], [FM-SKILL]).  x is fp64 here.
 */
static void orc_matvec(const orc_tensor* t, int mat, const double* x, double* y) {
  const int groups = t->in / t->G;
  for (int64_t r = 0; r < t->out; ++r) {
    double acc = 0.0;
    for (int g = 0; g < groups; ++g) {
      double part = 0.0;
      for (int k = 0; k < t->G; ++k) {
        const int64_t c = (int64_t)g * t->G + k;
        part += orc_weight(t, mat, r, c) * x[c];
      }
      acc += part;
    }
    y[r] = acc;
  }
}

/* Quantised matrix-vector product for M bf16 tokens: y[t][out] (fp64). */
ORC_API void oracle_qmv(const orc_tensor* t, int mat, const uint16_t* x_bf16, int M, double* y) {
#pragma omp parallel for num_threads(oracle_get_threads()) schedule(dynamic)
  for (int tok = 0; tok < M; ++tok) {
    double* x = (double*)malloc(sizeof(double) * (size_t)t->in);
    for (int c = 0; c < t->in; ++c) x[c] = orc_bf16(x_bf16[(int64_t)tok * t->in + c]);
    orc_matvec(t, mat, x, y + (int64_t)tok * t->out);
    free(x);
  }
}

/* Same with fp64 input vectors (used by the self-checks). */
ORC_API void oracle_qmv_f64(const orc_tensor* t, int mat, const double* x, int M, double* y) {
#pragma omp parallel for num_threads(oracle_get_threads()) schedule(dynamic)
  for (int tok = 0; tok < M; ++tok)
    orc_matvec(t, mat, x + (int64_t)tok * t->in, y + (int64_t)tok * t->out);
}

/*
 * Routing for one token ([MB-ROUTE] steps 3-4, [FM-SKILL] "softmax + topK"):
 *   l = router_scale * logits
 *   p = softmax(l)                      (max subtracted first)
 *   the K largest p, ties to the lower expert index, listed by p
 *   descending then index ascending
 *   w_k = p_k / sum of the K selected p   (if renorm; else w_k = p_k)
 * gap = (p_K - p_{K+1}) / p_K, the relative margin of the K-th choice
 * (1.0 when K == E).
 */
static void orc_route_one(const double* logits, int E, int K, int renorm, double router_scale,
                          int32_t* idx, double* wts, double* gap) {
  double* p = (double*)malloc(sizeof(double) * (size_t)E);
  char* taken = (char*)calloc((size_t)E, 1);
  double mx = -INFINITY;
  for (int e = 0; e < E; ++e) {
    p[e] = router_scale * logits[e];
    if (p[e] > mx) mx = p[e];
  }
  double z = 0.0;
  for (int e = 0; e < E; ++e) {
    p[e] = exp(p[e] - mx);
    z += p[e];
  }
  for (int e = 0; e < E; ++e) p[e] /= z;
  /* Softmax is strictly increasing in the scaled logit, so the K largest
   * scores are the K largest scaled logits (ties: lower index first).
   * Selecting on the logits gives that set even where exp() underflows and
   * several scores read as 0. */
  double sel = 0.0;
  for (int k = 0; k < K; ++k) {
    int best = -1;
    for (int e = 0; e < E; ++e)
      if (!taken[e] && (best < 0 || router_scale * logits[e] > router_scale * logits[best]))
        best = e;
    taken[best] = 1;
    idx[k] = best;
    wts[k] = p[best];
    sel += p[best];
  }
  if (renorm)
    for (int k = 0; k < K; ++k) wts[k] /= sel;
  if (gap) {
    /* relative gap of the K-th and (K+1)-th scores, (p_K - p_next) / p_K =
     * 1 - exp(l_next - l_K) on the scaled logits (defined under underflow) */
    int next = -1;
    for (int e = 0; e < E; ++e)
      if (!taken[e] && (next < 0 || router_scale * logits[e] > router_scale * logits[next]))
        next = e;
    *gap = next < 0 ? 1.0
                    : -expm1(router_scale * logits[next] - router_scale * logits[idx[K - 1]]);
  }
  free(taken);
  free(p);
}

ORC_API void oracle_route(const double* logits, int M, int E, int K, int renorm,
                          double router_scale, int32_t* idx, double* wts, double* gap) {
  for (int t = 0; t < M; ++t)
    orc_route_one(logits + (int64_t)t * E, E, K, renorm, router_scale, idx + (int64_t)t * K,
                  wts + (int64_t)t * K, gap ? gap + t : NULL);
}

/* Same routing on fp32 logits (the form the device produces or the
 * benchmark draws); the logits are widened exactly to fp64 first. */
ORC_API void oracle_route_f32(const float* logits, int M, int E, int K, int renorm,
                              double router_scale, int32_t* idx, double* wts, double* gap) {
  double* l = (double*)malloc(sizeof(double) * (size_t)E);
  for (int t = 0; t < M; ++t) {
    for (int e = 0; e < E; ++e) l[e] = (double)logits[(int64_t)t * E + e];
    orc_route_one(l, E, K, renorm, router_scale, idx + (int64_t)t * K, wts + (int64_t)t * K,
                  gap ? gap + t : NULL);
  }
  free(l);
}

/*
 * One expert on one token ([MB-ROUTE] step 5, [FM-SKILL] swiglu):
 *   g = Wg x, u = Wu x, h = g / (1 + exp(-g)) * u, d = Wd h.
 * h stays in fp64.
 */
static void orc_expert(const orc_tensor* Wg, const orc_tensor* Wu, const orc_tensor* Wd, int e,
                       const double* x, double* d, double* scratch_g, double* scratch_u) {
  orc_matvec(Wg, e, x, scratch_g);
  orc_matvec(Wu, e, x, scratch_u);
  for (int j = 0; j < Wg->out; ++j) {
    const double g = scratch_g[j];
    scratch_g[j] = g / (1.0 + exp(-g)) * scratch_u[j];
  }
  orc_matvec(Wd, e, scratch_g, d);
}

/*
 * Combine for one token ([FM-SKILL] moe_combine_residual, [MB-ROUTE]
 * step 6):  out = sum_k w_k d_k  +  sigmoid(Wsg x) * SE(x)  (+ residual),
 * where SE is the shared expert and Wsg the 1 x H sigmoid gate
 * ([FM-ISSUE]: mlp.shared_expert_gate).  Experts are summed in k order.
 */
static void orc_token(const orc_layer* L, const double* x, const int32_t* idx, const double* wts,
                      const float* residual, double* out) {
  const int H = L->H;
  const int Imax = L->I > (L->has_shared ? L->sh_gate.out : 0) ? L->I : L->sh_gate.out;
  double* d = (double*)malloc(sizeof(double) * (size_t)H);
  double* sg = (double*)malloc(sizeof(double) * (size_t)Imax);
  double* su = (double*)malloc(sizeof(double) * (size_t)Imax);
  for (int c = 0; c < H; ++c) out[c] = 0.0;
  for (int k = 0; k < L->K; ++k) {
    orc_expert(&L->gate, &L->up, &L->down, idx[k], x, d, sg, su);
    for (int c = 0; c < H; ++c) out[c] += wts[k] * d[c];
  }
  if (L->has_shared) {
    double glogit;
    orc_matvec(&L->sh_expert_gate, 0, x, &glogit);
    const double sigma = 1.0 / (1.0 + exp(-glogit));
    orc_expert(&L->sh_gate, &L->sh_up, &L->sh_down, 0, x, d, sg, su);
    for (int c = 0; c < H; ++c) out[c] += sigma * d[c];
  }
  if (residual)
    for (int c = 0; c < H; ++c) out[c] += (double)residual[c];
  free(su);
  free(sg);
  free(d);
}

/*
 * Experts + combine with the routing given (the moeq_expert_ffn contract):
 * out[t] = sum_k wts[t][k] * expert_{idx[t][k]}(x_t) (+ shared expert).
 */
ORC_API void oracle_expert_ffn(const orc_layer* L, const uint16_t* x_bf16, int M,
                               const int32_t* idx, const double* wts, const float* residual,
                               double* out) {
  const int H = L->H;
#pragma omp parallel for num_threads(oracle_get_threads()) schedule(dynamic)
  for (int t = 0; t < M; ++t) {
    double* x = (double*)malloc(sizeof(double) * (size_t)H);
    for (int c = 0; c < H; ++c) x[c] = orc_bf16(x_bf16[(int64_t)t * H + c]);
    orc_token(L, x, idx + (int64_t)t * L->K, wts + (int64_t)t * L->K,
              residual ? residual + (int64_t)t * H : NULL, out + (int64_t)t * H);
    free(x);
  }
}

/*
 * The whole layer for M tokens ([MB-ROUTE] "Forward Pass Sequence"):
 * router projection -> scale -> softmax -> top-K (-> renorm) -> experts ->
 * combine.  Each token is computed on its own ([MLX-3856]: a row's result
 * must not depend on the other rows).  Writes the routing too.
 */
ORC_API void oracle_layer(const orc_layer* L, const uint16_t* x_bf16, int M, const float* residual,
                          double* out, int32_t* idx_out, double* w_out, double* gap_out,
                          double* logits_out) {
  const int H = L->H, E = L->E, K = L->K;
#pragma omp parallel for num_threads(oracle_get_threads()) schedule(dynamic)
  for (int t = 0; t < M; ++t) {
    double* x = (double*)malloc(sizeof(double) * (size_t)H);
    double* logits = (double*)malloc(sizeof(double) * (size_t)E);
    for (int c = 0; c < H; ++c) x[c] = orc_bf16(x_bf16[(int64_t)t * H + c]);
    orc_matvec(&L->router, 0, x, logits);
    if (logits_out) memcpy(logits_out + (int64_t)t * E, logits, sizeof(double) * (size_t)E);
    orc_route_one(logits, E, K, L->renorm, L->router_scale, idx_out + (int64_t)t * K,
                  w_out + (int64_t)t * K, gap_out ? gap_out + t : NULL);
    orc_token(L, x, idx_out + (int64_t)t * K, w_out + (int64_t)t * K,
              residual ? residual + (int64_t)t * H : NULL, out + (int64_t)t * H);
    free(logits);
    free(x);
  }
}

/*
 * RMS norm of the combined output, the step the pages run after the
 * combine ("flash-moe-inference", per-layer pipeline: "CMD3: expert forward
 * + combine + norm"; rms_norm_pass1 = sum of squares, rms_norm_pass2 =
 * apply):  out[t][j] = y[t][j] / sqrt((1/H) sum_i y[t][i]^2 + eps) * g[j],
 * g the bf16 weight vector.  fp64 throughout.
 */
ORC_API void oracle_rmsnorm(const double* y, int M, int H, const uint16_t* g_bf16, double eps,
                            double* out) {
  for (int t = 0; t < M; ++t) {
    const double* r = y + (int64_t)t * H;
    double ss = 0.0;
    for (int i = 0; i < H; ++i) ss += r[i] * r[i];
    const double inv = 1.0 / sqrt(ss / H + eps);
    for (int j = 0; j < H; ++j) out[(int64_t)t * H + j] = r[j] * inv * orc_bf16(g_bf16[j]);
  }
}
