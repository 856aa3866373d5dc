/*
 * Seeded synthetic inputs: packed affine-quantised weight tensors, bf16
 * activations and Zipf-skewed router logits.  Host functions fill host
 * memory (OpenMP threads); device functions fill device memory with the
 * same bytes (see synth_core.h for why they agree bit for bit).
 *
 * This library is an input generator only.  It is linked neither into the
 * layer library nor into the CPU oracle; tests and the benchmark hand its
 * output to both.
 */
#include <cuda_runtime.h>
#include <math.h>
#include <stdlib.h>
#include <omp.h>
#include <stdint.h>
#include <string.h>

#include "synth_core.h"

#define SYN_API extern "C" __attribute__((visibility("default")))

static int syn_check_shape(int n_mats, int out_dim, int in_dim, int bits, int G) {
  if (n_mats <= 0 || out_dim <= 0 || in_dim <= 0) return 1;
  if (bits < 2 || bits > 8 || bits == 7) return 2;
  if (G != 32 && G != 64 && G != 128) return 2;
  if (in_dim % G != 0) return 3;
  return 0;
}

/* Matrix m of the tensor uses the stream syn_key(seed, tag + m). */
SYN_API int moeq_synth_tensor_host(uint64_t seed, uint64_t tag, int n_mats, int out_dim,
                                   int in_dim, int bits, int G, int requant_from4,
                                   uint32_t* w, uint16_t* scales, uint16_t* biases,
                                   int n_threads) {
  int rc = syn_check_shape(n_mats, out_dim, in_dim, bits, G);
  if (rc) return rc;
  const int64_t words_per_row = (int64_t)in_dim * bits / 32;
  const int groups = in_dim / G;
  const int64_t total_rows = (int64_t)n_mats * out_dim;
  if (n_threads <= 0) n_threads = omp_get_max_threads();
#pragma omp parallel for num_threads(n_threads) schedule(static)
  for (int64_t rr = 0; rr < total_rows; ++rr) {
    const int m = (int)(rr / out_dim);
    const int64_t row = rr % out_dim;
    const uint64_t key = syn_key(seed, tag + (uint64_t)m);
    for (int g = 0; g < groups; ++g)
      syn_make_group(key, row, in_dim, g, G, bits, requant_from4, w + rr * words_per_row,
                     scales + rr * groups + g, biases + rr * groups + g);
  }
  return 0;
}

__global__ void syn_tensor_kernel(uint64_t seed, uint64_t tag, int out_dim, int in_dim, int bits,
                                  int G, int requant_from4, int64_t total_groups, uint32_t* w,
                                  uint16_t* scales, uint16_t* biases) {
  const int groups = in_dim / G;
  const int64_t words_per_row = (int64_t)in_dim * bits / 32;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total_groups;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t rr = i / groups;
    const int g = (int)(i % groups);
    const int m = (int)(rr / out_dim);
    const int64_t row = rr % out_dim;
    const uint64_t key = syn_key(seed, tag + (uint64_t)m);
    syn_make_group(key, row, in_dim, g, G, bits, requant_from4, w + rr * words_per_row,
                   scales + rr * groups + g, biases + rr * groups + g);
  }
}

SYN_API int moeq_synth_tensor_dev(uint64_t seed, uint64_t tag, int n_mats, int out_dim,
                                  int in_dim, int bits, int G, int requant_from4, uint32_t* w,
                                  uint16_t* scales, uint16_t* biases, void* stream) {
  int rc = syn_check_shape(n_mats, out_dim, in_dim, bits, G);
  if (rc) return rc;
  const int64_t total_groups = (int64_t)n_mats * out_dim * (in_dim / G);
  int64_t blocks = (total_groups + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  syn_tensor_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
      seed, tag, out_dim, in_dim, bits, G, requant_from4, total_groups, w, scales, biases);
  return cudaGetLastError() == cudaSuccess ? 0 : 10;
}

/* MX FP4 banks: 4-bit E2M1 codes and one E8M0 byte per group of 32, from
 * the same weight streams as the affine tensors (syn_make_group_mx). */
SYN_API int moeq_synth_tensor_mx_host(uint64_t seed, uint64_t tag, int n_mats, int out_dim,
                                      int in_dim, uint32_t* w, uint8_t* e, int n_threads) {
  int rc = syn_check_shape(n_mats, out_dim, in_dim, 4, 32);
  if (rc) return rc;
  const int64_t words_per_row = (int64_t)in_dim / 8;
  const int groups = in_dim / 32;
  const int64_t total_rows = (int64_t)n_mats * out_dim;
  if (n_threads <= 0) n_threads = omp_get_max_threads();
#pragma omp parallel for num_threads(n_threads) schedule(static)
  for (int64_t rr = 0; rr < total_rows; ++rr) {
    const int m = (int)(rr / out_dim);
    const int64_t row = rr % out_dim;
    const uint64_t key = syn_key(seed, tag + (uint64_t)m);
    for (int g = 0; g < groups; ++g)
      syn_make_group_mx(key, row, in_dim, g, w + rr * words_per_row, e + rr * groups + g);
  }
  return 0;
}

__global__ void syn_tensor_mx_kernel(uint64_t seed, uint64_t tag, int out_dim, int in_dim,
                                     int64_t total_groups, uint32_t* w, uint8_t* e) {
  const int groups = in_dim / 32;
  const int64_t words_per_row = (int64_t)in_dim / 8;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total_groups;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t rr = i / groups;
    const int g = (int)(i % groups);
    const int m = (int)(rr / out_dim);
    const int64_t row = rr % out_dim;
    const uint64_t key = syn_key(seed, tag + (uint64_t)m);
    syn_make_group_mx(key, row, in_dim, g, w + rr * words_per_row, e + rr * groups + g);
  }
}

SYN_API int moeq_synth_tensor_mx_dev(uint64_t seed, uint64_t tag, int n_mats, int out_dim,
                                     int in_dim, uint32_t* w, uint8_t* e, void* stream) {
  int rc = syn_check_shape(n_mats, out_dim, in_dim, 4, 32);
  if (rc) return rc;
  const int64_t total_groups = (int64_t)n_mats * out_dim * (in_dim / 32);
  int64_t blocks = (total_groups + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  syn_tensor_mx_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
      seed, tag, out_dim, in_dim, total_groups, w, e);
  return cudaGetLastError() == cudaSuccess ? 0 : 10;
}

/* n bf16 values ~ N(0,1): element i = bf16_rne(syn_unit_normal(key, i)). */
SYN_API int moeq_synth_normal_bf16_host(uint64_t seed, uint64_t tag, int64_t n, uint16_t* out,
                                        int n_threads) {
  if (n < 0) return 1;
  const uint64_t key = syn_key(seed, tag);
  if (n_threads <= 0) n_threads = omp_get_max_threads();
#pragma omp parallel for num_threads(n_threads) schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = syn_bf16_rne(syn_unit_normal(key, (uint64_t)i));
  return 0;
}

__global__ void syn_normal_kernel(uint64_t key, int64_t n, uint16_t* out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = syn_bf16_rne(syn_unit_normal(key, (uint64_t)i));
}

SYN_API int moeq_synth_normal_bf16_dev(uint64_t seed, uint64_t tag, int64_t n, uint16_t* out,
                                       void* stream) {
  if (n < 0) return 1;
  if (n == 0) return 0;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  syn_normal_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(syn_key(seed, tag), n,
                                                                        out);
  return cudaGetLastError() == cudaSuccess ? 0 : 10;
}

/* Uniform double in (0, 1) from stream position i. */
static double syn_uniform_open(uint64_t key, uint64_t i) {
  uint64_t h = syn_mix64(key + (i + 1) * SYN_GOLDEN);
  return ((double)(h >> 11) + 0.5) * 0x1.0p-53;
}

/*
 * Router logits with a skewed expert load: expert popularity
 * p_e proportional to rank_e^(-zipf_s) (ranks 1..E from a seeded
 * Fisher-Yates permutation), logits[t][e] = ln p_e + Gumbel(0, 1).
 * Taking the top K of such logits samples K experts without replacement
 * with probability proportional to p (the Gumbel-top-k construction).
 * Host only: these drawn values are passed to both sides as inputs.
 */
SYN_API int moeq_synth_zipf_logits_host(uint64_t seed, uint64_t tag, int M, int E,
                                        double zipf_s, float* logits, int32_t* rank_out) {
  if (M < 0 || E <= 0) return 1;
  const uint64_t key = syn_key(seed, tag);
  int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
  if (!perm) return 11;
  for (int e = 0; e < E; ++e) perm[e] = e;
  for (int e = E - 1; e > 0; --e) {
    uint64_t h = syn_mix64(key ^ syn_mix64((uint64_t)e * 0xD1B54A32D192ED03ULL));
    int j = (int)(h % (uint64_t)(e + 1));
    int32_t t = perm[e];
    perm[e] = perm[j];
    perm[j] = t;
  }
  /* perm[r] = expert holding rank r+1 */
  double* lp = (double*)malloc(sizeof(double) * (size_t)E);
  if (!lp) {
    free(perm);
    return 11;
  }
  double z = 0.0;
  for (int r = 0; r < E; ++r) z += pow((double)(r + 1), -zipf_s);
  for (int r = 0; r < E; ++r) {
    lp[perm[r]] = log(pow((double)(r + 1), -zipf_s) / z);
    if (rank_out) rank_out[perm[r]] = r + 1;
  }
  const uint64_t gkey = syn_mix64(key + 0x5851F42D4C957F2DULL);
  for (int t = 0; t < M; ++t)
    for (int e = 0; e < E; ++e) {
      double u = syn_uniform_open(gkey, (uint64_t)t * (uint64_t)E + (uint64_t)e);
      logits[(size_t)t * E + e] = (float)(lp[e] - log(-log(u)));
    }
  free(lp);
  free(perm);
  return 0;
}

/* The fp32 draws of matrix `mat` before quantisation ([out][in]); used only
 * to check the quantiser's reconstruction error. */
SYN_API int moeq_synth_weights_f32_host(uint64_t seed, uint64_t tag, int mat, int out_dim,
                                        int in_dim, float* w) {
  if (out_dim <= 0 || in_dim <= 0) return 1;
  const uint64_t key = syn_key(seed, tag + (uint64_t)mat);
  for (int64_t i = 0; i < (int64_t)out_dim * in_dim; ++i) w[i] = syn_weight(key, (uint64_t)i);
  return 0;
}
