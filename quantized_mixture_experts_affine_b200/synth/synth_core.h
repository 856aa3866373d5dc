/*
 * Seeded synthetic-input recipe shared by the host generator (synth.cu, host
 * half) and the device generator (synth.cu, kernels).  Every step here is
 * integer arithmetic or one IEEE-754 correctly-rounded operation, so the host
 * and the device produce the same bytes for the same (seed, tag, index).
 *
 * This file holds no step of the layer forward itself.  It draws:
 *   - fp32 weights ~ N(0, 0.02) (Irwin-Hall sum of eight 16-bit uniforms,
 *     rescaled to unit variance; tails are cut at about 4.9 sigma),
 *   - bf16 activations ~ N(0, 1) by the same construction,
 * and quantises weights with the recipe the workload description fixes for
 * the affine packed format (MLX-style affine quantisation, as used by the
 * flash-moe and mlx pages): per group of G values along the input dimension,
 *   scale = bf16_rne((max - min) / (2^b - 1)),  bias = bf16_rne(min),
 *   q     = clamp(rint((w - bias) / scale), 0, 2^b - 1)   (q = 0 if scale == 0),
 * packed low bits first, 32/b values per uint32 word.
 *
 * The counter-based hash is SplitMix64 (Steele, Lea, Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014; finaliser constants as
 * published by Vigna).
 */
#ifndef MOEQ_SYNTH_CORE_H
#define MOEQ_SYNTH_CORE_H

#include <stdint.h>

#ifdef __CUDACC__
#define SYN_HD __host__ __device__ __forceinline__
#else
#define SYN_HD static inline
#endif

#define SYN_GOLDEN 0x9E3779B97F4A7C15ULL

SYN_HD uint64_t syn_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Key of one tensor stream: seed and a 64-bit tag naming the tensor. */
SYN_HD uint64_t syn_key(uint64_t seed, uint64_t tag) {
  return syn_mix64(seed ^ syn_mix64(tag + SYN_GOLDEN));
}

/* Odd integer in [-524280, 524280]: 2*S - 8*65535, S = sum of 8 uniforms. */
SYN_HD int32_t syn_irwin_hall8(uint64_t key, uint64_t i) {
  uint64_t h1 = syn_mix64(key + (2 * i + 1) * SYN_GOLDEN);
  uint64_t h2 = syn_mix64(key + (2 * i + 2) * SYN_GOLDEN);
  uint32_t s = 0;
  for (int j = 0; j < 4; ++j) {
    s += (uint32_t)((h1 >> (16 * j)) & 0xFFFFu);
    s += (uint32_t)((h2 >> (16 * j)) & 0xFFFFu);
  }
  return (int32_t)(2 * s) - 8 * 65535;
}

/* 0.02 / (2 * 65536 * sqrt(8/12)) and 1 / (2 * 65536 * sqrt(8/12)). */
#define SYN_KW 0x1.91530bd7c536fp-23
#define SYN_KX 0x1.3988e1409212ep-17

SYN_HD float syn_weight(uint64_t key, uint64_t i) {
  return (float)((double)syn_irwin_hall8(key, i) * SYN_KW);
}

SYN_HD float syn_unit_normal(uint64_t key, uint64_t i) {
  return (float)((double)syn_irwin_hall8(key, i) * SYN_KX);
}

SYN_HD uint16_t syn_bf16_rne(float f) {
  union { float f; uint32_t u; } v;
  v.f = f;
  if ((v.u & 0x7F800000u) == 0x7F800000u && (v.u & 0x007FFFFFu)) return (uint16_t)((v.u >> 16) | 0x40u);
  uint32_t r = v.u + 0x7FFFu + ((v.u >> 16) & 1u);
  return (uint16_t)(r >> 16);
}

SYN_HD float syn_bf16_to_f32(uint16_t h) {
  union { float f; uint32_t u; } v;
  v.u = ((uint32_t)h) << 16;
  return v.f;
}

/*
 * Quantise one group of n values (n = group size) at `bits` bits.
 * Writes q codes (one per value, unpacked) and the bf16 scale/bias bits.
 * The arithmetic is: one fp32 subtraction and one fp32 division for the
 * scale, one fp32 subtraction and one fp32 division per value, each
 * correctly rounded; rint is round-half-even.
 */
SYN_HD void syn_quantise_group(const float* w, int n, int bits, uint8_t* q,
                               uint16_t* scale_bits, uint16_t* bias_bits) {
  float mn = w[0], mx = w[0];
  for (int i = 1; i < n; ++i) {
    mn = w[i] < mn ? w[i] : mn;
    mx = w[i] > mx ? w[i] : mx;
  }
  const float levels = (float)((1 << bits) - 1);
  uint16_t sb = syn_bf16_rne((mx - mn) / levels);
  uint16_t bb = syn_bf16_rne(mn);
  float s = syn_bf16_to_f32(sb);
  float b = syn_bf16_to_f32(bb);
  for (int i = 0; i < n; ++i) {
    float v = 0.0f;
    if (s != 0.0f) {
#ifdef __CUDA_ARCH__
      v = rintf(__fdiv_rn(__fsub_rn(w[i], b), s));
#else
      v = rintf((w[i] - b) / s);
#endif
    }
    v = v < 0.0f ? 0.0f : v;
    v = v > levels ? levels : v;
    q[i] = (uint8_t)v;
  }
  *scale_bits = sb;
  *bias_bits = bb;
}

/* fp32 value of code q under bf16 scale/bias: one correctly rounded fma. */
SYN_HD float syn_dequant_f32(uint8_t q, uint16_t sb, uint16_t bb) {
#ifdef __CUDA_ARCH__
  return __fmaf_rn((float)q, syn_bf16_to_f32(sb), syn_bf16_to_f32(bb));
#else
  return fmaf((float)q, syn_bf16_to_f32(sb), syn_bf16_to_f32(bb));
#endif
}

/*
 * One (row, group) of a packed tensor: draws the G fp32 weights of that
 * group, quantises them (optionally first at 4 bits, dequantises, and
 * requantises at `bits`, the 4->2 bit requantisation of the flash-moe page),
 * and ORs the codes into the packed words of the row.  `words_row` points at
 * the first word of the row; the group covers words [g*G*bits/32, ...).
 */
SYN_HD void syn_make_group(uint64_t key, int64_t row, int in_dim, int g, int G,
                           int bits, int requant_from4, uint32_t* words_row,
                           uint16_t* scale_out, uint16_t* bias_out) {
  float w[128];
  uint8_t q[128];
  for (int i = 0; i < G; ++i)
    w[i] = syn_weight(key, (uint64_t)row * (uint64_t)in_dim + (uint64_t)(g * G + i));
  if (requant_from4) {
    uint16_t s4, b4;
    syn_quantise_group(w, G, 4, q, &s4, &b4);
    for (int i = 0; i < G; ++i) w[i] = syn_dequant_f32(q[i], s4, b4);
  }
  syn_quantise_group(w, G, bits, q, scale_out, bias_out);
  /* value j of the group at bit (g*G + j)*bits of the row's stream, low bits
   * first (3, 5 and 6 bits: a value may straddle two words); a group fills
   * whole words for every G in {32, 64, 128} */
  const int w0 = g * G * bits / 32, nw = G * bits / 32;
  for (int k = 0; k < nw; ++k) words_row[w0 + k] = 0;
  for (int j = 0; j < G; ++j) {
    const int bit = j * bits, k = bit / 32, off = bit % 32;
    words_row[w0 + k] |= (uint32_t)q[j] << off;
    if (off + bits > 32) words_row[w0 + k + 1] |= (uint32_t)q[j] >> (32 - off);
  }
}

/*
 * MX FP4 (OCP Microscaling Formats v1.0: E2M1 elements, one E8M0 scale per
 * block of 32; the mlx issue page's mode="mxfp4") of one group of 32 fp32
 * weights.  Shared exponent X = floor(log2(max|w|)) - 2 (2 = the largest
 * E2M1 exponent), stored as the byte X + 127 (clamped to 0..254); every
 * element is w / 2^X (exact) rounded to the nearest E2M1 value, ties to the
 * even mantissa, magnitudes above 6 saturating to 6; an all-zero group gets
 * the byte 0 and zero codes.  Codes: bit 3 sign, bits 2..1 exponent, bit 0
 * mantissa.
 */
SYN_HD uint8_t syn_e2m1_code(float v) {
  const uint8_t sign = v < 0.0f ? 8 : 0;
  const float a = v < 0.0f ? -v : v;
  uint8_t m;  /* magnitude code 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6 */
  if (a <= 0.25f) m = 0;
  else if (a < 0.75f) m = 1;
  else if (a <= 1.25f) m = 2;
  else if (a < 1.75f) m = 3;
  else if (a <= 2.5f) m = 4;
  else if (a < 3.5f) m = 5;
  else if (a <= 5.0f) m = 6;
  else m = 7;
  return (uint8_t)(sign | m);
}

SYN_HD void syn_make_group_mx(uint64_t key, int64_t row, int in_dim, int g, uint32_t* words_row,
                              uint8_t* e_out) {
  float w[32];
  float amax = 0.0f;
  for (int i = 0; i < 32; ++i) {
    w[i] = syn_weight(key, (uint64_t)row * (uint64_t)in_dim + (uint64_t)(g * 32 + i));
    const float a = w[i] < 0.0f ? -w[i] : w[i];
    amax = a > amax ? a : amax;
  }
  uint8_t q[32];
  uint8_t ebyte = 0;
  if (amax > 0.0f) {
    union { float f; uint32_t u; } v;
    v.f = amax;
    int ex = (int)((v.u >> 23) & 0xFFu) - 127;   /* floor(log2(amax)), amax normal */
    if (((v.u >> 23) & 0xFFu) == 0) ex = -127;   /* subnormal: below any scale used here */
    int X = ex - 2;
    X = X < -127 ? -127 : (X > 127 ? 127 : X);
    ebyte = (uint8_t)(X + 127);
    /* 2^-X as an fp32 power of two (X in [-126, 127]: normal; -127 clamps) */
    union { float f; uint32_t u; } inv;
    const int ie = -X + 127;
    inv.u = (uint32_t)(ie < 1 ? 1 : (ie > 254 ? 254 : ie)) << 23;
    for (int i = 0; i < 32; ++i) q[i] = syn_e2m1_code(w[i] * inv.f);
  } else {
    for (int i = 0; i < 32; ++i) q[i] = 0;
  }
  *e_out = ebyte;
  for (int k = 0; k < 4; ++k) {
    uint32_t word = 0;
    for (int j = 0; j < 8; ++j) word |= ((uint32_t)q[k * 8 + j]) << (4 * j);
    words_row[g * 4 + k] = word;
  }
}

#endif
