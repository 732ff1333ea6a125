/*
 * Seeded synthetic-input generator: definitions shared by the host (C) and
 * device (CUDA) halves of the generator module.
 *
 * This module produces the inputs of the layer (activations, weights, bias,
 * gain, MXFP4-packed weights).  It contains none of the layer's arithmetic;
 * both the CPU oracle and the CUDA library consume what it produces, and the
 * two halves below produce bit-identical values for the same
 * (seed, tensor id, element index).
 *
 * Random source: Philox-4x32-10, the counter-based generator of Salmon,
 * Moraes, Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3"
 * (SC'11).  Counter = (element index lo, element index hi, 0, 0),
 * key = (seed, tensor id).
 *
 * Normal variates: the eight 16-bit halves of one Philox output are summed
 * (an Irwin-Hall sum of 8 discrete uniforms), centred, converted to fp32
 * exactly (|sum| < 2^24) and multiplied once by an fp32 scale.  Every step
 * is exact or a single IEEE round-to-nearest operation, so the host and the
 * device agree bit for bit.  The result has mean 0 and the requested
 * standard deviation; its tails are bounded at about 4.9 sigma.
 *
 * MXFP4 (OCP Microscaling Formats v1.0): blocks of 32 consecutive elements
 * along K share one E8M0 scale 2^(floor(log2(amax)) - 2); each element is
 * rounded to nearest-even onto the E2M1 grid {0,0.5,1,1.5,2,3,4,6} after
 * division by the scale, saturating at 6.  Two codes per byte, the even K
 * index in the low nibble.
 */
#ifndef MOE_GEN_COMMON_H
#define MOE_GEN_COMMON_H

#include <stdint.h>

#ifdef __CUDACC__
#define GEN_HD __host__ __device__ __forceinline__
#else
#define GEN_HD static inline
#endif

#define GEN_PHILOX_M0 0xD2511F53u
#define GEN_PHILOX_M1 0xCD9E8D57u
#define GEN_PHILOX_W0 0x9E3779B9u
#define GEN_PHILOX_W1 0xBB67AE85u

GEN_HD void gen_mulhilo32(uint32_t a, uint32_t b, uint32_t* hi, uint32_t* lo) {
  uint64_t p = (uint64_t)a * (uint64_t)b;
  *hi = (uint32_t)(p >> 32);
  *lo = (uint32_t)p;
}

/* One Philox-4x32 round: two 32x32->64 multiplies, outputs crossed and
 * xored with the round key. */
GEN_HD void gen_philox_round(uint32_t c[4], uint32_t k0, uint32_t k1) {
  uint32_t hi0, lo0, hi1, lo1;
  gen_mulhilo32(GEN_PHILOX_M0, c[0], &hi0, &lo0);
  gen_mulhilo32(GEN_PHILOX_M1, c[2], &hi1, &lo1);
  uint32_t n0 = hi1 ^ c[1] ^ k0;
  uint32_t n2 = hi0 ^ c[3] ^ k1;
  c[0] = n0;
  c[1] = lo1;
  c[2] = n2;
  c[3] = lo0;
}

/* Philox-4x32 with 10 rounds; the key is bumped by the Weyl constants
 * between rounds. */
GEN_HD void gen_philox4x32_10_impl(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
  uint32_t k0 = key[0], k1 = key[1];
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += GEN_PHILOX_W0;
      k1 += GEN_PHILOX_W1;
    }
    gen_philox_round(c, k0, k1);
  }
  out[0] = c[0];
  out[1] = c[1];
  out[2] = c[2];
  out[3] = c[3];
}

/* Centred Irwin-Hall sum of the eight 16-bit halves of Philox(index).
 * Range [-262140, 262140]; exactly representable in fp32. */
GEN_HD int32_t gen_ih8_centred(uint32_t seed, uint32_t tensor_id, uint64_t index) {
  uint32_t ctr[4] = {(uint32_t)index, (uint32_t)(index >> 32), 0u, 0u};
  uint32_t key[2] = {seed, tensor_id};
  uint32_t w[4];
  gen_philox4x32_10_impl(ctr, key, w);
  int32_t s = 0;
  for (int i = 0; i < 4; ++i) s += (int32_t)(w[i] & 0xFFFFu) + (int32_t)(w[i] >> 16);
  return s - 4 * 65535;
}

/* fp32 -> bf16 bits, round to nearest even (inputs here are finite). */
GEN_HD uint16_t gen_f32_to_bf16_bits(float f) {
  union {
    float f;
    uint32_t u;
  } v;
  v.f = f;
  uint32_t u = v.u;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

GEN_HD uint32_t gen_f32_bits(float f) {
  union {
    float f;
    uint32_t u;
  } v;
  v.f = f;
  return v.u;
}

GEN_HD float gen_bits_f32(uint32_t u) {
  union {
    float f;
    uint32_t u;
  } v;
  v.u = u;
  return v.f;
}

/* E2M1 code (0..7, magnitude only) of |q|, round to nearest even with
 * saturation at 6.  Grid: code 0..7 -> 0, 0.5, 1, 1.5, 2, 3, 4, 6.  At a
 * midpoint the code with the even last bit wins. */
GEN_HD uint32_t gen_e2m1_magnitude_code(float a) {
  if (a <= 0.25f) return 0u;
  if (a < 0.75f) return 1u;
  if (a <= 1.25f) return 2u;
  if (a < 1.75f) return 3u;
  if (a <= 2.5f) return 4u;
  if (a < 3.5f) return 5u;
  if (a <= 5.0f) return 6u;
  return 7u;
}

/* Quantise one block of 32 fp32 values to MXFP4: writes 16 packed bytes and
 * returns the E8M0 scale byte. */
GEN_HD uint8_t gen_mxfp4_block(const float v[32], uint8_t packed[16]) {
  float amax = 0.0f;
  for (int i = 0; i < 32; ++i) {
    float a = v[i] < 0.0f ? -v[i] : v[i];
    if (a > amax) amax = a;
  }
  int32_t e;
  if (amax == 0.0f) {
    e = -127;
  } else {
    int32_t biased = (int32_t)((gen_f32_bits(amax) >> 23) & 0xFFu);
    e = (biased == 0 ? -127 : biased - 127) - 2; /* floor(log2 amax) - emax(E2M1) */
  }
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  /* 2^-e as an fp32 (exact power of two; 127 - e in [0, 254]) */
  int32_t inv_biased = 127 - e;
  float inv_scale = inv_biased >= 1 ? gen_bits_f32((uint32_t)inv_biased << 23)
                                    : gen_bits_f32(0x00400000u); /* 2^-127, subnormal */
  for (int i = 0; i < 16; ++i) packed[i] = 0;
  for (int i = 0; i < 32; ++i) {
    float q = v[i] * inv_scale;
    float a = q < 0.0f ? -q : q;
    uint32_t code = gen_e2m1_magnitude_code(a);
    if (q < 0.0f && code != 0u) code |= 8u;
    packed[i >> 1] |= (uint8_t)(code << ((i & 1) * 4));
  }
  return (uint8_t)(e + 127);
}

#endif /* MOE_GEN_COMMON_H */
