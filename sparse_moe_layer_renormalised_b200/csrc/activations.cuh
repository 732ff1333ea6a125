// Element-wise functions of the layer, in fp32 (CUDA's expf / tanhf).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace moe {

// Router score: sigmoid of the logit ("ルーターは計算の割当器": s = Sigmoid(W_r x)).
__device__ __forceinline__ float sigmoid_f32(float l) { return 1.0f / (1.0f + expf(-l)); }

// SiTU-GLU: SwiGLU sigmoid(g) * g * v with the linear factor g and the up
// branch v replaced by the smooth caps c * tanh(. / c)  (tech-report summary,
// section "幅のスケーリング：Stable LatentMoE"; closed form is this library's
// reading of that description).  Used by the fp32 path.
__device__ __forceinline__ float situ_glu_f32(float g, float v, float c) {
  return sigmoid_f32(g) * (c * tanhf(g / c)) * (c * tanhf(v / c));
}

// e^y - 1 given A = e^y: for |y| < 0.1 the five-term Taylor series of e^y - 1
// about 0 (truncation below 2e-8 relative), else A - 1 (whose cancellation
// costs at most ~6e-7 relative there).
__device__ __forceinline__ float expm1_from(float y, float A) {
  const float s = y * (1.0f + y * (0.5f + y * (1.0f / 6.0f + y * (1.0f / 24.0f + y * (1.0f / 120.0f)))));
  return fabsf(y) < 0.1f ? s : A - 1.0f;
}

// The same SiTU-GLU for bf16-stored outputs, from CUDA's fast exponential
// and division intrinsics.  With A = e^(2g/c), B = e^(2v/c) and C = e^(-g):
//   sigmoid(g) = 1 / (1 + C),  tanh(g/c) = (A - 1) / (A + 1),  tanh(v/c) = (B - 1) / (B + 1),
// so  h = c^2 (A - 1)(B - 1) / ((1 + C)(A + 1)(B + 1)):  three exponentials and
// one division (four MUFU operations instead of six for the factors
// separately); A - 1 and B - 1 come from expm1_from so they do not cancel
// near zero.  The exponents are clamped so no product overflows: 2x/c to
// [-20, 20] (tanh is +-1 in fp32 beyond |x/c| = 9.1) and -g to at most 40,
// so for g < -40 the result is only known to be below 5e-18 c^2 in size.
// Elsewhere the relative error is below 2e-6 (this algebra in fp32 against
// the fp64 definition, c = 1, 10, 100), far below the 2^-9 relative rounding
// of the stored bf16 h.
__device__ __forceinline__ float situ_glu_fast(float g, float v, float c, float inv_c) {
  const float two_inv_c = 2.0f * inv_c;
  const float yg = fminf(fmaxf(g * two_inv_c, -20.0f), 20.0f);
  const float yv = fminf(fmaxf(v * two_inv_c, -20.0f), 20.0f);
  const float A = __expf(yg);
  const float B = __expf(yv);
  const float C = __expf(fminf(-g, 40.0f));
  const float num = expm1_from(yg, A) * expm1_from(yv, B);
  const float den = ((1.0f + C) * (A + 1.0f)) * (B + 1.0f);
  return (c * c) * __fdividef(num, den);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Low (hi = 0) or high (hi = 1) bf16 of a packed pair.
__device__ __forceinline__ __nv_bfloat16 bf16_half(uint32_t packed, int hi) {
  const unsigned short bits = static_cast<unsigned short>(hi ? (packed >> 16) : (packed & 0xFFFFu));
  return __ushort_as_bfloat16(bits);
}

}  // namespace moe
