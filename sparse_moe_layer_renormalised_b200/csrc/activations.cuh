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

// The same SiTU-GLU for bf16-stored outputs, from CUDA's fast exponential and
// division intrinsics: sigmoid(g) = 1 / (1 + e^-g) and
// tanh(x) = 1 - 2 / (e^(2x) + 1).  Relative error is around 1e-6, far below
// the 2^-9 rounding of the bf16 result; e^(2x) overflowing to +inf gives
// tanh = 1 and underflowing to 0 gives -1, as it should.
__device__ __forceinline__ float fast_tanh(float x) { return 1.0f - __fdividef(2.0f, __expf(2.0f * x) + 1.0f); }

__device__ __forceinline__ float situ_glu_fast(float g, float v, float c, float inv_c) {
  const float sg = __fdividef(1.0f, 1.0f + __expf(-g));
  return sg * (c * fast_tanh(g * inv_c)) * (c * fast_tanh(v * inv_c));
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
