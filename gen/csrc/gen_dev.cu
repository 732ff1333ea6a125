// Device half of the seeded synthetic-input generator.  Fills device buffers
// with exactly the values the host half (gen_host.c) produces for the same
// (seed, tensor id, element index): the multiply and the add below are the
// explicitly rounded fp32 operations, so no contraction into an FMA can
// change a bit.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gen_common.h"

namespace {

__device__ __forceinline__ float gen_value_dev(uint32_t seed, uint32_t tid, uint64_t index, float scale,
                                               float offset) {
  float c = (float)gen_ih8_centred(seed, tid, index);
  return __fadd_rn(__fmul_rn(c, scale), offset);
}

__global__ void gen_f32_kernel(uint32_t seed, uint32_t tid, uint64_t start, uint64_t count, float scale,
                               float offset, float* out) {
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride)
    out[i] = gen_value_dev(seed, tid, start + i, scale, offset);
}

__global__ void gen_bf16_kernel(uint32_t seed, uint32_t tid, uint64_t start, uint64_t count, float scale,
                                float offset, uint16_t* out) {
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride)
    out[i] = gen_f32_to_bf16_bits(gen_value_dev(seed, tid, start + i, scale, offset));
}

// One thread per 32-element block of one row.
__global__ void gen_mxfp4_kernel(uint32_t seed, uint32_t tid, uint64_t row_start, uint64_t nrows, uint64_t K,
                                 float scale, uint8_t* codes, uint8_t* scales) {
  uint64_t bpr = K / 32;
  uint64_t nblk = nrows * bpr;
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t g = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; g < nblk; g += stride) {
    uint64_t r = g / bpr, b = g % bpr;
    uint64_t row = row_start + r;
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = gen_value_dev(seed, tid, row * K + b * 32 + (uint64_t)i, scale, 0.0f);
    uint8_t packed[16];
    uint8_t s = gen_mxfp4_block(v, packed);
    uint4 w;
    w.x = (uint32_t)packed[0] | ((uint32_t)packed[1] << 8) | ((uint32_t)packed[2] << 16) | ((uint32_t)packed[3] << 24);
    w.y = (uint32_t)packed[4] | ((uint32_t)packed[5] << 8) | ((uint32_t)packed[6] << 16) | ((uint32_t)packed[7] << 24);
    w.z = (uint32_t)packed[8] | ((uint32_t)packed[9] << 8) | ((uint32_t)packed[10] << 16) | ((uint32_t)packed[11] << 24);
    w.w = (uint32_t)packed[12] | ((uint32_t)packed[13] << 8) | ((uint32_t)packed[14] << 16) | ((uint32_t)packed[15] << 24);
    *reinterpret_cast<uint4*>(codes + r * (K / 2) + b * 16) = w;
    scales[r * bpr + b] = s;
  }
}

int grid_for(uint64_t n) {
  uint64_t g = (n + 255) / 256;
  if (g > 148ull * 64ull) g = 148ull * 64ull;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace

extern "C" {

int gen_dev_fill_f32(uint32_t seed, uint32_t tid, uint64_t start, uint64_t count, float scale, float offset,
                     float* out, cudaStream_t stream) {
  if (count == 0) return 0;
  gen_f32_kernel<<<grid_for(count), 256, 0, stream>>>(seed, tid, start, count, scale, offset, out);
  return (int)cudaGetLastError();
}

int gen_dev_fill_bf16(uint32_t seed, uint32_t tid, uint64_t start, uint64_t count, float scale, float offset,
                      uint16_t* out, cudaStream_t stream) {
  if (count == 0) return 0;
  gen_bf16_kernel<<<grid_for(count), 256, 0, stream>>>(seed, tid, start, count, scale, offset, out);
  return (int)cudaGetLastError();
}

// codes must be 16-byte aligned; K % 32 == 0.
int gen_dev_fill_mxfp4(uint32_t seed, uint32_t tid, uint64_t row_start, uint64_t nrows, uint64_t K, float scale,
                       uint8_t* codes, uint8_t* scales, cudaStream_t stream) {
  if (nrows == 0) return 0;
  if (K % 32 != 0 || (((uintptr_t)codes) & 15u) != 0) return (int)cudaErrorInvalidValue;
  gen_mxfp4_kernel<<<grid_for(nrows * (K / 32)), 256, 0, stream>>>(seed, tid, row_start, nrows, K, scale, codes,
                                                                    scales);
  return (int)cudaGetLastError();
}

}  // extern "C"
