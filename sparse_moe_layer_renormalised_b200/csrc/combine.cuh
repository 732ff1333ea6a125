// Weighted combine of the k expert outputs of each token, fused with RMSNorm
// (page "Kimi K3の896エキスパートを「896人の専門家」と呼ぶと何がズレるか",
// section "K3のエキスパートは896個の小型LLMではない": u = sum_i p_i E_i(z),
// y = ... + W_up RMSNorm(u)).
//
// Block = one token, 128 threads, thread i owns float4 columns i, i+128, ...
// u is a gather over y_perm rows in fixed slot order (no float atomics), the
// sum of squares is reduced in a fixed tree, so results are deterministic.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "activations.cuh"

namespace moe {

constexpr int COMBINE_THREADS = 128;

template <typename OutT>
__device__ __forceinline__ void store4(OutT* dst, float4 v);

template <>
__device__ __forceinline__ void store4<float>(float* dst, float4 v) {
  *reinterpret_cast<float4*>(dst) = v;
}

template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* dst, float4 v) {
  uint2 u;
  u.x = pack_bf16x2(v.x, v.y);
  u.y = pack_bf16x2(v.z, v.w);
  *reinterpret_cast<uint2*>(dst) = u;
}

// VPT = float4 vectors per thread (L <= 4 * 128 * VPT).
template <typename OutT, int VPT>
__global__ void __launch_bounds__(COMBINE_THREADS)
    combine_rmsnorm_kernel(const float* __restrict__ y_perm, const int32_t* __restrict__ inv_perm,
                           const float* __restrict__ topk_w, const float* __restrict__ gamma, int k, int L, float eps,
                           float* __restrict__ u_out, OutT* __restrict__ n_out) {
  const long long t = blockIdx.x;
  const int nv = L >> 2;
  float4 acc[VPT];
#pragma unroll
  for (int v = 0; v < VPT; ++v) acc[v] = make_float4(0.f, 0.f, 0.f, 0.f);
  const int32_t* ip = inv_perm + t * k;
  const float* pw = topk_w + t * k;
  for (int j = 0; j < k; ++j) {
    const long long pos = ip[j];
    const float pj = pw[j];
    const float4* row = reinterpret_cast<const float4*>(y_perm + pos * L);
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const int i = threadIdx.x + COMBINE_THREADS * v;
      if (i < nv) {
        const float4 y = row[i];
        acc[v].x = fmaf(pj, y.x, acc[v].x);
        acc[v].y = fmaf(pj, y.y, acc[v].y);
        acc[v].z = fmaf(pj, y.z, acc[v].z);
        acc[v].w = fmaf(pj, y.w, acc[v].w);
      }
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    ss = fmaf(acc[v].x, acc[v].x, ss);
    ss = fmaf(acc[v].y, acc[v].y, ss);
    ss = fmaf(acc[v].z, acc[v].z, ss);
    ss = fmaf(acc[v].w, acc[v].w, ss);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  __shared__ float red[COMBINE_THREADS / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < COMBINE_THREADS / 32; ++w) tot += red[w];
  const float r = rsqrtf(tot / static_cast<float>(L) + eps);
  const float4* g4 = reinterpret_cast<const float4*>(gamma);
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    const int i = threadIdx.x + COMBINE_THREADS * v;
    if (i < nv) {
      const float4 g = g4[i];
      const float4 a = acc[v];
      const float4 n = make_float4(g.x * (a.x * r), g.y * (a.y * r), g.z * (a.z * r), g.w * (a.w * r));
      store4<OutT>(n_out + t * L + 4 * i, n);
      if (u_out != nullptr) *reinterpret_cast<float4*>(u_out + t * L + 4 * i) = a;
    }
  }
}

}  // namespace moe
