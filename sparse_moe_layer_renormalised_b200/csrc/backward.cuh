// Backward pass of the layer with the expert selection held fixed: the top-k
// choice is a discrete function of the biased keys and has no gradient, while
// the mixture weights p_j = s_{e_j} / sum_j' s_{e_j'} are differentiable in the
// router scores s = Sigmoid(W_r x), so gradients reach the router through p
// only and the selection bias gets none (page "Kimi K3の896エキスパートを
// 「896人の専門家」と呼ぶと何がズレるか", sections "ルーターは計算の割当器" and
// "ルーター専用の独立訓練はない": the router is trained with the model, only its
// bias is set by Quantile Balancing).
//
// The forward quantities the gradients need are recomputed in fp32 from the
// inputs (no bf16 storage rounding), so the result is the gradient of the
// layer function itself.  Contractions run on a strided CUDA-core GEMM with
// fp32 accumulation; every reduction has a fixed order, so the results are
// deterministic.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "activations.cuh"
#include "ptx.cuh"

namespace moe {

// ------------------------------------------------------------------------------ strided GEMM
//   C[m, n] = beta * C[m, n] + sum_k A(m, k) * B(k, n)
// A(m, k) = a[m * a_m + k * a_k], B(k, n) = b[k * b_k + n * b_n] (element
// types TA / TB, fp32 or bf16), C fp32 [M, N] with row stride ldc; beta is 0
// or 1.  Three ways of grouping the problems by expert (blockIdx.z or the tile
// table), chosen by `mode`:
//   kBwDense:   one problem;
//   kBwRows:    rows M come from a tile table {expert, row0, nrows} (rows of
//               the expert-major buffers; A and C are offset by row0 rows and
//               B by expert * b_e elements);
//   kBwKRows:   one problem per expert (blockIdx.z): K runs over the expert's
//               rows offsets[e] .. offsets[e+1]-1 (A and B offset by those
//               rows), C offset by expert * c_e elements (weight gradients).
enum BwMode : int { kBwDense = 0, kBwRows = 1, kBwKRows = 2 };

struct BwGemm {
  const void* a;
  long long a_m, a_k;
  const void* b;
  long long b_k, b_n, b_e;
  float* c;
  long long ldc, c_e;
  int M, N, K;
  float beta;
  const int4* tile_table;  // kBwRows
  const int* num_tiles;    // kBwRows
  const int* offsets;      // kBwKRows: [E + 1]
  long long a_row, b_row;  // kBwKRows: elements per row step of A (along k) and B (along k)
};

constexpr int BW_TILE = 64;
constexpr int BW_KC = 16;
constexpr int BW_THREADS = 256;

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// 64 x 64 output tile per block, 4 x 4 per thread, K in chunks of 16 staged
// through shared memory (converted to fp32).  The k-sum of each output runs
// in ascending k.
template <typename TA, typename TB, int MODE>
__global__ void __launch_bounds__(BW_THREADS) bw_gemm_kernel(const BwGemm g) {
  __shared__ float As[BW_KC][BW_TILE + 1];
  __shared__ float Bs[BW_KC][BW_TILE + 1];
  const TA* A = static_cast<const TA*>(g.a);
  const TB* B = static_cast<const TB*>(g.b);
  float* C = g.c;
  int M = g.M, K = g.K;
  int m0 = blockIdx.y * BW_TILE;
  const int n0 = blockIdx.x * BW_TILE;
  long long k_base = 0;
  if (MODE == kBwRows) {
    if (static_cast<int>(blockIdx.y) >= *g.num_tiles) return;
    const int4 t = g.tile_table[blockIdx.y];
    A += static_cast<long long>(t.y) * g.a_m;
    C += static_cast<long long>(t.y) * g.ldc;
    B += static_cast<long long>(t.x) * g.b_e;
    M = t.z;
    m0 = 0;
  } else if (MODE == kBwKRows) {
    const int e = blockIdx.z;
    const int r0 = g.offsets[e], r1 = g.offsets[e + 1];
    k_base = r0;
    K = r1 - r0;
    C += static_cast<long long>(e) * g.c_e;
  }
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  const long long a_kstep = MODE == kBwKRows ? g.a_row : g.a_k;
  const long long b_kstep = MODE == kBwKRows ? g.b_row : g.b_k;
  // consecutive threads walk the operand's contiguous index (coalesced loads)
  const bool a_k_fast = a_kstep == 1, b_k_fast = b_kstep == 1;
  for (int kc = 0; kc < K; kc += BW_KC) {
    for (int i = threadIdx.x; i < BW_KC * BW_TILE; i += BW_THREADS) {
      int kk, mm;
      if (a_k_fast) {
        mm = i / BW_KC;
        kk = i - mm * BW_KC;
      } else {
        kk = i / BW_TILE;
        mm = i - kk * BW_TILE;
      }
      const int m = m0 + mm, k = kc + kk;
      float av = 0.f;
      if (m < M && k < K) av = to_f32(A[static_cast<long long>(m) * g.a_m + (k_base + k) * a_kstep]);
      As[kk][mm] = av;
    }
    for (int i = threadIdx.x; i < BW_KC * BW_TILE; i += BW_THREADS) {
      int kk, nn;
      if (b_k_fast) {
        nn = i / BW_KC;
        kk = i - nn * BW_KC;
      } else {
        kk = i / BW_TILE;
        nn = i - kk * BW_TILE;
      }
      const int n = n0 + nn, k = kc + kk;
      float bv = 0.f;
      if (n < g.N && k < K) bv = to_f32(B[(k_base + k) * b_kstep + static_cast<long long>(n) * g.b_n]);
      Bs[kk][nn] = bv;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BW_KC; ++kk) {
      float a4[4], b4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a4[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b4[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a4[i], b4[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= g.N) continue;
      float* cp = C + static_cast<long long>(m) * g.ldc + n;
      *cp = g.beta != 0.f ? *cp + acc[i][j] : acc[i][j];
    }
  }
}

// ------------------------------------------------------------------------------ element-wise steps
constexpr int BW_EW_THREADS = 256;

__device__ __forceinline__ float sig(float x) { return 1.0f / (1.0f + expf(-x)); }

// s = sigmoid(logits), in place.
__global__ void bw_sigmoid_kernel(float* s, long long n) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) s[i] = sig(s[i]);
}

// p[t, j] = s[t, idx[t, j]] / sum_j' s[t, idx[t, j']]  (sum in slot order)
__global__ void bw_mix_kernel(const float* s, const int32_t* idx, long long T, int E, int k, float* p) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= T) return;
  float sum = 0.f;
  for (int j = 0; j < k; ++j) sum += s[t * E + idx[t * k + j]];
  for (int j = 0; j < k; ++j) p[t * k + j] = s[t * E + idx[t * k + j]] / sum;
}

// g, v pre-activations -> h = SiTU-GLU(g, v) (fp32, exact CUDA functions)
__global__ void bw_situ_kernel(const float* g, const float* v, long long n, float c, float* h) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) h[i] = situ_glu_f32(g[i], v[i], c);
}

// (dg, dv) from dh:  h = sigma(g) * c tanh(g/c) * c tanh(v/c)
//   dh/dg = c tanh(v/c) * c * [sigma(g)(1 - sigma(g)) tanh(g/c) + sigma(g)(1 - tanh(g/c)^2) / c]
//   dh/dv = sigma(g) * c tanh(g/c) * (1 - tanh(v/c)^2)
// dg overwrites g and dv overwrites v.
__global__ void bw_situ_grad_kernel(float* g, float* v, const float* dh, long long n, float c) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float gg = g[i], vv = v[i], d = dh[i];
  const float sg = sig(gg), tg = tanhf(gg / c), tv = tanhf(vv / c);
  const float dhdg = (c * tv) * c * (sg * (1.0f - sg) * tg + sg * (1.0f - tg * tg) / c);
  const float dhdv = sg * (c * tg) * (1.0f - tv * tv);
  g[i] = d * dhdg;
  v[i] = d * dhdv;
}

// Block = token.  u = sum_j p_j y_perm[inv(t, j)] (slot order); r = sqrt(mean(u^2) + eps);
// n = gamma * u / r.  Writes u, n and r.
__global__ void __launch_bounds__(BW_EW_THREADS)
    bw_combine_kernel(const float* y_perm, const int32_t* inv_perm, const float* p, const float* gamma, int k, int L,
                      float eps, float* u, float* n, float* r_out) {
  const long long t = blockIdx.x;
  __shared__ float red[BW_EW_THREADS / 32];
  float ss = 0.f;
  for (int l = threadIdx.x; l < L; l += BW_EW_THREADS) {
    float a = 0.f;
    for (int j = 0; j < k; ++j) a = fmaf(p[t * k + j], y_perm[static_cast<long long>(inv_perm[t * k + j]) * L + l], a);
    u[t * L + l] = a;
    ss = fmaf(a, a, ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < BW_EW_THREADS / 32; ++w) tot += red[w];
  const float r = sqrtf(tot / static_cast<float>(L) + eps);
  for (int l = threadIdx.x; l < L; l += BW_EW_THREADS) n[t * L + l] = gamma[l] * u[t * L + l] / r;
  if (threadIdx.x == 0) r_out[t] = r;
}

// Block = token.  RMSNorm and combine backward:
//   du = gamma dn / r - u * (sum_l gamma_l dn_l u_l) / (L r^3)
//   dp_j = <du, y_j>;  dy_perm[inv(t, j)] = p_j du
__global__ void __launch_bounds__(BW_EW_THREADS)
    bw_combine_grad_kernel(const float* dn, const float* u, const float* r_in, const float* gamma, const float* y_perm,
                           const int32_t* inv_perm, const float* p, int k, int L, float* du, float* dp,
                           float* dy_perm) {
  const long long t = blockIdx.x;
  __shared__ float red[BW_EW_THREADS / 32];
  const float r = r_in[t];
  float dot = 0.f;
  for (int l = threadIdx.x; l < L; l += BW_EW_THREADS) dot = fmaf(gamma[l] * dn[t * L + l], u[t * L + l], dot);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = dot;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < BW_EW_THREADS / 32; ++w) tot += red[w];
  __syncthreads();
  const float coef = tot / (static_cast<float>(L) * r * r * r);
  for (int l = threadIdx.x; l < L; l += BW_EW_THREADS) {
    const float d = gamma[l] * dn[t * L + l] / r - u[t * L + l] * coef;
    du[t * L + l] = d;
    for (int j = 0; j < k; ++j) dy_perm[static_cast<long long>(inv_perm[t * k + j]) * L + l] = p[t * k + j] * d;
  }
  // dp_j = <du, y_j>, one block-wide reduction per slot (fixed order)
  for (int j = 0; j < k; ++j) {
    float a = 0.f;
    const float* yj = y_perm + static_cast<long long>(inv_perm[t * k + j]) * L;
    for (int l = threadIdx.x; l < L; l += BW_EW_THREADS) {
      const float d = gamma[l] * dn[t * L + l] / r - u[t * L + l] * coef;
      a = fmaf(d, yj[l], a);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    if (threadIdx.x == 0) {
      float s = 0.f;
      for (int w = 0; w < BW_EW_THREADS / 32; ++w) s += red[w];
      dp[t * k + j] = s;
    }
    __syncthreads();
  }
}

// dgamma[l] = sum_t dn[t, l] * u[t, l] / r[t]  (t ascending)
__global__ void bw_dgamma_kernel(const float* dn, const float* u, const float* r, long long T, int L, float* dgamma) {
  const int l = blockIdx.x * blockDim.x + threadIdx.x;
  if (l >= L) return;
  float a = 0.f;
  for (long long t = 0; t < T; ++t) a = fmaf(dn[t * L + l], u[t * L + l] / r[t], a);
  dgamma[l] = a;
}

// Router backward: with S = sum_j s_{e_j},  ds_{e_j} = (dp_j - sum_j' p_j' dp_j') / S,
// dl = ds * s (1 - s) at the selected experts, 0 elsewhere.  dl [T, E] is
// cleared and written here.
__global__ void bw_router_grad_kernel(const float* s, const int32_t* idx, const float* p, const float* dp, long long T,
                                      int E, int k, float* dl) {
  const long long t = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) dl[t * E + e] = 0.f;
  __syncthreads();
  if (threadIdx.x == 0) {
    float S = 0.f, pdp = 0.f;
    for (int j = 0; j < k; ++j) {
      S += s[t * E + idx[t * k + j]];
      pdp = fmaf(p[t * k + j], dp[t * k + j], pdp);
    }
    for (int j = 0; j < k; ++j) {
      const int e = idx[t * k + j];
      const float se = s[t * E + e];
      dl[t * E + e] = (dp[t * k + j] - pdp) / S * se * (1.0f - se);
    }
  }
}

// dz[t] = sum_j dz_perm[inv(t, j)]  (slot order)
__global__ void bw_gather_sum_kernel(const float* dz_perm, const int32_t* inv_perm, long long T, int k, int L,
                                     float* dz) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= T * L) return;
  const long long t = i / L;
  const int l = static_cast<int>(i - t * L);
  float a = 0.f;
  for (int j = 0; j < k; ++j) a += dz_perm[static_cast<long long>(inv_perm[t * k + j]) * L + l];
  dz[i] = a;
}

// dst[r] = src[rows[r]] for fp32 or bf16 rows (z in expert-major order, fp32 out)
template <typename T>
__global__ void bw_gather_rows_f32_kernel(const T* src, const int32_t* rows, long long R, int L, float* dst) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= R * L) return;
  const long long r = i / L;
  const int l = static_cast<int>(i - r * L);
  dst[i] = to_f32(src[static_cast<long long>(rows[r]) * L + l]);
}

}  // namespace moe
