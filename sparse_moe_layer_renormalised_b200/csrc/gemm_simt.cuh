// fp32 CUDA-core GEMM with the same tiling semantics as the tcgen05 kernel
// (dense or grouped rows, K segments, paired gate/up B, the same epilogues).
// Used for layers held in fp32, which the bf16 tensor-core path does not take.
// Block tile: 32 rows x 32 output columns, 256 threads (1 row x 4 columns each).
#pragma once

#include "activations.cuh"
#include "gemm_tc.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int SIMT_MAX_SEG = 4;

struct SimtParams {
  const float* A[SIMT_MAX_SEG];
  long long lda[SIMT_MAX_SEG];
  const float* B[SIMT_MAX_SEG];  // PAIRED: B[0] gate rows, B[1] up rows
  long long ldb[SIMT_MAX_SEG];
  int seg_k[SIMT_MAX_SEG];
  int nseg;
  int M;                      // dense rows
  const int4* tile_table;     // grouped (128-row tiles), or nullptr
  const int* num_m_tiles_dev;
  int N;
  int b_rows_per_expert;
  void* out;  // float
  long long ldo;
  float situ_c;
};

template <int EPI, bool PAIRED>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const SimtParams p) {
  __shared__ float As[32][33];
  __shared__ float Bs[32][33];
  __shared__ float Bv[PAIRED ? 32 : 1][33];
  int row0, nrows;
  long long b_base;
  if (p.tile_table != nullptr) {
    const int mt = blockIdx.y >> 2, sub = blockIdx.y & 3;
    if (mt >= *p.num_m_tiles_dev) return;
    const int4 e = p.tile_table[mt];
    row0 = e.y + sub * 32;
    nrows = min(32, e.z - sub * 32);
    b_base = static_cast<long long>(e.x) * p.b_rows_per_expert;
  } else {
    row0 = blockIdx.y * 32;
    nrows = min(32, p.M - row0);
    b_base = 0;
  }
  if (nrows <= 0) return;
  const int col0 = blockIdx.x * 32;
  const int tr = threadIdx.x >> 3;
  const int tc = (threadIdx.x & 7) * 4;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float accv[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < p.nseg; ++s) {
    const int K = p.seg_k[s];
    for (int k0 = 0; k0 < K; k0 += 32) {
      for (int i = threadIdx.x; i < 32 * 32; i += 256) {
        const int rr = i >> 5, kk = i & 31;
        const int kg = k0 + kk;
        As[rr][kk] = (rr < nrows && kg < K) ? p.A[s][static_cast<long long>(row0 + rr) * p.lda[s] + kg] : 0.f;
        const int cg = col0 + rr;
        const bool bok = cg < p.N && kg < K;
        const float* Bsrc = PAIRED ? p.B[0] : p.B[s];
        Bs[rr][kk] = bok ? Bsrc[(b_base + cg) * p.ldb[PAIRED ? 0 : s] + kg] : 0.f;
        if (PAIRED) Bv[rr][kk] = bok ? p.B[1][(b_base + cg) * p.ldb[1] + kg] : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < 32; ++kk) {
        const float a = As[tr][kk];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[i] = fmaf(a, Bs[tc + i][kk], acc[i]);
          if (PAIRED) accv[i] = fmaf(a, Bv[tc + i][kk], accv[i]);
        }
      }
      __syncthreads();
    }
  }
  if (tr >= nrows) return;
  float* out = reinterpret_cast<float*>(p.out);
  const long long grow = row0 + tr;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int col = col0 + tc + i;
    if (col >= p.N) break;
    float v = acc[i];
    if (EPI == kEpiSigmoidF32) v = sigmoid_f32(v);
    if (PAIRED) v = situ_glu_f32(acc[i], accv[i], p.situ_c);
    out[grow * p.ldo + col] = v;
  }
}

}  // namespace moe
