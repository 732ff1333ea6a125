// Quantile Balancing bias update (the training-time step beside the router).
//
// Source: "Kimi K3の896エキスパート…" (lilting.ch), section
// 「ルーター専用の独立訓練はない」 — each expert's bias is updated from the
// boundary, read off quantiles of the router scores, at which it receives its
// target number of tokens; the Kimi K3 tech-report summary, section
// 「幅のスケーリング：Stable LatentMoE」 — the quantiles come from a histogram of
// the router's score margins.
//
// Margin of expert e for token t: m = key_e - theta, key = fl32(s + b), theta
// = the k-th largest key among the other experts (the token's (k+1)-th key if
// e is in its top k, else its k-th); ties rank the lower index first.  The
// update is b_e <- b_e - q_e with q_e the rank-c boundary of e's margins, c =
// floor(T k / E), read from an nb-bin histogram on [lo, hi) with the margins
// spread evenly inside a bin.
//
//   qb_hist_kernel      one warp per token: keys, top-(k+1) by warp arg-max
//                       rounds, margins, fp32 bin index, global atomic count.
//                       HBM-bound: T*E*4 bytes of scores read.
//   qb_quantile_kernel  one warp per expert: scan its nb counts from the top
//                       bin, locate rank c, interpolate, write q_e and b_e - q_e.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int QB_WARPS = 8;

__global__ void qb_zero_kernel(uint32_t* __restrict__ p, long long n) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    p[i] = 0u;
}

__global__ void __launch_bounds__(QB_WARPS * 32)
    qb_hist_kernel(const float* __restrict__ scores, const float* __restrict__ bias, long long T, int E, int k,
                   int nb, float lo, float inv_w, uint32_t* __restrict__ hist) {
  const int lane = threadIdx.x & 31;
  const long long t = static_cast<long long>(blockIdx.x) * QB_WARPS + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* srow = scores + t * E;
  float key[32];
  uint32_t live = 0u;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int e = lane + 32 * i;
    key[i] = -INFINITY;
    if (e < E) {
      float kk = __fadd_rn(srow[e], bias[e]);
      if (kk != kk) kk = -INFINITY;  // a NaN key ranks below every number
      key[i] = kk;
      live |= 1u << i;
    }
  }
  // k + 1 rounds of (key desc, index asc) arg-max; the first k winners are the
  // token's selection, the k-th and (k+1)-th keys the two possible thresholds.
  uint32_t sel = 0u;
  float kth = -INFINITY, k1th = -INFINITY;
  for (int j = 0; j <= k; ++j) {
    float bk = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if ((live >> i) & 1u) {
        const int e = lane + 32 * i;
        if (key[i] > bk || (key[i] == bk && e < be)) {
          bk = key[i];
          be = e;
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (ok > bk || (ok == bk && oe < be)) {
        bk = ok;
        be = oe;
      }
    }
    // k < E, so a live entry always exists and be is a valid expert.
    if (lane == (be & 31)) {
      live &= ~(1u << (be >> 5));
      if (j < k) sel |= 1u << (be >> 5);
    }
    if (j == k - 1) kth = bk;
    if (j == k) k1th = bk;
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      const float theta = ((sel >> i) & 1u) ? k1th : kth;
      const float m = __fsub_rn(key[i], theta);
      float u = __fmul_rn(__fsub_rn(m, lo), inv_w);
      if (u != u) u = 0.f;
      u = fminf(fmaxf(u, -1.0f), static_cast<float>(nb));
      const int bin = min(max(static_cast<int>(floorf(u)), 0), nb - 1);
      atomicAdd(&hist[static_cast<long long>(e) * nb + bin], 1u);
    }
  }
}

// One warp per expert; nb is a multiple of 32.
__global__ void __launch_bounds__(32)
    qb_quantile_kernel(const uint32_t* __restrict__ hist, int E, int nb, long long c, float lo, float w,
                       const float* __restrict__ bias_in, float* __restrict__ bias_out, float* __restrict__ q_out) {
  const int e = blockIdx.x;
  const int lane = threadIdx.x;
  if (e >= E) return;
  const uint32_t* h = hist + static_cast<long long>(e) * nb;
  long long above = 0;  // margins in the bins already passed (above the current chunk)
  float q = lo;         // every margin below the range: the boundary is the range's bottom
  for (int base = nb - 32; base >= 0; base -= 32) {
    const int j = base + 31 - lane;  // lane 0 holds the chunk's top bin
    const long long n = h[j];
    long long incl = n;  // inclusive prefix over lanes = margins in this chunk's bins >= j
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    const long long before = above + incl - n;  // margins above bin j
    const uint32_t hit = __ballot_sync(0xffffffffu, before < c && before + n >= c);
    if (hit) {
      const int src = __ffs(hit) - 1;
      const float qj = __fmaf_rn(w, static_cast<float>(j + 1) - static_cast<float>(c - before) / static_cast<float>(n), lo);
      q = __shfl_sync(0xffffffffu, qj, src);
      break;
    }
    above += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) {
    bias_out[e] = __fsub_rn(bias_in[e], q);
    if (q_out) q_out[e] = q;
  }
}

}  // namespace moe
