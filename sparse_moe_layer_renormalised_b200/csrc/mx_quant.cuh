// MXFP8 / MXFP4 activations and scale-factor tiles for the block-scaled
// expert GEMMs.
//
// Formats (OCP Microscaling Formats v1.0, the format family of the routed
// weights on page "ai-tech-express.jp" on K3, section "量子化を前提とした学習
// 「MXFP4 Quantization-Aware Training」"; the pages give no activation format,
// MXFP8 E4M3 or MXFP4 E2M1 is the library's reading): a row is cut into
// blocks of 32 consecutive elements along K; a block holds one E8M0 scale
// X = 2^s and 32 element codes q with value q * X.  The scale follows the
// spec's rule:
//   s = floor(log2(max_i |v_i|)) - emax     (emax = largest element exponent:
//                                            8 for E4M3, 2 for E2M1)
// clamped to [-127, 127] (an all-zero block gets s = -127), and
//   q_i = element(v_i / X), rounded to nearest even, saturated to the
//         largest finite element (+-448 for E4M3, +-6 for E2M1).
// Inputs are bf16, so v / X is exact in fp32 (or below the smallest element
// step, where it rounds to a signed zero either way) and the one rounding is
// the conversion instruction's.  E4M3 codes take a byte each; E2M1 codes two
// to a byte, the even element in the low nibble.
//
// Scale-factor tiles: the block-scaled MMA reads scales from tensor memory,
// where tcgen05.cp puts them from shared memory in 512-byte atoms of 128 rows
// x 4 k-blocks; byte 16 * (m % 32) + 4 * (m / 32) + j of an atom is the scale
// of row m, k-block j.  The kernels below write scales in that order so that
// one TMA box per stage brings them in:
//   activations  [tile][K/128][2 atoms][512]   (token tiles of <= 256 rows)
//   weights      [E][weight tile][CTA][K/128][512]
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace moe {

constexpr int MXQ_WARPS = 8;

// Byte offset of (tile row i, k-block b) in an activation scale tile.
__device__ __forceinline__ long long mx8_sf_offset(long long tile, int nkb128, int i, int b) {
  return ((tile * nkb128 + (b >> 2)) * 2 + (i >> 7)) * 512 + 16 * (i & 31) + 4 * ((i >> 5) & 3) + (b & 3);
}

// E8M0 exponent s of a block whose largest |bf16| has bit pattern amax_bits
// (sign cleared), for elements whose largest exponent is emax: floor(log2) is
// the bf16 exponent field - 127 (a subnormal or zero maximum gives a value
// below -127, which the clamp absorbs).
__device__ __forceinline__ int mx_block_exponent(uint32_t amax_bits, int emax) {
  if (amax_bits == 0u) return -127;
  const int e = static_cast<int>(amax_bits >> 7) - 127;
  return max(-127, min(127, e - emax));
}

// 2^-s as fp32 for s in [-127, 126] (normal for every such s).
__device__ __forceinline__ float mx_inv_scale(int s) { return __int_as_float((127 - s) << 23); }

// Two fp32 values -> E4M3 codes (round to nearest even, saturated), lo in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two fp32 values -> E2M1 codes (round to nearest even, saturated), lo in the low nibble.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Quantises 32 bf16 values (4 x uint4) with exponent s into 32 E2M1 codes (one uint4).
__device__ __forceinline__ void mx4_encode32(const uint4 (&v)[4], float inv, uint4& out) {
  uint32_t w[4];
  const uint32_t* u = reinterpret_cast<const uint32_t*>(v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // words 4i .. 4i+3 hold elements 8i .. 8i+7, one byte of codes per word
    uint32_t acc = 0u;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint32_t a = u[4 * i + b];
      acc |= e2m1x2(__uint_as_float(a << 16) * inv, __uint_as_float(a & 0xFFFF0000u) * inv) << (8 * b);
    }
    w[i] = acc;
  }
  out = make_uint4(w[0], w[1], w[2], w[3]);
}

// Quantises 32 bf16 values (4 x uint4) with exponent s into 32 E4M3 codes (2 x uint4).
__device__ __forceinline__ void mx8_encode32(const uint4 (&v)[4], float inv, uint4 (&out)[2]) {
  uint32_t w[8];
  const uint32_t* u = reinterpret_cast<const uint32_t*>(v);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    // words 2i, 2i+1 hold elements 4i .. 4i+3
    const uint32_t a = u[2 * i], b = u[2 * i + 1];
    const float f0 = __uint_as_float(a << 16) * inv, f1 = __uint_as_float(a & 0xFFFF0000u) * inv;
    const float f2 = __uint_as_float(b << 16) * inv, f3 = __uint_as_float(b & 0xFFFF0000u) * inv;
    w[i] = e4m3x2(f0, f1) | (e4m3x2(f2, f3) << 16);
  }
  out[0] = make_uint4(w[0], w[1], w[2], w[3]);
  out[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

// Quantises rows to MXFP8 (FP4 = false) or MXFP4 (FP4 = true).  With a tile
// table (tiles != NULL): the rows of the grouped-GEMM token tiles, row r
// (tile rows row0 .. row0 + ntok - 1) reading source row src_row[r] (or r
// when src_row is NULL), scales written into the tile's scale atoms.
// Without one: rows 0 .. n_rows - 1 (src_row ignored), scales row-major
// [n_rows, K/32].  Codes go to codes [r, K] (FP4: [r, K/2]).  One warp per
// row; lane j handles the blocks j, j + 32, ...  Source rows outside
// [0, src_rows) record `site` in the fault flag and are skipped.
template <bool FP4>
__global__ void __launch_bounds__(MXQ_WARPS * 32)
    mx_quant_tiles_kernel(const __nv_bfloat16* __restrict__ src, long long src_rows,
                          const int32_t* __restrict__ src_row, const int4* __restrict__ tiles,
                          const int32_t* __restrict__ num_tiles, long long n_rows, int K,
                          uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, int site) {
  const bool tiled = tiles != nullptr;
  const long long nt = tiled ? num_tiles[0] : (n_rows + 127) / 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nblk = K >> 5, nkb128 = K >> 7;
  for (long long t = blockIdx.x; t < nt; t += gridDim.x) {
    const int4 e = tiled ? tiles[t]
                         : make_int4(0, static_cast<int>(t * 128), static_cast<int>(min(128LL, n_rows - t * 128)), 0);
    for (int i = warp; i < e.z; i += MXQ_WARPS) {
      const long long r = static_cast<long long>(e.y) + i;
      const long long sr = tiled && src_row != nullptr ? static_cast<long long>(src_row[r]) : r;
      if (sr < 0 || sr >= src_rows) {
        record_fault(site);
        continue;
      }
      const uint4* s4 = reinterpret_cast<const uint4*>(src + sr * K);
      uint4* c4 = reinterpret_cast<uint4*>(codes + r * (FP4 ? K / 2 : K));
      for (int b = lane; b < nblk; b += 32) {
        uint4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = __ldg(s4 + 4 * b + j);
        uint32_t amax = 0u;
        const uint32_t* u = reinterpret_cast<const uint32_t*>(v);
#pragma unroll
        for (int j = 0; j < 16; ++j) amax = max(amax, max(u[j] & 0x7FFFu, (u[j] >> 16) & 0x7FFFu));
        const int sexp = mx_block_exponent(amax, FP4 ? 2 : 8);
        if constexpr (FP4) {
          mx4_encode32(v, mx_inv_scale(sexp), c4[b]);
        } else {
          uint4 q[2];
          mx8_encode32(v, mx_inv_scale(sexp), q);
          c4[2 * b] = q[0];
          c4[2 * b + 1] = q[1];
        }
        sf[tiled ? mx8_sf_offset(t, nkb128, i, b) : r * nblk + b] = static_cast<uint8_t>(sexp + 127);
      }
    }
  }
}

// Re-orders row-major E8M0 weight scales [E * rows, K/32] into the weight
// scale tiles read by the block-scaled expert kernel (one 512-byte atom per
// expert, weight tile, CTA of the pair and 128-wide K chunk).
//   paired: a weight tile is 128 intermediate rows; CTA c holds rows
//           wt*128 + c*64 .. +63 of S0 (atom rows 0-63) and of S1 (64-127).
//   else:   a weight tile is 256 rows; CTA c holds rows wt*256 + c*128 .. +127.
__global__ void mx_tile_weight_scales_kernel(const uint8_t* __restrict__ S0, const uint8_t* __restrict__ S1,
                                             int rows_per_expert, int K, int paired, long long total,
                                             uint8_t* __restrict__ out) {
  const int nkb128 = K >> 7, kb32 = K >> 5;
  const int n_wt = paired ? rows_per_expert / 128 : rows_per_expert / 256;
  for (long long o = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; o < total;
       o += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int j = static_cast<int>(o & 511);
    long long blk = o >> 9;
    const int c = static_cast<int>(blk % nkb128);
    blk /= nkb128;
    const int cta = static_cast<int>(blk & 1);
    blk >>= 1;
    const int wt = static_cast<int>(blk % n_wt);
    const long long e = blk / n_wt;
    const int m = (j >> 4) + 32 * ((j >> 2) & 3);  // atom row
    const int kblock = 4 * c + (j & 3);
    const uint8_t* S;
    int row;
    if (paired) {
      S = m < 64 ? S0 : S1;
      row = wt * 128 + cta * 64 + (m & 63);
    } else {
      S = S0;
      row = wt * 256 + cta * 128 + m;
    }
    out[o] = S[(e * rows_per_expert + row) * kb32 + kblock];
  }
}

}  // namespace moe
