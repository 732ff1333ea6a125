// Persistent tcgen05 GEMM for sm_100a:  out[r, n] = epilogue( sum_k A[r, k] * B[n, k] ).
//
// A and B are bf16, K-major, loaded by TMA with the 128-byte swizzle into a
// TC_STAGES-deep shared-memory ring; one thread issues tcgen05.mma (M=128,
// N=256, K=16 per instruction) into one of two TMEM accumulators of 256 fp32
// columns, so the epilogue of tile i overlaps the main loop of tile i+1.
//
// Warp roles (192 threads, one CTA per SM):
//   warp 0       TMA producer (one elected lane)
//   warp 1       TMEM owner and MMA issuer (one elected lane)
//   warps 2..5   epilogue: TMEM -> registers -> epilogue -> global
//
// Work items are (m-tile, n-tile) pairs, m-tile-major, strided over the grid.
//   dense   : m-tile i covers rows [128 i, 128 i + 128) of A and of out.
//   grouped : m-tile i is entry i of a device-side table {expert, row0, nrows}
//             built from the expert offsets; B rows are offset by
//             expert * b_rows_per_expert (B is the [E * R, K] view of the
//             per-expert weights).  The host never reads the table.
// K may be split into up to TC_MAX_SEG segments with their own A and B tensor
// maps (the output projection concatenates [h_shared | n] along K against
// [W_so | W_up]).
// PAIRED mode: the 256 accumulator columns are 128 columns of B map 0 (gate
// projection rows) followed by the same 128 rows of B map 1 (up projection);
// the epilogue forms SiTU-GLU(g, v) for 128 intermediate columns.
#pragma once

#include "activations.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int TC_BM = 128;
constexpr int TC_BN = 256;
constexpr int TC_BK = 64;
constexpr int TC_STAGES = 4;
constexpr int TC_THREADS = 192;
constexpr uint32_t TC_A_BYTES = TC_BM * TC_BK * 2;
constexpr uint32_t TC_B_BYTES = TC_BN * TC_BK * 2;
constexpr uint32_t TC_B_HALF_BYTES = TC_B_BYTES / 2;
constexpr uint32_t TC_STAGE_BYTES = TC_A_BYTES + TC_B_BYTES;
constexpr uint32_t TC_TMEM_COLS = 2 * TC_BN;
constexpr size_t TC_SMEM_BYTES = 1024 + static_cast<size_t>(TC_STAGES) * TC_STAGE_BYTES + 256;
constexpr int TC_MAX_SEG = 4;

enum TcEpilogue : int { kEpiF32 = 0, kEpiBF16 = 1, kEpiSigmoidF32 = 2, kEpiSituBF16 = 3 };

struct TcMaps {
  CUtensorMap a[TC_MAX_SEG];
  CUtensorMap b[TC_MAX_SEG];
};

struct TcParams {
  int M;                       // dense: rows of A and out
  int num_m_tiles;             // dense: ceil(M / 128)
  const int4* tile_table;      // grouped: {expert, row0, nrows, 0}; nullptr when dense
  const int* num_m_tiles_dev;  // grouped: number of valid table entries
  int n_tiles;
  int N;             // valid output columns (PAIRED: intermediate columns)
  int num_k_blocks;  // total K / 64 over all segments
  int seg_end[TC_MAX_SEG];  // cumulative k-block end of each segment (unused ones = num_k_blocks)
  int b_rows_per_expert;
  void* out;
  long long ldo;  // elements between output rows
  float situ_c;
  int fault_site;  // base code recorded on a wait timeout
};

struct TcTile {
  int row0, nrows, b_row, col0;
};

template <bool PAIRED>
__device__ __forceinline__ TcTile tc_decode(int w, const TcParams& p) {
  const int mt = w / p.n_tiles;
  const int nt = w - mt * p.n_tiles;
  TcTile t;
  if (p.tile_table != nullptr) {
    const int4 e = p.tile_table[mt];
    t.row0 = e.y;
    t.nrows = e.z;
    t.b_row = e.x * p.b_rows_per_expert;
  } else {
    t.row0 = mt * TC_BM;
    t.nrows = min(TC_BM, p.M - t.row0);
    t.b_row = 0;
  }
  constexpr int kCols = PAIRED ? TC_BN / 2 : TC_BN;
  t.col0 = nt * kCols;
  t.b_row += nt * kCols;
  return t;
}

// 32 consecutive bf16 (four 16-byte vectors) at dst, of which the first
// `valid` are inside the row.
__device__ __forceinline__ void store_bf16_chunk(__nv_bfloat16* dst, uint4 q0, uint4 q1, uint4 q2, uint4 q3,
                                                 int valid) {
  if (valid >= 32) {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    d4[0] = q0;
    d4[1] = q1;
    d4[2] = q2;
    d4[3] = q3;
  } else {
    const uint32_t w[16] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w,
                            q2.x, q2.y, q2.z, q2.w, q3.x, q3.y, q3.z, q3.w};
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < valid) dst[i] = bf16_half(w[i >> 1], i & 1);
  }
}

template <int EPI, bool PAIRED>
__global__ void __launch_bounds__(TC_THREADS, 1) tc_gemm_kernel(const __grid_constant__ TcMaps maps, const TcParams p) {
  extern __shared__ uint8_t tc_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + TC_STAGES * TC_A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + TC_STAGES * TC_B_BYTES);
  uint64_t* empty = full + TC_STAGES;
  uint64_t* acc_full = empty + TC_STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < TC_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < TC_MAX_SEG; ++s) {
      if (s == 0 || p.seg_end[s - 1] < p.num_k_blocks) {
        tma_prefetch_desc(&maps.a[s]);
        tma_prefetch_desc(&maps.b[s]);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, TC_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int num_m_tiles = p.tile_table != nullptr ? *p.num_m_tiles_dev : p.num_m_tiles;
  const int total = num_m_tiles * p.n_tiles;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0u, issued_parity = 0u;  // per stage: ever loaded / parity of its last load
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        const TcTile t = tc_decode<PAIRED>(w, p);
        int seg = 0;
        int seg_start = 0;
        for (int kb = 0; kb < p.num_k_blocks; ++kb) {
          while (kb >= p.seg_end[seg]) {
            seg_start = p.seg_end[seg];
            ++seg;
          }
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort, p.fault_site + 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], TC_STAGE_BYTES);
          const int kc = (kb - seg_start) * TC_BK;
          uint8_t* a_dst = sA + stage * TC_A_BYTES;
          uint8_t* b_dst = sB + stage * TC_B_BYTES;
          tma_load_2d(a_dst, &maps.a[seg], &full[stage], kc, t.row0);
          if (PAIRED) {
            tma_load_2d(b_dst, &maps.b[0], &full[stage], kc, t.b_row);
            tma_load_2d(b_dst + TC_B_HALF_BYTES, &maps.b[1], &full[stage], kc, t.b_row);
          } else {
            tma_load_2d(b_dst, &maps.b[seg], &full[stage], kc, t.b_row);
            tma_load_2d(b_dst + TC_B_HALF_BYTES, &maps.b[seg], &full[stage], kc, t.b_row + TC_BN / 2);
          }
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == TC_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Every load this thread issued must have landed before the CTA exits.
      volatile int never = 0;
      for (int s = 0; s < TC_STAGES; ++s)
        if ((issued >> s) & 1u) mbar_wait(&full[s], (issued_parity >> s) & 1u, &never, p.fault_site + 2);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(TC_BM, TC_BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort, p.fault_site + 3)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * TC_BN);
        for (int kb = 0; kb < p.num_k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort, p.fault_site + 4)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * TC_A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * TC_B_BYTES);
#pragma unroll
          for (int kk = 0; kk < TC_BK / 16; ++kk) {
            tc_mma_bf16(d_tmem, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32), idesc,
                        (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == TC_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&acc_full[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // All MMAs issued by this thread complete before TMEM is released.
      tc_commit(drain);
      volatile int never = 0;
      mbar_wait(drain, 0u, &never, p.fault_site + 5);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      const TcTile t = tc_decode<PAIRED>(w, p);
      // warp-uniform decision: tcgen05.ld below needs the whole warp
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[acc], acc_phase, abort, p.fault_site + 6))) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * TC_BN);
      const bool row_ok = r < t.nrows;
      const bool warp_has_rows = q * 32 < t.nrows;  // warp-uniform
      const long long grow = static_cast<long long>(t.row0) + r;
      if (warp_has_rows) {
        if constexpr (PAIRED) {
          __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
          const float c = p.situ_c;
          const float inv_c = 1.0f / c;
#pragma unroll 1
          for (int ch = 0; ch < TC_BN / 64; ++ch) {
            const int col = t.col0 + ch * 32;
            if (col >= p.N) break;  // warp-uniform
            float g[32], v[32];
            tmem_ld32(tbase + ch * 32, g);
            tmem_ld32(tbase + TC_BN / 2 + ch * 32, v);
            if (row_ok) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(situ_glu_fast(g[2 * i], v[2 * i], c, inv_c),
                                    situ_glu_fast(g[2 * i + 1], v[2 * i + 1], c, inv_c));
              __nv_bfloat16* dst = out + grow * p.ldo + col;
              if (col + 32 <= p.N) {
                uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
                for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (col + i < p.N) dst[i] = bf16_half(pk[i >> 1], i & 1);
              }
            }
          }
        } else {
#pragma unroll 1
          for (int ch = 0; ch < TC_BN / 32; ++ch) {
            const int col = t.col0 + ch * 32;
            if (col >= p.N) break;  // warp-uniform
            float a[32];
            tmem_ld32(tbase + ch * 32, a);
            if (row_ok) {
              if (EPI == kEpiSigmoidF32) {
#pragma unroll
                for (int i = 0; i < 32; ++i) a[i] = sigmoid_f32(a[i]);
              }
              if (EPI == kEpiBF16) {
                uint4 q[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  q[i] = make_uint4(pack_bf16x2(a[8 * i], a[8 * i + 1]), pack_bf16x2(a[8 * i + 2], a[8 * i + 3]),
                                    pack_bf16x2(a[8 * i + 4], a[8 * i + 5]), pack_bf16x2(a[8 * i + 6], a[8 * i + 7]));
                store_bf16_chunk(reinterpret_cast<__nv_bfloat16*>(p.out) + grow * p.ldo + col, q[0], q[1], q[2], q[3],
                                 min(32, p.N - col));
              } else {
                float* dst = reinterpret_cast<float*>(p.out) + grow * p.ldo + col;
                if (col + 32 <= p.N) {
                  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
                  for (int i = 0; i < 8; ++i) d4[i] = make_float4(a[4 * i], a[4 * i + 1], a[4 * i + 2], a[4 * i + 3]);
                } else {
#pragma unroll
                  for (int i = 0; i < 32; ++i)
                    if (col + i < p.N) dst[i] = a[i];
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, TC_TMEM_COLS);
  }
}

}  // namespace moe
