// Selection and dispatch kernels: bias + top-k + renormalisation over fp32
// router scores, and the stable expert-major permutation of the T*k
// (token, slot) pairs with the grouped-GEMM tile table.  All integer work is
// deterministic: no order-dependent atomics.
#pragma once

#include <stdint.h>

#include "ptx.cuh"

namespace moe {

// Device fault sites (low range; the GEMMs use 100 + 10 * kernel id + role).
constexpr int kFaultExpertRange = 11;     // topk_idx entry outside [0, E)
constexpr int kFaultDuplicateExpert = 12;  // a token lists the same expert twice
constexpr int kFaultTokenRange = 13;       // perm_token entry outside [0, T)
constexpr int kFaultOffsets = 14;          // expert_offsets not monotone / out of range
constexpr int kFaultRowIndex = 15;         // moe_gather_rows index outside [0, src_rows)

// ------------------------------------------------------------------------------ top-k
// One warp per token.  Lane l holds experts l, l+32, l+64, ... (E <= 1024).
// key_e = fl32(s_e + b_e); k rounds of a warp arg-max under the order
// (key descending, expert index ascending); slot j gets the j-th winner.
// p_j = s_j / sum_j' s_j' with the sum taken in slot order.
constexpr int TOPK_WARPS = 8;

__global__ void __launch_bounds__(TOPK_WARPS * 32)
    topk_renorm_kernel(const float* __restrict__ scores, const float* __restrict__ bias, long long T, int E, int k,
                       int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
  const int lane = threadIdx.x & 31;
  const long long t = static_cast<long long>(blockIdx.x) * TOPK_WARPS + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* srow = scores + t * E;
  float key[32], sc[32];
  uint32_t live = 0u;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int e = lane + 32 * i;
    key[i] = -INFINITY;
    sc[i] = 0.f;
    if (e < E) {
      const float s = srow[e];
      float kk = s + bias[e];
      if (kk != kk) kk = -INFINITY;  // a NaN key never wins over a number
      key[i] = kk;
      sc[i] = s;
      live |= 1u << i;
    }
  }
  float my_s = 0.f, sum = 0.f;
  int my_e = 0;
  for (int j = 0; j < k; ++j) {
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
    // k <= E, so a live entry always exists and be is a valid expert.
    const int owner = be & 31;
    const int slot = be >> 5;
    float s_sel = 0.f;
    if (lane == owner) {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i == slot) s_sel = sc[i];
      live &= ~(1u << slot);
    }
    s_sel = __shfl_sync(0xffffffffu, s_sel, owner);
    sum += s_sel;
    if (lane == j) {
      my_s = s_sel;
      my_e = be;
    }
  }
  if (lane < k) {
    idx_out[t * k + lane] = my_e;
    w_out[t * k + lane] = my_s / sum;
  }
}

// ------------------------------------------------------------------------------ permute
constexpr int PERM_TILE = 128;  // tokens per rank tile

// Block = one tile of 128 tokens (thread = token).  A bitmask bits[e][w] marks
// which tokens of the tile chose expert e; the rank of pair (t, j) among the
// tile's pairs of expert e is the popcount of the tokens before t.  Writes the
// per-tile expert counts and the in-tile ranks.
__global__ void __launch_bounds__(PERM_TILE)
    perm_rank_kernel(const int32_t* __restrict__ idx, long long T, int E, int k, int32_t* __restrict__ tile_counts,
                     int32_t* __restrict__ rank) {
  extern __shared__ uint32_t bits[];  // [E][4]
  const long long tile = blockIdx.x;
  for (int i = threadIdx.x; i < E * 4; i += PERM_TILE) bits[i] = 0u;
  __syncthreads();
  const long long t = tile * PERM_TILE + threadIdx.x;
  const bool tok = t < T;
  const int w = threadIdx.x >> 5;
  const uint32_t bit = 1u << (threadIdx.x & 31);
  if (tok) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[t * k + j];
      if (e < 0 || e >= E) {
        record_fault(kFaultExpertRange);
        continue;
      }
      const uint32_t old = atomicOr(&bits[e * 4 + w], bit);
      if (old & bit) record_fault(kFaultDuplicateExpert);
    }
  }
  __syncthreads();
  if (tok) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[t * k + j];
      int r = 0;
      if (e >= 0 && e < E) {
        for (int ww = 0; ww < w; ++ww) r += __popc(bits[e * 4 + ww]);
        r += __popc(bits[e * 4 + w] & (bit - 1u));
      }
      rank[t * k + j] = r;
    }
  }
  for (int e = threadIdx.x; e < E; e += PERM_TILE) {
    const uint32_t* b = bits + e * 4;
    tile_counts[tile * E + e] = __popc(b[0]) + __popc(b[1]) + __popc(b[2]) + __popc(b[3]);
  }
}

// Inclusive block-wide scan (Hillis-Steele) of one value per thread; 1024 threads.
__device__ __forceinline__ int block_incl_scan_1024(int v, int* buf) {
  buf[threadIdx.x] = v;
  __syncthreads();
  for (int d = 1; d < 1024; d <<= 1) {
    const int add = threadIdx.x >= static_cast<unsigned>(d) ? buf[threadIdx.x - d] : 0;
    __syncthreads();
    buf[threadIdx.x] += add;
    __syncthreads();
  }
  return buf[threadIdx.x];
}

// Number of grouped-GEMM tiles of expert e: ceil(n_e / max_rows).
__device__ __forceinline__ int tiles_of(int cnt, int max_rows) { return (cnt + max_rows - 1) / max_rows; }

// Writes the grouped-GEMM tile table: expert e with n_e rows starting at
// offset o_e contributes ceil(n_e / max_rows) entries {e, row0, rows} of
// near-equal height (at most max_rows).
__device__ __forceinline__ void emit_tiles(int e, int off, int cnt, int first, int max_rows, int4* tile_table) {
  const int nt = tiles_of(cnt, max_rows);
  if (nt == 0) return;
  const int size = (cnt + nt - 1) / nt;
  for (int i = 0; i < nt; ++i) tile_table[first + i] = make_int4(e, off + size * i, min(size, cnt - size * i), 0);
}

// One block of 1024 threads, thread = expert.  Turns the per-tile counts into
// per-tile exclusive bases (in place), the expert counts, the CSR offsets, the
// tile table, its length (num_m_tiles[0]) and the number of its leading tiles
// that belong to experts with more than one tile (num_m_tiles[1]);
// tile_table / num_m_tiles may be NULL when the caller runs no grouped GEMM
// on the result.
__global__ void __launch_bounds__(1024)
    perm_scan_kernel(int32_t* __restrict__ tile_counts, int ntiles, int E, int32_t* __restrict__ counts_out,
                     int32_t* __restrict__ offsets, int max_tile_rows, int4* __restrict__ tile_table,
                     int32_t* __restrict__ num_m_tiles) {
  __shared__ int buf[1024];
  const int e = threadIdx.x;
  int run = 0;
  if (e < E) {
    for (int tl = 0; tl < ntiles; ++tl) {
      int32_t* p = tile_counts + static_cast<long long>(tl) * E + e;
      const int c = *p;
      *p = run;
      run += c;
    }
  }
  const int cnt = e < E ? run : 0;
  const int mt = tiles_of(cnt, max_tile_rows);
  // Tiles of experts with several tiles (their weight tiles are re-read from
  // L2 by each) come first, then the tiles of single-tile experts (weights
  // streamed once); each part in expert order.
  const int mt_multi = mt >= 2 ? mt : 0, mt_single = mt == 1 ? 1 : 0;
  const int incl_off = block_incl_scan_1024(cnt, buf);
  __syncthreads();
  const int incl_multi = block_incl_scan_1024(mt_multi, buf);
  const int n_multi = buf[1023];
  __syncthreads();
  const int incl_single = block_incl_scan_1024(mt_single, buf);
  if (e < E) {
    offsets[e] = incl_off - cnt;
    if (counts_out != nullptr) counts_out[e] = cnt;
    const int first = mt >= 2 ? incl_multi - mt_multi : n_multi + incl_single - mt_single;
    if (tile_table != nullptr) emit_tiles(e, incl_off - cnt, cnt, first, max_tile_rows, tile_table);
  }
  if (e == E - 1) {
    offsets[E] = incl_off;
    if (num_m_tiles != nullptr) {
      num_m_tiles[0] = n_multi + incl_single;
      num_m_tiles[1] = n_multi;
    }
  }
}

// Tile table from caller-supplied CSR offsets (moe_expert_ffn).  Offsets that
// are not monotone or exceed max_rows are recorded as a fault and the expert
// is given no rows, so no tile addresses memory outside [0, max_rows).
__global__ void __launch_bounds__(1024)
    tile_table_kernel(const int32_t* __restrict__ offsets, int E, long long max_rows, int max_tile_rows,
                      int4* __restrict__ tile_table, int32_t* __restrict__ num_m_tiles) {
  __shared__ int buf[1024];
  const int e = threadIdx.x;
  int off = 0, cnt = 0;
  if (e < E) {
    off = offsets[e];
    const int end = offsets[e + 1];
    if (off < 0 || end < off || end > max_rows) {
      record_fault(kFaultOffsets);
      off = 0;
    } else {
      cnt = end - off;
    }
  }
  const int mt = tiles_of(cnt, max_tile_rows);
  const int incl_mt = block_incl_scan_1024(mt, buf);
  if (e < E) emit_tiles(e, off, cnt, incl_mt - mt, max_tile_rows, tile_table);
  if (e == E - 1) {
    num_m_tiles[0] = incl_mt;
    num_m_tiles[1] = 0;  // one list, in expert order
  }
}

// Tile table over n_blocks CSR blocks of the same E experts (rows received
// from several ranks, each block expert-major): block b's rows of expert e are
// offsets[b*(E+1)+e] .. offsets[b*(E+1)+e+1]-1.  Tiles are emitted expert by
// expert (all blocks of expert 0, then expert 1, ...), so the tiles of one
// expert stay adjacent in the grouped GEMM's work order.  Bad offsets are
// recorded as a fault and that segment gets no rows.
__global__ void __launch_bounds__(1024)
    tile_table_blocks_kernel(const int32_t* __restrict__ offsets, int n_blocks, int E, long long max_rows,
                             int max_tile_rows, int4* __restrict__ tile_table, int32_t* __restrict__ num_m_tiles) {
  __shared__ int buf[1024];
  const int e = threadIdx.x;
  int mt = 0;
  if (e < E) {
    for (int b = 0; b < n_blocks; ++b) {
      const int32_t* o = offsets + static_cast<long long>(b) * (E + 1);
      const int off = o[e], end = o[e + 1];
      if (off < 0 || end < off || end > max_rows)
        record_fault(kFaultOffsets);
      else
        mt += tiles_of(end - off, max_tile_rows);
    }
  }
  const int incl_mt = block_incl_scan_1024(mt, buf);
  if (e < E) {
    int first = incl_mt - mt;
    for (int b = 0; b < n_blocks; ++b) {
      const int32_t* o = offsets + static_cast<long long>(b) * (E + 1);
      const int off = o[e], end = o[e + 1];
      if (off < 0 || end < off || end > max_rows) continue;
      emit_tiles(e, off, end - off, first, max_tile_rows, tile_table);
      first += tiles_of(end - off, max_tile_rows);
    }
  }
  if (e == E - 1) {
    num_m_tiles[0] = incl_mt;
    num_m_tiles[1] = 0;  // one list, in expert order
  }
}

// Tile table of a dense problem run on the grouped expert kernels: rows
// 0 .. T-1 as consecutive tiles of tile_rows rows of "expert" 0.
// num_m_tiles[0] = number of tiles; num_m_tiles[1] = the same (one expert with
// several tiles: its weight tiles are re-read through L2).
__global__ void dense_tile_table_kernel(long long T, int tile_rows, int4* __restrict__ tile_table,
                                        int32_t* __restrict__ num_m_tiles) {
  const long long ntiles = (T + tile_rows - 1) / tile_rows;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < ntiles;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r0 = i * tile_rows;
    tile_table[i] = make_int4(0, static_cast<int>(r0), static_cast<int>(min(static_cast<long long>(tile_rows), T - r0)), 0);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    num_m_tiles[0] = static_cast<int32_t>(ntiles);
    num_m_tiles[1] = static_cast<int32_t>(ntiles);
  }
}

// Thread = pair (t, j): position = offset of its expert + base of its tile +
// rank in the tile.  Token-ascending within each expert by construction.
__global__ void __launch_bounds__(256)
    perm_scatter_kernel(const int32_t* __restrict__ idx, long long T, int E, int k,
                        const int32_t* __restrict__ tile_base, const int32_t* __restrict__ rank,
                        const int32_t* __restrict__ offsets, int32_t* __restrict__ perm_token,
                        int32_t* __restrict__ inv_perm) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= T * k) return;
  const long long t = i / k;
  const int e = idx[i];
  if (e < 0 || e >= E) {
    inv_perm[i] = 0;
    return;
  }
  const int pos = offsets[e] + tile_base[(t / PERM_TILE) * E + e] + rank[i];
  perm_token[pos] = static_cast<int32_t>(t);
  inv_perm[i] = pos;
}

// Warp = one destination row: dst[row] = src[perm_token[row]] for
// row < *n_rows, moved in 16-byte vectors.  row_vecs = row bytes / 16.
constexpr int GATHER_WARPS = 8;

__global__ void __launch_bounds__(GATHER_WARPS * 32)
    gather_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, const int32_t* __restrict__ perm_token,
                       const int32_t* __restrict__ n_rows, long long T, int row_vecs) {
  const long long row = static_cast<long long>(blockIdx.x) * GATHER_WARPS + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= *n_rows) return;
  const int t = perm_token[row];
  uint4* d = dst + row * row_vecs;
  if (t < 0 || t >= T) {
    if (lane == 0) record_fault(kFaultTokenRange);
    for (int i = lane; i < row_vecs; i += 32) d[i] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const uint4* s = src + static_cast<long long>(t) * row_vecs;
  // four 16-byte loads in flight per lane before their stores
  int i = lane;
  for (; i + 96 < row_vecs; i += 128) {
    const uint4 a = s[i], b = s[i + 32], c = s[i + 64], e = s[i + 96];
    d[i] = a;
    d[i + 32] = b;
    d[i + 64] = c;
    d[i + 96] = e;
  }
  for (; i < row_vecs; i += 32) d[i] = s[i];
}

// dst[r] = src[idx[r]] for r < n, rows of row_vecs 16-byte words (the
// expert-parallel exchange's reordering of token rows by destination and back).
// One warp per row; an index outside [0, src_rows) records kFaultRowIndex and
// zero-fills the row.
__global__ void __launch_bounds__(GATHER_WARPS * 32)
    gather_rows_idx_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, const int32_t* __restrict__ idx,
                           long long n, long long src_rows, int row_vecs) {
  const long long row = static_cast<long long>(blockIdx.x) * GATHER_WARPS + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n) return;
  const long long t = idx[row];
  uint4* d = dst + row * row_vecs;
  if (t < 0 || t >= src_rows) {
    if (lane == 0) record_fault(kFaultRowIndex);
    for (int i = lane; i < row_vecs; i += 32) d[i] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const uint4* s = src + t * row_vecs;
  int i = lane;
  for (; i + 96 < row_vecs; i += 128) {
    const uint4 a = s[i], b = s[i + 32], c = s[i + 64], e = s[i + 96];
    d[i] = a;
    d[i + 32] = b;
    d[i + 64] = c;
    d[i + 96] = e;
  }
  for (; i < row_vecs; i += 32) d[i] = s[i];
}

}  // namespace moe
