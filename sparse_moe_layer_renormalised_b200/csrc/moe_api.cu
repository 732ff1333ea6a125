// C-ABI entry points of the Stable LatentMoE layer library (see include/moe.h):
// host-side validation, workspace layout, TMA descriptor encoding and the
// launch sequence.  Every step of the layer runs in the kernels included here.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <functional>
#include <mutex>

#include "backward.cuh"
#include "combine.cuh"
#include "gemm_expert.cuh"
#include "gemm_expert2.cuh"
#include "gemm_expert_bs.cuh"
#include "mx_quant.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"
#include "ptx.cuh"
#include "routing.cuh"
#include "qb.cuh"
#include "../../include/moe.h"

namespace moe {
namespace {

thread_local int g_last_launches = 0;

constexpr size_t kAlign = 256;

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

// ------------------------------------------------------------------------------ validation
bool dims_ok(const moe_dims* d) {
  if (d == nullptr) return false;
  if (d->T < 0 || d->H <= 0 || d->L <= 0 || d->E <= 0 || d->k <= 0 || d->I <= 0 || d->S < 0) return false;
  if (d->S > 0 && d->Is <= 0) return false;
  if (d->k > d->E || d->k > 32 || d->E > 1024) return false;
  if (!(d->situ_c > 0.f) || !std::isfinite(d->situ_c) || !(d->rms_eps >= 0.f) || !std::isfinite(d->rms_eps))
    return false;
  if (d->act != MOE_F32 && d->act != MOE_BF16) return false;
  if (d->routed != MOE_F32 && d->routed != MOE_BF16 && d->routed != MOE_MXFP4 && d->routed != MOE_MXFP4_A8 &&
      d->routed != MOE_MXFP4_A4)
    return false;
  if (d->y_out != MOE_F32 && d->y_out != d->act) return false;
  if (d->L % 8 != 0 || d->H % 8 != 0 || d->I % 8 != 0) return false;
  if (d->S > 0 && d->Is % 8 != 0) return false;
  if (d->T * static_cast<long long>(d->k) > 0x7fffffffLL) return false;
  return true;
}

// Valid dims that this build does not implement.
bool dims_supported(const moe_dims* d) {
  if (d->routed == MOE_MXFP4 || d->routed == MOE_MXFP4_A8 || d->routed == MOE_MXFP4_A4) {
    // MXFP4 routed weights: bf16 activations; code and scale rows must suit TMA
    // (K/2 and K/32 bytes per row, multiples of 16) for both expert GEMMs.
    // (The block-scaled path also needs K % 128 and 2-CTA weight tiles, which
    // these multiples give.)
    if (d->act != MOE_BF16 || d->L % 512 != 0 || d->I % 512 != 0) return false;
  } else if (d->routed != d->act) {
    return false;
  }
  if (d->L > 4 * COMBINE_THREADS * 16) return false;
  if (d->act == MOE_BF16) {
    if (d->H % 64 || d->L % 64 || d->I % 64) return false;
    if (d->S > 0 && d->Is % 64) return false;
    if (d->S > TC_MAX_SEG - 1) return false;
  } else {
    if (d->S > SIMT_MAX_SEG - 1) return false;
  }
  return true;
}

moe_status check_dims(const moe_dims* d) {
  if (!dims_ok(d)) return MOE_ERR_INVALID_ARG;
  if (!dims_supported(d)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

inline size_t act_bytes(const moe_dims& d) { return d.act == MOE_F32 ? 4 : 2; }

// Expert kernel pairing: 2-CTA pairs when the weight tiles divide evenly.
int expert_cg(const moe_dims& d) { return (d.I % 128 == 0 && d.L % 256 == 0) ? 2 : 1; }

// Largest token tile of the grouped expert GEMMs (MMA N = 256 on pairs; a
// single CTA stages at most 128 token rows; the fp32 path uses 128-row tiles;
// the block-scaled paths 208, which leaves tensor memory for their scales).
int expert_tile_rows(const moe_dims& d) {
  if (d.routed == MOE_MXFP4_A8 || d.routed == MOE_MXFP4_A4) return BS_MAX_TILE_ROWS;
  return d.act == MOE_BF16 ? 128 * expert_cg(d) : 128;
}

// Block-scaled routed experts (MXFP8 or MXFP4 inputs); a4: the MXFP4 one.
inline bool routed_bs(const moe_dims& d) { return d.routed == MOE_MXFP4_A8 || d.routed == MOE_MXFP4_A4; }
inline bool routed_a4(const moe_dims& d) { return d.routed == MOE_MXFP4_A4; }
// Bytes of one row of K activation codes in the block-scaled input format.
inline size_t bs_code_bytes(const moe_dims& d, size_t K) { return routed_a4(d) ? K / 2 : K; }


// ------------------------------------------------------------------------------ workspace
struct WsLayout {
  size_t scores, topk_idx, topk_w, rank, tile_base, counts, offsets, tile_table, num_m_tiles, perm_token,
      inv_perm, z, z_perm, h_perm, y_perm, n, h_s, dense_tiles, dense_num, h_q, sf_z, sf_h, total;
};

WsLayout ws_layout(const moe_dims& d) {
  WsLayout w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += round_up(bytes, kAlign);
    return o;
  };
  const size_t T = static_cast<size_t>(d.T), R = T * d.k, es = act_bytes(d);
  const size_t ntok_tiles = cdiv(static_cast<long long>(T), PERM_TILE);
  const size_t max_m_tiles = cdiv(static_cast<long long>(R), TC_BM) + d.E;
  w.scores = take(T * d.E * 4);
  w.topk_idx = take(R * 4);
  w.topk_w = take(R * 4);
  w.rank = take(R * 4);
  w.tile_base = take(ntok_tiles * d.E * 4);
  w.counts = take(static_cast<size_t>(d.E) * 4);
  w.offsets = take(static_cast<size_t>(d.E + 1) * 4);
  w.tile_table = take(max_m_tiles * 16);
  w.num_m_tiles = take(16);
  w.perm_token = take(R * 4);
  w.inv_perm = take(R * 4);
  w.z = take(T * d.L * es);
  w.z_perm = take(R * d.L * es);
  w.h_perm = take(R * d.I * es);
  w.y_perm = take(R * d.L * 4);
  w.n = take(T * d.L * es);
  w.h_s = take(T * static_cast<size_t>(d.S) * d.Is * es);
  w.dense_tiles = take(static_cast<size_t>(cdiv(static_cast<long long>(T), 128) + 1) * 16);
  w.dense_num = take(16);
  // block-scaled paths: the codes of h and the activation scale tiles (the
  // codes of the expert-major z rows reuse z_perm)
  const bool bs = routed_bs(d);
  w.h_q = take(bs ? R * bs_code_bytes(d, d.I) : 0);
  w.sf_z = take(bs ? max_m_tiles * (d.L / 128) * 1024 : 0);
  w.sf_h = take(bs ? max_m_tiles * (d.I / 128) * 1024 : 0);
  w.total = off;
  return w;
}

template <typename P>
inline P* at(void* base, size_t off) {
  return reinterpret_cast<P*>(static_cast<uint8_t*>(base) + off);
}

// ------------------------------------------------------------------------------ TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// bf16 matrix [rows, cols] with `ld` elements between rows, box `box_rows`
// rows x 64 columns, 128-byte swizzle, out-of-bounds elements read as zero.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
              uint32_t box_rows = TC_BM) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr || rows == 0 || cols == 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(TC_BK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// uint8 matrix [rows, cols] (cols in bytes), box box_rows x box_cols bytes, no
// swizzle (MXFP4 codes and scales).
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                 uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr || rows == 0 || cols == 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed E2M1 codes [rows, K] (K elements, K/2 bytes a row), boxes of 128
// elements x box_rows rows landing as 16-byte slots of 16 codes and 8 bytes of
// gap (the shared-memory layout tcgen05.mma kind::mxf8f6f4 reads for 4-bit
// operands), 128-byte swizzle.  The driver requires a 32-byte aligned base,
// K % 128 == 0 and a row pitch that is a multiple of 32 bytes.
bool make_map_e2m1(CUtensorMap* m, const void* base, uint64_t rows, uint64_t K, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr || rows == 0 || K == 0) return false;
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {K / 2};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// uint8 matrix [rows, cols] with boxes 128 bytes wide x box_rows rows and
// 128-byte swizzle (E4M3 activation codes as an MMA operand).
bool make_map_u8_sw128(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr || rows == 0 || cols == 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// ------------------------------------------------------------------------------ GEMM launch helpers
struct Seg {
  const void* a;  // A segment base (bf16 / f32)
  long long a_ld;
  const void* b;  // B segment base
  long long b_ld;
  long long b_rows;  // rows of the B view
  int K;
};

struct GemmDesc {
  int epi;
  bool paired;
  long long M;  // dense rows, or rows of the permuted buffer when grouped
  const int4* tile_table;
  const int* num_m_tiles_dev;
  int max_m_tiles;  // grouped: upper bound of the table length
  int N;
  int b_rows_per_expert;
  int nseg;
  Seg seg[TC_MAX_SEG];
  const void* b_up;  // PAIRED: B rows of the up projection (same view as seg[0].b)
  void* out;
  long long ldo;
  float situ_c;
  int fault_site;
};

template <int EPI, bool PAIRED>
cudaError_t launch_tc_inst(const TcMaps& maps, const TcParams& p, int grid, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel<EPI, PAIRED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(TC_SMEM_BYTES));
  if (e != cudaSuccess) return e;
  tc_gemm_kernel<EPI, PAIRED><<<grid, TC_THREADS, TC_SMEM_BYTES, s>>>(maps, p);
  return cudaGetLastError();
}

moe_status run_gemm_tc(const GemmDesc& g, cudaStream_t s) {
  TcMaps maps;
  std::memset(&maps, 0, sizeof maps);
  TcParams p;
  std::memset(&p, 0, sizeof p);
  int kb = 0;
  for (int i = 0; i < g.nseg; ++i) {
    const Seg& sg = g.seg[i];
    if (!make_map(&maps.a[i], sg.a, static_cast<uint64_t>(g.M), static_cast<uint64_t>(sg.K),
                  static_cast<uint64_t>(sg.a_ld)))
      return MOE_ERR_CUDA;
    if (!make_map(&maps.b[i], sg.b, static_cast<uint64_t>(sg.b_rows), static_cast<uint64_t>(sg.K),
                  static_cast<uint64_t>(sg.b_ld)))
      return MOE_ERR_CUDA;
    kb += static_cast<int>(cdiv(sg.K, TC_BK));
    p.seg_end[i] = kb;
  }
  if (g.paired) {
    if (!make_map(&maps.b[1], g.b_up, static_cast<uint64_t>(g.seg[0].b_rows), static_cast<uint64_t>(g.seg[0].K),
                  static_cast<uint64_t>(g.seg[0].b_ld)))
      return MOE_ERR_CUDA;
  }
  for (int i = g.nseg; i < TC_MAX_SEG; ++i) p.seg_end[i] = kb;
  p.num_k_blocks = kb;
  p.M = static_cast<int>(g.M);
  p.num_m_tiles = static_cast<int>(cdiv(g.M, TC_BM));
  p.tile_table = g.tile_table;
  p.num_m_tiles_dev = g.num_m_tiles_dev;
  p.N = g.N;
  p.n_tiles = static_cast<int>(cdiv(g.N, g.paired ? TC_BN / 2 : TC_BN));
  p.b_rows_per_expert = g.b_rows_per_expert;
  p.out = g.out;
  p.ldo = g.ldo;
  p.situ_c = g.situ_c;
  p.fault_site = g.fault_site;
  const long long m_tiles = g.tile_table ? g.max_m_tiles : p.num_m_tiles;
  long long work = m_tiles * p.n_tiles;
  const int sms = num_sms();
  const int grid = static_cast<int>(work < sms ? (work > 0 ? work : 1) : sms);
  cudaError_t e;
  if (g.paired)
    e = launch_tc_inst<kEpiSituBF16, true>(maps, p, grid, s);
  else if (g.epi == kEpiF32)
    e = launch_tc_inst<kEpiF32, false>(maps, p, grid, s);
  else if (g.epi == kEpiBF16)
    e = launch_tc_inst<kEpiBF16, false>(maps, p, grid, s);
  else
    e = launch_tc_inst<kEpiSigmoidF32, false>(maps, p, grid, s);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status run_gemm_simt(const GemmDesc& g, cudaStream_t s) {
  SimtParams p;
  std::memset(&p, 0, sizeof p);
  for (int i = 0; i < g.nseg; ++i) {
    p.A[i] = static_cast<const float*>(g.seg[i].a);
    p.lda[i] = g.seg[i].a_ld;
    p.B[i] = static_cast<const float*>(g.seg[i].b);
    p.ldb[i] = g.seg[i].b_ld;
    p.seg_k[i] = g.seg[i].K;
  }
  p.nseg = g.nseg;
  if (g.paired) {
    p.B[1] = static_cast<const float*>(g.b_up);
    p.ldb[1] = g.seg[0].b_ld;
  }
  p.M = static_cast<int>(g.M);
  p.tile_table = g.tile_table;
  p.num_m_tiles_dev = g.num_m_tiles_dev;
  p.N = g.N;
  p.b_rows_per_expert = g.b_rows_per_expert;
  p.out = g.out;
  p.ldo = g.ldo;
  p.situ_c = g.situ_c;
  const long long rows = g.tile_table ? static_cast<long long>(g.max_m_tiles) * 4 : cdiv(g.M, 32);
  dim3 grid(static_cast<unsigned>(cdiv(g.N, 32)), static_cast<unsigned>(rows));
  if (g.paired)
    simt_gemm_kernel<kEpiSituBF16, true><<<grid, 256, 0, s>>>(p);
  else if (g.epi == kEpiSigmoidF32)
    simt_gemm_kernel<kEpiSigmoidF32, false><<<grid, 256, 0, s>>>(p);
  else
    simt_gemm_kernel<kEpiF32, false><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status run_gemm(const moe_dims& d, const GemmDesc& g, cudaStream_t s) {
  ++g_last_launches;
  return d.act == MOE_BF16 ? run_gemm_tc(g, s) : run_gemm_simt(g, s);
}

// ------------------------------------------------------------------------------ stages
moe_status stage_router(const moe_dims& d, const void* x, const void* Wr, float* scores, cudaStream_t s) {
  GemmDesc g{};
  g.epi = kEpiSigmoidF32;
  g.M = d.T;
  g.N = d.E;
  g.nseg = 1;
  g.seg[0] = Seg{x, d.H, Wr, d.H, d.E, d.H};
  g.out = scores;
  g.ldo = d.E;
  g.situ_c = d.situ_c;
  g.fault_site = 100;
  return run_gemm(d, g, s);
}

moe_status stage_topk(const moe_dims& d, const float* scores, const float* bias, int32_t* idx, float* w,
                      cudaStream_t s) {
  const unsigned blocks = static_cast<unsigned>(cdiv(d.T, TOPK_WARPS));
  topk_renorm_kernel<<<blocks, TOPK_WARPS * 32, 0, s>>>(scores, bias, d.T, d.E, d.k, idx, w);
  ++g_last_launches;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status stage_dense(const moe_dims& d, int epi, const void* A, long long lda, const void* B, long long N,
                       int K, void* out, long long ldo, int site, cudaStream_t s) {
  GemmDesc g{};
  g.epi = epi;
  g.M = d.T;
  g.N = static_cast<int>(N);
  g.nseg = 1;
  g.seg[0] = Seg{A, lda, B, K, N, K};
  g.out = out;
  g.ldo = ldo;
  g.situ_c = d.situ_c;
  g.fault_site = site;
  return run_gemm(d, g, s);
}

moe_status stage_shared_gate_up(const moe_dims& d, const moe_weights& w, const void* x, void* h_s, cudaStream_t s,
                                int4* dense_tiles = nullptr, int32_t* dense_num = nullptr);

moe_status stage_shared_gate_up_simple(const moe_dims& d, const moe_weights& w, const void* x, void* h_s,
                                       cudaStream_t s) {
  GemmDesc g{};
  g.epi = kEpiSituBF16;
  g.paired = true;
  g.M = d.T;
  g.N = d.S * d.Is;
  g.nseg = 1;
  g.seg[0] = Seg{x, d.H, w.Wsg, d.H, static_cast<long long>(d.S) * d.Is, d.H};
  g.b_up = w.Wsv;
  g.out = h_s;
  g.ldo = static_cast<long long>(d.S) * d.Is;
  g.situ_c = d.situ_c;
  g.fault_site = 130;
  return run_gemm(d, g, s);
}

moe_status stage_permute(const moe_dims& d, const int32_t* idx, const WsLayout& L, void* ws, int32_t* offsets,
                         int32_t* counts_out, int32_t* perm_token, int32_t* inv_perm, cudaStream_t s) {
  const long long ntiles = cdiv(d.T, PERM_TILE);
  int32_t* tile_base = at<int32_t>(ws, L.tile_base);
  int32_t* rank = at<int32_t>(ws, L.rank);
  perm_rank_kernel<<<static_cast<unsigned>(ntiles), PERM_TILE, static_cast<size_t>(d.E) * 16, s>>>(
      idx, d.T, d.E, d.k, tile_base, rank);
  perm_scan_kernel<<<1, 1024, 0, s>>>(tile_base, static_cast<int>(ntiles), d.E, counts_out, offsets,
                                      expert_tile_rows(d), at<int4>(ws, L.tile_table), at<int32_t>(ws, L.num_m_tiles));
  const long long pairs = d.T * d.k;
  perm_scatter_kernel<<<static_cast<unsigned>(cdiv(pairs, 256)), 256, 0, s>>>(idx, d.T, d.E, d.k, tile_base, rank,
                                                                              offsets, perm_token, inv_perm);
  g_last_launches += 3;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status stage_gather(const moe_dims& d, const void* z, void* z_perm, const int32_t* perm_token,
                        const int32_t* n_rows, cudaStream_t s) {
  const long long R = d.T * d.k;
  const int row_vecs = static_cast<int>(static_cast<size_t>(d.L) * act_bytes(d) / 16);
  gather_rows_kernel<<<static_cast<unsigned>(cdiv(R, GATHER_WARPS)), GATHER_WARPS * 32, 0, s>>>(
      static_cast<const uint4*>(z), static_cast<uint4*>(z_perm), perm_token, n_rows, d.T, row_vecs);
  ++g_last_launches;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Maps of the expert-major activation rows [R, K] with 128-, 64-, 32- and
// 16-row boxes (token tiles are staged as a sum of these).
bool make_token_maps(CUtensorMap* maps4, const void* base, uint64_t rows, uint64_t K) {
  for (int i = 0; i < 4; ++i)
    if (!make_map(&maps4[i], base, rows, K, K, 128u >> i)) return false;
  return true;
}

// One CTA pair per two SMs that can co-schedule a cluster of `kern`, asked
// once per device and kernel.
template <typename K>
int cluster_pairs(K kern, cudaLaunchConfig_t cfg, int* cache) {
  int dev = 0;
  cudaGetDevice(&dev);
  int pairs = dev >= 0 && dev < 128 ? cache[dev] : 0;
  if (pairs == 0) {
    cfg.gridDim = dim3(2 * 74);
    int nc = 0;
    if (cudaOccupancyMaxActiveClusters(&nc, kern, &cfg) != cudaSuccess || nc <= 0) nc = num_sms() / 2;
    pairs = nc;
    if (dev >= 0 && dev < 128) cache[dev] = pairs;
  }
  return pairs;
}

template <int EPI, bool PAIRED, int CG, bool MX>
cudaError_t launch_expert_inst(const ExMaps& maps, const ExParams& p, cudaStream_t s) {
  auto kern = tc_expert_kernel<EPI, PAIRED, CG, MX>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(ExCfg<MX>::kSmem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(ExCfg<MX>::kThreads);
  cfg.dynamicSmemBytes = ExCfg<MX>::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (CG == 2) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    static int pairs_cache[128] = {};  // per instantiation and device
    cfg.gridDim = dim3(2 * cluster_pairs(kern, cfg, pairs_cache));
  } else {
    cfg.gridDim = dim3(num_sms());
    cfg.numAttrs = 0;
  }
  return cudaLaunchKernelEx(&cfg, kern, maps, p);
}

template <int EPI, bool PAIRED>
cudaError_t launch_expert(int cg, bool mx, const ExMaps& maps, const ExParams& p, cudaStream_t s) {
  if (mx)
    return cg == 2 ? launch_expert_inst<EPI, PAIRED, 2, true>(maps, p, s)
                   : launch_expert_inst<EPI, PAIRED, 1, true>(maps, p, s);
  return cg == 2 ? launch_expert_inst<EPI, PAIRED, 2, false>(maps, p, s)
                 : launch_expert_inst<EPI, PAIRED, 1, false>(maps, p, s);
}

template <int EPI, bool PAIRED, int CG>
cudaError_t launch_expert2_inst(const X2Maps& maps, const X2Params& p, cudaStream_t s) {
  auto kern = tc_expert2_kernel<EPI, PAIRED, CG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(X2_SMEM));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(X2_THREADS);
  cfg.dynamicSmemBytes = X2_SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (CG == 2) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    static int pairs_cache[128] = {};  // per instantiation and device
    cfg.gridDim = dim3(2 * cluster_pairs(kern, cfg, pairs_cache));
  } else {
    cfg.gridDim = dim3(num_sms());
    cfg.numAttrs = 0;
  }
  return cudaLaunchKernelEx(&cfg, kern, maps, p);
}

// Which grouped expert kernel runs bf16 weights.  The two-weight-tile kernel
// (gemm_expert2.cuh) halves the token rows moved per flop and issues MMAs from
// two threads; its accumulators are single-buffered, and two epilogue warp
// sets drain them.  Measured on B200 at the K3 shapes it is the faster of the
// two: prefill (~290 rows per expert) gate/up 14.67 against 15.15 ms and down
// 7.19 against 7.29 ms, decode (a few rows per expert) 3.5% faster.  So it
// runs whenever its tiles divide evenly.  MOE_EXPERT_KERNEL=one / =two in the
// environment forces either (both compute the same result; used to compare
// them).
bool use_two_tile(const moe_dims& d, bool paired) {
  if (d.act != MOE_BF16 || d.routed != MOE_BF16) return false;
  const int rows = 128 * expert_cg(d);
  if (paired ? d.I % rows != 0 : d.L % rows != 0) return false;
  const char* env = std::getenv("MOE_EXPERT_KERNEL");
  if (env != nullptr && std::strcmp(env, "one") == 0) return false;
  return true;
}

moe_status stage_expert2(const moe_dims& d, bool paired, const void* w0, const void* w1, const void* act, int K,
                         const int4* tile_table, const int32_t* num_tiles, void* out, cudaStream_t s) {
  const long long R = d.T * d.k;
  const int cg = expert_cg(d);
  const int rows_per_expert = paired ? d.I : d.L;
  X2Maps maps;
  std::memset(&maps, 0, sizeof maps);
  const uint64_t wrows = static_cast<uint64_t>(d.E) * rows_per_expert;
  bool ok = make_token_maps(maps.b, act, static_cast<uint64_t>(R), K) && make_map(&maps.a0, w0, wrows, K, K, 128);
  if (paired) ok = ok && make_map(&maps.a1, w1, wrows, K, K, 128);
  if (!ok) return MOE_ERR_CUDA;
  X2Params p{};
  p.tile_table = tile_table;
  p.num_tiles_dev = num_tiles;
  p.n_wtiles = rows_per_expert / (128 * cg);
  p.n_items = paired ? p.n_wtiles : (p.n_wtiles + 1) / 2;
  p.w_rows_per_expert = rows_per_expert;
  p.num_k_blocks = K / EX_BK;
  p.out = out;
  p.ldo = rows_per_expert;
  p.out_cols = rows_per_expert;
  p.situ_c = d.situ_c;
  p.fault_site = paired ? 170 : 180;
  cudaError_t e;
  if (paired)
    e = cg == 2 ? launch_expert2_inst<kEpiSituBF16, true, 2>(maps, p, s)
                : launch_expert2_inst<kEpiSituBF16, true, 1>(maps, p, s);
  else
    e = cg == 2 ? launch_expert2_inst<kEpiF32, false, 2>(maps, p, s) : launch_expert2_inst<kEpiF32, false, 1>(maps, p, s);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status stage_expert_gate_up(const moe_dims& d, const moe_weights& w, const void* z_perm,
                                const int4* tile_table, const int32_t* num_tiles, void* h_perm, cudaStream_t s,
                                int max_tiles = -1) {
  const long long R = d.T * d.k;
  ++g_last_launches;
  if (d.act != MOE_BF16) {
    GemmDesc g{};
    g.epi = kEpiSituBF16;
    g.paired = true;
    g.M = R;
    g.tile_table = tile_table;
    g.num_m_tiles_dev = num_tiles;
    g.max_m_tiles = max_tiles > 0 ? max_tiles : static_cast<int>(cdiv(R, 128) + d.E);
    g.N = d.I;
    g.b_rows_per_expert = d.I;
    g.nseg = 1;
    g.seg[0] = Seg{z_perm, d.L, w.Wg, d.L, static_cast<long long>(d.E) * d.I, d.L};
    g.b_up = w.Wv;
    g.out = h_perm;
    g.ldo = d.I;
    g.situ_c = d.situ_c;
    return run_gemm_simt(g, s);
  }
  if (use_two_tile(d, true)) return stage_expert2(d, true, w.Wg, w.Wv, z_perm, d.L, tile_table, num_tiles, h_perm, s);
  const int cg = expert_cg(d);
  const bool mx = d.routed == MOE_MXFP4;
  ExMaps maps;
  std::memset(&maps, 0, sizeof maps);
  const uint64_t wrows = static_cast<uint64_t>(d.E) * d.I;
  bool ok = make_token_maps(maps.b, z_perm, static_cast<uint64_t>(R), d.L);
  if (mx)
    ok = ok && make_map_u8(&maps.a0, w.Wg, wrows, d.L / 2, 32, 64) && make_map_u8(&maps.a1, w.Wv, wrows, d.L / 2, 32, 64) &&
         make_map_u8(&maps.s0, w.Sg, wrows, d.L / 32, 16, 64) && make_map_u8(&maps.s1, w.Sv, wrows, d.L / 32, 16, 64);
  else
    ok = ok && make_map(&maps.a0, w.Wg, wrows, d.L, d.L, 64) && make_map(&maps.a1, w.Wv, wrows, d.L, d.L, 64);
  if (!ok) return MOE_ERR_CUDA;
  ExParams p{};
  p.tile_table = tile_table;
  p.num_tiles_dev = num_tiles;
  p.n_wtiles = d.I / (64 * cg);
  p.w_rows_per_expert = d.I;
  p.num_k_blocks = d.L / EX_BK;
  p.out = h_perm;
  p.ldo = d.I;
  p.out_cols = d.I;
  p.situ_c = d.situ_c;
  p.fault_site = 140;
  return launch_expert<kEpiSituBF16, true>(cg, mx, maps, p, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status stage_expert_down(const moe_dims& d, const moe_weights& w, const void* h_perm, const int4* tile_table,
                             const int32_t* num_tiles, float* y_perm, cudaStream_t s, int max_tiles = -1) {
  const long long R = d.T * d.k;
  ++g_last_launches;
  if (d.act != MOE_BF16) {
    GemmDesc g{};
    g.epi = kEpiF32;
    g.M = R;
    g.tile_table = tile_table;
    g.num_m_tiles_dev = num_tiles;
    g.max_m_tiles = max_tiles > 0 ? max_tiles : static_cast<int>(cdiv(R, 128) + d.E);
    g.N = d.L;
    g.b_rows_per_expert = d.L;
    g.nseg = 1;
    g.seg[0] = Seg{h_perm, d.I, w.Wo, d.I, static_cast<long long>(d.E) * d.L, d.I};
    g.out = y_perm;
    g.ldo = d.L;
    g.situ_c = d.situ_c;
    return run_gemm_simt(g, s);
  }
  if (use_two_tile(d, false)) return stage_expert2(d, false, w.Wo, nullptr, h_perm, d.I, tile_table, num_tiles, y_perm, s);
  const int cg = expert_cg(d);
  const bool mx = d.routed == MOE_MXFP4;
  ExMaps maps;
  std::memset(&maps, 0, sizeof maps);
  const uint64_t wrows = static_cast<uint64_t>(d.E) * d.L;
  bool ok = make_token_maps(maps.b, h_perm, static_cast<uint64_t>(R), d.I);
  if (mx)
    ok = ok && make_map_u8(&maps.a0, w.Wo, wrows, d.I / 2, 32, 128) && make_map_u8(&maps.s0, w.So, wrows, d.I / 32, 16, 128);
  else
    ok = ok && make_map(&maps.a0, w.Wo, wrows, d.I, d.I, 128);
  if (!ok) return MOE_ERR_CUDA;
  ExParams p{};
  p.tile_table = tile_table;
  p.num_tiles_dev = num_tiles;
  p.n_wtiles = d.L / (128 * cg);
  p.w_rows_per_expert = d.L;
  p.num_k_blocks = d.I / EX_BK;
  p.out = y_perm;
  p.ldo = d.L;
  p.out_cols = d.L;
  p.situ_c = d.situ_c;
  p.fault_site = 150;
  return launch_expert<kEpiF32, false>(cg, mx, maps, p, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ------------------------------------------------------------------------------ block-scaled routed experts
// Quantises rows of the grouped-GEMM token tiles to the block-scaled input
// format of d (MXFP8 codes [R, K] or MXFP4 codes [R, K/2], and scale tiles;
// see mx_quant.cuh).  Row r reads src row src_row[r] (or r).
moe_status stage_quant_mx(const moe_dims& d, const void* src, long long src_rows, const int32_t* src_row,
                          const int4* table, const int32_t* n_tiles, int max_tiles, int K, uint8_t* codes, uint8_t* sf,
                          int site, cudaStream_t s) {
  const int grid = std::max(1, std::min(max_tiles, 8 * num_sms()));
  auto kern = routed_a4(d) ? mx_quant_tiles_kernel<true> : mx_quant_tiles_kernel<false>;
  kern<<<grid, MXQ_WARPS * 32, 0, s>>>(static_cast<const __nv_bfloat16*>(src), src_rows, src_row, table, n_tiles, 0, K,
                                       codes, sf, site);
  ++g_last_launches;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

template <int EPI, bool PAIRED, bool A4>
cudaError_t launch_expert_bs(const BsMaps& maps, const ExParams& p, cudaStream_t s) {
  auto kern = tc_expert_bs_kernel<EPI, PAIRED, A4>;
  constexpr size_t smem = BsStage<A4>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(BS_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static int pairs_cache[128] = {};  // per instantiation and device
  cfg.gridDim = dim3(2 * cluster_pairs(kern, cfg, pairs_cache));
  return cudaLaunchKernelEx(&cfg, kern, maps, p);
}

// Bytes of the re-ordered weight scales of the block-scaled kernels.
size_t tiled_scales_gate_up(const moe_dims& d) {
  return static_cast<size_t>(d.E) * (d.I / 128) * 2 * (d.L / 128) * 512;
}
size_t tiled_scales_down(const moe_dims& d) {
  return static_cast<size_t>(d.E) * (d.L / 256) * 2 * (d.I / 128) * 512;
}

// One block-scaled grouped GEMM: paired = gate/up (W_g / W_v over the latent
// rows, SiTU-GLU -> bf16 h [R, I]); else down (W_o over h -> fp32 [R, L]).
moe_status stage_expert_bs(const moe_dims& d, bool paired, const moe_weights& w, const uint8_t* act_q,
                           const uint8_t* act_sf, long long R, const int4* table, const int32_t* n_tiles,
                           int max_tiles, void* out, int site, cudaStream_t s) {
  ++g_last_launches;
  const int K = paired ? d.L : d.I;
  const int out_rows = paired ? d.I : d.L;  // weight rows per expert
  BsMaps maps;
  std::memset(&maps, 0, sizeof maps);
  const uint64_t wrows = static_cast<uint64_t>(d.E) * out_rows;
  const size_t sa_bytes = paired ? tiled_scales_gate_up(d) : tiled_scales_down(d);
  bool ok = true;
  // scale tiles as 16-byte rows: per stage one box of the weight atoms (one
  // per 128-wide K chunk) and one of the token atoms (two per chunk).  The
  // MXFP4-input kernel reads the packed weight codes as plain bytes.
  const bool a4 = routed_a4(d);
  const uint32_t sfa_rows = (a4 ? BsStage<true>::SFA_BYTES : BsStage<false>::SFA_BYTES) / 16;
  const uint32_t sfb_rows = (a4 ? BsStage<true>::SFB_BYTES : BsStage<false>::SFB_BYTES) / 16;
  const uint32_t b_max_rows = a4 ? BsStage<true>::B_MAX_ROWS : BsStage<false>::B_MAX_ROWS;
  auto wmap = [&](CUtensorMap* m, const void* codes, uint32_t box_rows) {
    return a4 ? make_map_u8_sw128(m, codes, wrows, K / 2, box_rows) : make_map_e2m1(m, codes, wrows, K, box_rows);
  };
  if (paired)
    ok = wmap(&maps.a0, w.Wg, 64) && wmap(&maps.a1, w.Wv, 64) &&
         make_map_u8(&maps.sa, w.Sgv_tiled, sa_bytes / 16, 16, 16, sfa_rows);
  else
    ok = wmap(&maps.a0, w.Wo, 128) && make_map_u8(&maps.sa, w.So_tiled, sa_bytes / 16, 16, 16, sfa_rows);
  for (int i = 0; i < 4 && ok; ++i)
    ok = make_map_u8_sw128(&maps.b[i], act_q, static_cast<uint64_t>(R), bs_code_bytes(d, K),
                           i == 0 ? b_max_rows : 128u >> i);
  const uint64_t sf_rows = static_cast<uint64_t>(max_tiles) * (K / 128) * 64;
  ok = ok && make_map_u8(&maps.sb, act_sf, sf_rows, 16, 16, sfb_rows);
  if (!ok) return MOE_ERR_CUDA;
  ExParams p{};
  p.tile_table = table;
  p.num_tiles_dev = n_tiles;
  p.n_wtiles = paired ? d.I / 128 : d.L / 256;
  p.w_rows_per_expert = out_rows;
  p.num_k_blocks = K / (a4 ? BsStage<true>::K : BsStage<false>::K);
  p.out = out;
  p.ldo = out_rows;
  p.out_cols = out_rows;
  p.situ_c = d.situ_c;
  p.fault_site = site;
  cudaError_t e;
  if (a4)
    e = paired ? launch_expert_bs<kEpiSituBF16, true, true>(maps, p, s) : launch_expert_bs<kEpiF32, false, true>(maps, p, s);
  else
    e = paired ? launch_expert_bs<kEpiSituBF16, true, false>(maps, p, s)
               : launch_expert_bs<kEpiF32, false, false>(maps, p, s);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Buffers of the block-scaled routed-expert sequence.
struct BsBufs {
  uint8_t* xq;   // codes of the expert-major latent rows ([R, L] E4M3 or [R, L/2] packed E2M1)
  uint8_t* sfx;  // their scale tiles
  void* h;       // [R, I] bf16 SiTU-GLU output
  uint8_t* hq;   // codes of h
  uint8_t* sfh;  // their scale tiles
};

// The routed experts on a block-scaled path after the latent rows have been
// quantised: gate/up -> h, h -> MXFP8 / MXFP4, down -> y [R, L] fp32.
moe_status run_routed_bs_after_quant(const moe_dims& d, const moe_weights& w, const BsBufs& b, long long R,
                                     const int4* table, const int32_t* n_tiles, int max_tiles, float* y,
                                     cudaStream_t s, const std::function<void(int, int)>& mark) {
  moe_status st;
  mark(MOE_STAGE_EXPERT_GATE_UP, 0);
  if ((st = stage_expert_bs(d, true, w, b.xq, b.sfx, R, table, n_tiles, max_tiles, b.h, 160, s)) != MOE_OK) return st;
  mark(MOE_STAGE_EXPERT_GATE_UP, 1);
  mark(MOE_STAGE_EXPERT_DOWN, 0);
  if ((st = stage_quant_mx(d, b.h, R, nullptr, table, n_tiles, max_tiles, d.I, b.hq, b.sfh, 181, s)) != MOE_OK)
    return st;
  st = stage_expert_bs(d, false, w, b.hq, b.sfh, R, table, n_tiles, max_tiles, y, 170, s);
  mark(MOE_STAGE_EXPERT_DOWN, 1);
  return st;
}

// The shared experts' gate/up projection with the SiTU-GLU epilogue.  With
// bf16 weights it runs on the 2-CTA grouped expert kernel as one "expert"
// whose S*Is weight rows are W_sg / W_sv (paired row by row) over token tiles
// of 256 rows covering all T rows (its 2-CTA M = 256 tiles move less data per
// MMA than the dense kernel's M = 128 tiles); MOE_SHARED_KERNEL=dense in the
// environment, no workspace for the tile table, or dims that do not tile
// evenly select the one-CTA dense kernel.
moe_status stage_shared_gate_up(const moe_dims& d, const moe_weights& w, const void* x, void* h_s, cudaStream_t s,
                                int4* dense_tiles, int32_t* dense_num) {
  const int rows = d.S * d.Is;
  const char* env = std::getenv("MOE_SHARED_KERNEL");
  const bool pairs = d.act == MOE_BF16 && dense_tiles != nullptr && dense_num != nullptr && rows % 128 == 0 &&
                     d.H % 64 == 0 && !(env != nullptr && std::strcmp(env, "dense") == 0);
  if (!pairs) return stage_shared_gate_up_simple(d, w, x, h_s, s);
  dense_tile_table_kernel<<<1, 256, 0, s>>>(d.T, 256, dense_tiles, dense_num);
  ++g_last_launches;
  ExMaps maps;
  std::memset(&maps, 0, sizeof maps);
  bool ok = make_token_maps(maps.b, x, static_cast<uint64_t>(d.T), d.H) &&
            make_map(&maps.a0, w.Wsg, rows, d.H, d.H, 64) && make_map(&maps.a1, w.Wsv, rows, d.H, d.H, 64);
  if (!ok) return MOE_ERR_CUDA;
  ExParams p{};
  p.tile_table = dense_tiles;
  p.num_tiles_dev = dense_num;
  p.n_wtiles = rows / 128;
  p.w_rows_per_expert = rows;
  p.num_k_blocks = d.H / EX_BK;
  p.out = h_s;
  p.ldo = rows;
  p.out_cols = rows;
  p.situ_c = d.situ_c;
  p.fault_site = 130;
  ++g_last_launches;
  return launch_expert<kEpiSituBF16, true>(2, false, maps, p, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

template <typename OutT>
cudaError_t launch_combine_t(const moe_dims& d, const float* y_perm, const int32_t* inv_perm, const float* w,
                             const float* gamma, float* u, OutT* n, cudaStream_t s) {
  const int nv = d.L / 4;
  const unsigned grid = static_cast<unsigned>(d.T);
  const float eps = d.rms_eps;
  if (nv <= COMBINE_THREADS * 1)
    combine_rmsnorm_kernel<OutT, 1><<<grid, COMBINE_THREADS, 0, s>>>(y_perm, inv_perm, w, gamma, d.k, d.L, eps, u, n);
  else if (nv <= COMBINE_THREADS * 2)
    combine_rmsnorm_kernel<OutT, 2><<<grid, COMBINE_THREADS, 0, s>>>(y_perm, inv_perm, w, gamma, d.k, d.L, eps, u, n);
  else if (nv <= COMBINE_THREADS * 4)
    combine_rmsnorm_kernel<OutT, 4><<<grid, COMBINE_THREADS, 0, s>>>(y_perm, inv_perm, w, gamma, d.k, d.L, eps, u, n);
  else if (nv <= COMBINE_THREADS * 7)
    combine_rmsnorm_kernel<OutT, 7><<<grid, COMBINE_THREADS, 0, s>>>(y_perm, inv_perm, w, gamma, d.k, d.L, eps, u, n);
  else if (nv <= COMBINE_THREADS * 8)
    combine_rmsnorm_kernel<OutT, 8><<<grid, COMBINE_THREADS, 0, s>>>(y_perm, inv_perm, w, gamma, d.k, d.L, eps, u, n);
  else
    combine_rmsnorm_kernel<OutT, 16><<<grid, COMBINE_THREADS, 0, s>>>(y_perm, inv_perm, w, gamma, d.k, d.L, eps, u, n);
  return cudaGetLastError();
}

moe_status stage_combine(const moe_dims& d, const float* y_perm, const int32_t* inv_perm, const float* w,
                         const float* gamma, float* u, void* n, cudaStream_t s) {
  ++g_last_launches;
  cudaError_t e = d.act == MOE_BF16
                      ? launch_combine_t<__nv_bfloat16>(d, y_perm, inv_perm, w, gamma, u, static_cast<__nv_bfloat16*>(n), s)
                      : launch_combine_t<float>(d, y_perm, inv_perm, w, gamma, u, static_cast<float*>(n), s);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status stage_output(const moe_dims& d, const moe_weights& w, const void* h_s, const void* n, void* y,
                        cudaStream_t s) {
  const size_t es = act_bytes(d);
  GemmDesc g{};
  g.epi = (d.y_out == MOE_F32) ? kEpiF32 : kEpiBF16;
  g.M = d.T;
  g.N = d.H;
  g.nseg = d.S + 1;
  for (int i = 0; i < d.S; ++i) {
    const uint8_t* a = static_cast<const uint8_t*>(h_s) + static_cast<size_t>(i) * d.Is * es;
    const uint8_t* b = static_cast<const uint8_t*>(w.Wso) + static_cast<size_t>(i) * d.H * d.Is * es;
    g.seg[i] = Seg{a, static_cast<long long>(d.S) * d.Is, b, d.Is, d.H, d.Is};
  }
  g.seg[d.S] = Seg{n, d.L, w.Wup, d.L, d.H, d.L};
  g.out = y;
  g.ldo = d.H;
  g.situ_c = d.situ_c;
  g.fault_site = 160;
  return run_gemm(d, g, s);
}

// MXFP4 routed weights need their E8M0 scale arrays; other types take none.
moe_status check_scales(const moe_dims& d, const moe_weights& w) {
  if (routed_bs(d)) {
    // block-scaled path: the re-ordered scales (the row-major ones are not
    // read and may be NULL); the packed codes are read as 4-bit TMA tensors,
    // which need 32-byte aligned bases
    if (w.Sgv_tiled == nullptr || w.So_tiled == nullptr || !aligned16(w.Sgv_tiled) || !aligned16(w.So_tiled))
      return MOE_ERR_INVALID_ARG;
    const void* codes[] = {w.Wg, w.Wv, w.Wo};
    for (const void* p : codes)
      if ((reinterpret_cast<uintptr_t>(p) & 31u) != 0) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
  }
  const bool mx = d.routed == MOE_MXFP4;
  const void* sc[] = {w.Sg, w.Sv, w.So};
  for (const void* p : sc) {
    if (mx && (p == nullptr || !aligned16(p))) return MOE_ERR_INVALID_ARG;
    if (!mx && p != nullptr) return MOE_ERR_INVALID_ARG;
  }
  if (w.Sgv_tiled != nullptr || w.So_tiled != nullptr) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

// Workspace of moe_expert_ffn_blocks: h for every row, and a tile table for
// up to ceil(n_rows / 128) + E * n_blocks tiles.
struct BlocksWsLayout {
  size_t h, tile_table, num_tiles, xq, sfx, hq, sfh, total;  // xq .. sfh: block-scaled path only
  int max_tiles;
};

BlocksWsLayout blocks_ws_layout(const moe_dims& d, long long n_rows, int n_blocks) {
  BlocksWsLayout l{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += round_up(bytes, kAlign);
    return o;
  };
  l.max_tiles = static_cast<int>(cdiv(n_rows, 128) + static_cast<long long>(d.E) * n_blocks);
  l.h = take(static_cast<size_t>(n_rows) * d.I * act_bytes(d));
  l.tile_table = take(static_cast<size_t>(l.max_tiles) * 16);
  l.num_tiles = take(16);
  const bool bs = routed_bs(d);
  const size_t rows = static_cast<size_t>(n_rows), mt = static_cast<size_t>(l.max_tiles);
  l.xq = take(bs ? rows * bs_code_bytes(d, d.L) : 0);
  l.sfx = take(bs ? mt * (d.L / 128) * 1024 : 0);
  l.hq = take(bs ? rows * bs_code_bytes(d, d.I) : 0);
  l.sfh = take(bs ? mt * (d.I / 128) * 1024 : 0);
  l.total = off;
  return l;
}

bool ws_ok(const moe_dims& d, const void* ws, size_t ws_bytes) {
  return ws != nullptr && (reinterpret_cast<uintptr_t>(ws) % kAlign) == 0 && ws_bytes >= ws_layout(d).total;
}

// ------------------------------------------------------------------------------ backward pass
struct BwLayout {
  size_t s, p, tile_base, rank, offsets, perm_token, inv_perm, tile_table, num_tiles, z, z_perm, g, v, h, y_perm, u,
      n, r, gs, vs, hs, dn, du, dp, dy_perm, dh, dz_perm, dz, dhs, dl, total;
  int max_tiles;
};

BwLayout bw_layout(const moe_dims& d) {
  BwLayout l{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += round_up(bytes, kAlign);
    return o;
  };
  const size_t T = static_cast<size_t>(d.T), R = T * d.k, E = d.E, L = d.L, I = d.I, SI = static_cast<size_t>(d.S) * d.Is;
  l.max_tiles = static_cast<int>(cdiv(static_cast<long long>(R), BW_TILE) + d.E);
  l.s = take(T * E * 4);
  l.p = take(R * 4);
  l.tile_base = take(static_cast<size_t>(cdiv(d.T, PERM_TILE)) * E * 4);
  l.rank = take(R * 4);
  l.offsets = take((E + 1) * 4);
  l.perm_token = take(R * 4);
  l.inv_perm = take(R * 4);
  l.tile_table = take(static_cast<size_t>(l.max_tiles) * 16);
  l.num_tiles = take(16);
  l.z = take(T * L * 4);
  l.z_perm = take(R * L * 4);
  l.g = take(R * I * 4);
  l.v = take(R * I * 4);
  l.h = take(R * I * 4);
  l.y_perm = take(R * L * 4);
  l.u = take(T * L * 4);
  l.n = take(T * L * 4);
  l.r = take(T * 4);
  l.gs = take(T * SI * 4);
  l.vs = take(T * SI * 4);
  l.hs = take(T * SI * 4);
  l.dn = take(T * L * 4);
  l.du = take(T * L * 4);
  l.dp = take(R * 4);
  l.dy_perm = take(R * L * 4);
  l.dh = take(R * I * 4);
  l.dz_perm = take(R * L * 4);
  l.dz = take(T * L * 4);
  l.dhs = take(T * SI * 4);
  l.dl = take(T * E * 4);
  l.total = off;
  return l;
}

// One strided GEMM launch (backward.cuh).  ta / tb: element types of A and B
// (true = bf16, false = fp32).
template <typename TA, typename TB>
void bw_launch_t(int mode, const BwGemm& g, int e_count, int max_tiles, cudaStream_t s) {
  const unsigned gx = static_cast<unsigned>(cdiv(g.N, BW_TILE));
  if (mode == kBwDense)
    bw_gemm_kernel<TA, TB, kBwDense><<<dim3(gx, static_cast<unsigned>(cdiv(g.M, BW_TILE))), BW_THREADS, 0, s>>>(g);
  else if (mode == kBwRows)
    bw_gemm_kernel<TA, TB, kBwRows><<<dim3(gx, static_cast<unsigned>(max_tiles)), BW_THREADS, 0, s>>>(g);
  else
    bw_gemm_kernel<TA, TB, kBwKRows>
        <<<dim3(gx, static_cast<unsigned>(cdiv(g.M, BW_TILE)), static_cast<unsigned>(e_count)), BW_THREADS, 0, s>>>(g);
}

void bw_launch(bool a_bf16, bool b_bf16, int mode, const BwGemm& g, int e_count, int max_tiles, cudaStream_t s) {
  ++g_last_launches;
  if (a_bf16 && b_bf16)
    bw_launch_t<__nv_bfloat16, __nv_bfloat16>(mode, g, e_count, max_tiles, s);
  else if (a_bf16)
    bw_launch_t<__nv_bfloat16, float>(mode, g, e_count, max_tiles, s);
  else if (b_bf16)
    bw_launch_t<float, __nv_bfloat16>(mode, g, e_count, max_tiles, s);
  else
    bw_launch_t<float, float>(mode, g, e_count, max_tiles, s);
}

// C[M, N] (+)= A(m, k) B(k, n) with explicit strides (a dense problem).
BwGemm bw_dense(const void* a, long long a_m, long long a_k, const void* b, long long b_k, long long b_n, float* c,
                long long ldc, int M, int N, int K, float beta) {
  BwGemm g{};
  g.a = a;
  g.a_m = a_m;
  g.a_k = a_k;
  g.b = b;
  g.b_k = b_k;
  g.b_n = b_n;
  g.c = c;
  g.ldc = ldc;
  g.M = M;
  g.N = N;
  g.K = K;
  g.beta = beta;
  return g;
}

moe_status run_backward(const moe_dims& d, const moe_weights& w, const void* x, const float* dy, const int32_t* idx,
                        const moe_grads& gr, void* ws, cudaStream_t st) {
  const BwLayout Lw = bw_layout(d);
  const bool bf = d.act == MOE_BF16;
  const int T = static_cast<int>(d.T), H = d.H, L = d.L, E = d.E, k = d.k, I = d.I, S = d.S, Is = d.Is;
  const long long R = static_cast<long long>(T) * k;
  const int SI = S * Is;
  const size_t es = act_bytes(d);
  float* s = at<float>(ws, Lw.s);
  float* p = at<float>(ws, Lw.p);
  int32_t* offsets = at<int32_t>(ws, Lw.offsets);
  int32_t* perm_token = at<int32_t>(ws, Lw.perm_token);
  int32_t* inv_perm = at<int32_t>(ws, Lw.inv_perm);
  const int4* table = at<int4>(ws, Lw.tile_table);
  const int32_t* ntiles = at<int32_t>(ws, Lw.num_tiles);
  float *z = at<float>(ws, Lw.z), *z_perm = at<float>(ws, Lw.z_perm), *g = at<float>(ws, Lw.g),
        *v = at<float>(ws, Lw.v), *h = at<float>(ws, Lw.h), *y_perm = at<float>(ws, Lw.y_perm),
        *u = at<float>(ws, Lw.u), *n = at<float>(ws, Lw.n), *r = at<float>(ws, Lw.r), *gs = at<float>(ws, Lw.gs),
        *vs = at<float>(ws, Lw.vs), *hs = at<float>(ws, Lw.hs), *dn = at<float>(ws, Lw.dn),
        *du = at<float>(ws, Lw.du), *dp = at<float>(ws, Lw.dp), *dy_perm = at<float>(ws, Lw.dy_perm),
        *dh = at<float>(ws, Lw.dh), *dz_perm = at<float>(ws, Lw.dz_perm), *dz = at<float>(ws, Lw.dz),
        *dhs = at<float>(ws, Lw.dhs), *dl = at<float>(ws, Lw.dl);
  const int mt = Lw.max_tiles;
  auto ew = [](long long count) { return static_cast<unsigned>(cdiv(count, BW_EW_THREADS)); };

  // ---- forward quantities, fp32
  bw_launch(bf, bf, kBwDense, bw_dense(x, H, 1, w.Wr, 1, H, s, E, T, E, H, 0.f), 0, 0, st);  // logits
  bw_sigmoid_kernel<<<ew(static_cast<long long>(T) * E), BW_EW_THREADS, 0, st>>>(s, static_cast<long long>(T) * E);
  bw_mix_kernel<<<ew(T), BW_EW_THREADS, 0, st>>>(s, idx, T, E, k, p);
  bw_launch(bf, bf, kBwDense, bw_dense(x, H, 1, w.Wdown, 1, H, z, L, T, L, H, 0.f), 0, 0, st);  // z
  const long long ntok = cdiv(d.T, PERM_TILE);
  perm_rank_kernel<<<static_cast<unsigned>(ntok), PERM_TILE, static_cast<size_t>(E) * 16, st>>>(
      idx, d.T, E, k, at<int32_t>(ws, Lw.tile_base), at<int32_t>(ws, Lw.rank));
  perm_scan_kernel<<<1, 1024, 0, st>>>(at<int32_t>(ws, Lw.tile_base), static_cast<int>(ntok), E, nullptr, offsets,
                                       BW_TILE, at<int4>(ws, Lw.tile_table), at<int32_t>(ws, Lw.num_tiles));
  perm_scatter_kernel<<<static_cast<unsigned>(cdiv(R, 256)), 256, 0, st>>>(
      idx, d.T, E, k, at<int32_t>(ws, Lw.tile_base), at<int32_t>(ws, Lw.rank), offsets, perm_token, inv_perm);
  g_last_launches += 5;
  bw_gather_rows_f32_kernel<float><<<ew(R * L), BW_EW_THREADS, 0, st>>>(z, perm_token, R, L, z_perm);
  // g / v / h / y_perm of the routed experts over the expert-major rows
  BwGemm gg = bw_dense(z_perm, L, 1, w.Wg, 1, L, g, I, 0, I, L, 0.f);
  gg.tile_table = table;
  gg.num_tiles = ntiles;
  gg.b_e = static_cast<long long>(I) * L;
  bw_launch(false, bf, kBwRows, gg, 0, mt, st);
  gg.b = w.Wv;
  gg.c = v;
  bw_launch(false, bf, kBwRows, gg, 0, mt, st);
  bw_situ_kernel<<<ew(R * I), BW_EW_THREADS, 0, st>>>(g, v, R * I, d.situ_c, h);
  BwGemm gy = bw_dense(h, I, 1, w.Wo, 1, I, y_perm, L, 0, L, I, 0.f);
  gy.tile_table = table;
  gy.num_tiles = ntiles;
  gy.b_e = static_cast<long long>(L) * I;
  bw_launch(false, bf, kBwRows, gy, 0, mt, st);
  bw_combine_kernel<<<static_cast<unsigned>(T), BW_EW_THREADS, 0, st>>>(y_perm, inv_perm, p, w.gamma, k, L, d.rms_eps,
                                                                       u, n, r);
  for (int i = 0; i < S; ++i) {  // shared experts' pre-activations
    const uint8_t* wsg = static_cast<const uint8_t*>(w.Wsg) + static_cast<size_t>(i) * Is * H * es;
    const uint8_t* wsv = static_cast<const uint8_t*>(w.Wsv) + static_cast<size_t>(i) * Is * H * es;
    bw_launch(bf, bf, kBwDense, bw_dense(x, H, 1, wsg, 1, H, gs + i * Is, SI, T, Is, H, 0.f), 0, 0, st);
    bw_launch(bf, bf, kBwDense, bw_dense(x, H, 1, wsv, 1, H, vs + i * Is, SI, T, Is, H, 0.f), 0, 0, st);
  }
  if (S > 0) bw_situ_kernel<<<ew(static_cast<long long>(T) * SI), BW_EW_THREADS, 0, st>>>(gs, vs, static_cast<long long>(T) * SI, d.situ_c, hs);

  // ---- gradients
  bw_launch(false, bf, kBwDense, bw_dense(dy, H, 1, w.Wup, L, 1, dn, L, T, L, H, 0.f), 0, 0, st);       // dn
  bw_launch(false, false, kBwDense, bw_dense(dy, 1, H, n, L, 1, gr.dWup, L, H, L, T, 0.f), 0, 0, st);   // dW_up
  for (int i = 0; i < S; ++i) {
    const uint8_t* wso = static_cast<const uint8_t*>(w.Wso) + static_cast<size_t>(i) * H * Is * es;
    bw_launch(false, bf, kBwDense, bw_dense(dy, H, 1, wso, Is, 1, dhs + i * Is, SI, T, Is, H, 0.f), 0, 0, st);
    bw_launch(false, false, kBwDense,
              bw_dense(dy, 1, H, hs + i * Is, SI, 1, gr.dWso + static_cast<size_t>(i) * H * Is, Is, H, Is, T, 0.f), 0,
              0, st);
  }
  if (S > 0) {
    bw_situ_grad_kernel<<<ew(static_cast<long long>(T) * SI), BW_EW_THREADS, 0, st>>>(gs, vs, dhs,
                                                                                      static_cast<long long>(T) * SI,
                                                                                      d.situ_c);
    for (int i = 0; i < S; ++i) {
      bw_launch(false, bf, kBwDense,
                bw_dense(gs + i * Is, 1, SI, x, H, 1, gr.dWsg + static_cast<size_t>(i) * Is * H, H, Is, H, T, 0.f), 0,
                0, st);
      bw_launch(false, bf, kBwDense,
                bw_dense(vs + i * Is, 1, SI, x, H, 1, gr.dWsv + static_cast<size_t>(i) * Is * H, H, Is, H, T, 0.f), 0,
                0, st);
    }
  }
  bw_combine_grad_kernel<<<static_cast<unsigned>(T), BW_EW_THREADS, 0, st>>>(dn, u, r, w.gamma, y_perm, inv_perm, p,
                                                                            k, L, du, dp, dy_perm);
  bw_dgamma_kernel<<<static_cast<unsigned>(cdiv(L, 128)), 128, 0, st>>>(dn, u, r, d.T, L, gr.dgamma);
  // routed experts
  BwGemm gdh = bw_dense(dy_perm, L, 1, w.Wo, I, 1, dh, I, 0, I, L, 0.f);
  gdh.tile_table = table;
  gdh.num_tiles = ntiles;
  gdh.b_e = static_cast<long long>(L) * I;
  bw_launch(false, bf, kBwRows, gdh, 0, mt, st);  // dh = dy_perm W_o[e]
  BwGemm gwo{};
  gwo.a = dy_perm;
  gwo.a_m = 1;
  gwo.a_row = L;
  gwo.b = h;
  gwo.b_row = I;
  gwo.b_n = 1;
  gwo.c = gr.dWo;
  gwo.ldc = I;
  gwo.c_e = static_cast<long long>(L) * I;
  gwo.M = L;
  gwo.N = I;
  gwo.offsets = offsets;
  bw_launch(false, false, kBwKRows, gwo, E, 0, st);  // dW_o[e] = dy_e^T h_e
  bw_situ_grad_kernel<<<ew(R * I), BW_EW_THREADS, 0, st>>>(g, v, dh, R * I, d.situ_c);  // g, v <- dg, dv
  BwGemm gwg = gwo;
  gwg.a = g;
  gwg.a_row = I;
  gwg.b = z_perm;
  gwg.b_row = L;
  gwg.c = gr.dWg;
  gwg.ldc = L;
  gwg.c_e = static_cast<long long>(I) * L;
  gwg.M = I;
  gwg.N = L;
  bw_launch(false, false, kBwKRows, gwg, E, 0, st);  // dW_g[e] = dg_e^T z_e
  gwg.a = v;
  gwg.c = gr.dWv;
  bw_launch(false, false, kBwKRows, gwg, E, 0, st);  // dW_v[e] = dv_e^T z_e
  BwGemm gdz = bw_dense(g, I, 1, w.Wg, L, 1, dz_perm, L, 0, L, I, 0.f);
  gdz.tile_table = table;
  gdz.num_tiles = ntiles;
  gdz.b_e = static_cast<long long>(I) * L;
  bw_launch(false, bf, kBwRows, gdz, 0, mt, st);  // dz_perm = dg W_g[e]
  gdz.a = v;
  gdz.b = w.Wv;
  gdz.beta = 1.f;
  bw_launch(false, bf, kBwRows, gdz, 0, mt, st);  //        + dv W_v[e]
  bw_gather_sum_kernel<<<ew(static_cast<long long>(T) * L), BW_EW_THREADS, 0, st>>>(dz_perm, inv_perm, d.T, k, L, dz);
  bw_router_grad_kernel<<<static_cast<unsigned>(T), 128, 0, st>>>(s, idx, p, dp, d.T, E, k, dl);
  g_last_launches += 11;
  // latent projection and router weight gradients, then dx
  bw_launch(false, bf, kBwDense, bw_dense(dz, 1, L, x, H, 1, gr.dWdown, H, L, H, T, 0.f), 0, 0, st);
  bw_launch(false, bf, kBwDense, bw_dense(dl, 1, E, x, H, 1, gr.dWr, H, E, H, T, 0.f), 0, 0, st);
  bw_launch(false, bf, kBwDense, bw_dense(dz, L, 1, w.Wdown, H, 1, gr.dx, H, T, H, L, 0.f), 0, 0, st);
  bw_launch(false, bf, kBwDense, bw_dense(dl, E, 1, w.Wr, H, 1, gr.dx, H, T, H, E, 1.f), 0, 0, st);
  for (int i = 0; i < S; ++i) {
    const uint8_t* wsg = static_cast<const uint8_t*>(w.Wsg) + static_cast<size_t>(i) * Is * H * es;
    const uint8_t* wsv = static_cast<const uint8_t*>(w.Wsv) + static_cast<size_t>(i) * Is * H * es;
    bw_launch(false, bf, kBwDense, bw_dense(gs + i * Is, SI, 1, wsg, H, 1, gr.dx, H, T, H, Is, 1.f), 0, 0, st);
    bw_launch(false, bf, kBwDense, bw_dense(vs + i * Is, SI, 1, wsv, H, 1, gr.dx, H, T, H, Is, 1.f), 0, 0, st);
  }
  (void)du;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace
// MXFP8 / MXFP4 quantisation of row-major bf16 rows (row-major scales).
moe_status mx_quantize_rows(bool fp4, const void* x, int64_t rows, int32_t K, uint8_t* codes, uint8_t* scales,
                            moe_stream_t stream, int site) {
  if (rows < 0 || K <= 0 || K % 32 != 0 || rows > 0x7fffffffLL) return MOE_ERR_INVALID_ARG;
  if (rows > 0 && (x == nullptr || codes == nullptr || scales == nullptr || !aligned16(x) || !aligned16(codes)))
    return MOE_ERR_INVALID_ARG;
  g_last_launches = 0;
  if (rows == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long tiles = cdiv(rows, 128);
  const int grid = static_cast<int>(std::min<long long>(tiles, 8LL * num_sms()));
  auto kern = fp4 ? mx_quant_tiles_kernel<true> : mx_quant_tiles_kernel<false>;
  kern<<<grid, MXQ_WARPS * 32, 0, s>>>(static_cast<const __nv_bfloat16*>(x), rows, nullptr, nullptr, nullptr, rows, K,
                                       codes, scales, site);
  g_last_launches = 1;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_size(const moe_dims* d) {
  if (!dims_ok(d)) return 0;
  return ws_layout(*d).total;
}

const char* moe_status_str(moe_status s) {
  switch (s) {
    case MOE_OK:
      return "MOE_OK";
    case MOE_ERR_INVALID_ARG:
      return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED:
      return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_CUDA:
      return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE:
      return "MOE_ERR_DEVICE";
  }
  return "unknown moe_status";
}

int moe_last_launch_count(void) { return g_last_launches; }

moe_status moe_router_topk(const moe_dims* d, const void* x, const void* Wr, const float* bias, float* scores,
                           int from_scores, int32_t* topk_idx, float* topk_w, moe_stream_t stream) {
  moe_status st = check_dims(d);
  if (st != MOE_OK) return st;
  if (!aligned16(scores) || scores == nullptr || bias == nullptr || topk_idx == nullptr || topk_w == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (!from_scores && (x == nullptr || Wr == nullptr || !aligned16(x) || !aligned16(Wr))) return MOE_ERR_INVALID_ARG;
  g_last_launches = 0;
  if (d->T == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!from_scores) {
    st = stage_router(*d, x, Wr, scores, s);
    if (st != MOE_OK) return st;
  }
  return stage_topk(*d, scores, bias, topk_idx, topk_w, s);
}

moe_status moe_permute(const moe_dims* d, const int32_t* topk_idx, const void* z, int32_t* expert_offsets,
                       int32_t* perm_token, int32_t* inv_perm, void* z_perm, void* ws, size_t ws_bytes,
                       moe_stream_t stream) {
  moe_status st = check_dims(d);
  if (st != MOE_OK) return st;
  if (topk_idx == nullptr || expert_offsets == nullptr || perm_token == nullptr || inv_perm == nullptr)
    return MOE_ERR_INVALID_ARG;
  if ((z == nullptr) != (z_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  if (z != nullptr && (!aligned16(z) || !aligned16(z_perm))) return MOE_ERR_INVALID_ARG;
  if (!ws_ok(*d, ws, ws_bytes)) return MOE_ERR_INVALID_ARG;
  g_last_launches = 0;
  if (d->T == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(*d);
  st = stage_permute(*d, topk_idx, L, ws, expert_offsets, nullptr, perm_token, inv_perm, s);
  if (st != MOE_OK) return st;
  if (z != nullptr) st = stage_gather(*d, z, z_perm, perm_token, expert_offsets + d->E, s);
  return st;
}

moe_status moe_expert_ffn(const moe_dims* d, const moe_weights* w, const void* z_perm,
                          const int32_t* expert_offsets, float* y_perm, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
  moe_status st = check_dims(d);
  if (st != MOE_OK) return st;
  if (w == nullptr || z_perm == nullptr || expert_offsets == nullptr || y_perm == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w->Wg) || !aligned16(w->Wv) || !aligned16(w->Wo) || w->Wg == nullptr || w->Wv == nullptr ||
      w->Wo == nullptr || !aligned16(z_perm) || !aligned16(y_perm))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_scales(*d, *w)) != MOE_OK) return st;
  if (!ws_ok(*d, ws, ws_bytes)) return MOE_ERR_INVALID_ARG;
  g_last_launches = 0;
  if (d->T == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(*d);
  tile_table_kernel<<<1, 1024, 0, s>>>(expert_offsets, d->E, d->T * d->k, expert_tile_rows(*d),
                                       at<int4>(ws, L.tile_table), at<int32_t>(ws, L.num_m_tiles));
  ++g_last_launches;
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  const int4* table = at<int4>(ws, L.tile_table);
  const int32_t* n_tiles = at<int32_t>(ws, L.num_m_tiles);
  if (routed_bs(*d)) {
    const long long R = d->T * d->k;
    const int max_tiles = static_cast<int>(cdiv(R, TC_BM) + d->E);
    const BsBufs b{at<uint8_t>(ws, L.z_perm), at<uint8_t>(ws, L.sf_z), at<void>(ws, L.h_perm), at<uint8_t>(ws, L.h_q),
                   at<uint8_t>(ws, L.sf_h)};
    if ((st = stage_quant_mx(*d, z_perm, R, nullptr, table, n_tiles, max_tiles, d->L, b.xq, b.sfx, 180, s)) != MOE_OK)
      return st;
    return run_routed_bs_after_quant(*d, *w, b, R, table, n_tiles, max_tiles, y_perm, s, [](int, int) {});
  }
  st = stage_expert_gate_up(*d, *w, z_perm, table, n_tiles, at<void>(ws, L.h_perm), s);
  if (st != MOE_OK) return st;
  return stage_expert_down(*d, *w, at<void>(ws, L.h_perm), table, n_tiles, y_perm, s);
}

moe_status moe_combine(const moe_dims* d, const float* y_perm, const int32_t* inv_perm, const float* topk_w,
                       const float* gamma, float* u_out, void* n_out, moe_stream_t stream) {
  moe_status st = check_dims(d);
  if (st != MOE_OK) return st;
  if (y_perm == nullptr || inv_perm == nullptr || topk_w == nullptr || gamma == nullptr || n_out == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_perm) || !aligned16(gamma) || !aligned16(n_out) || !aligned16(u_out)) return MOE_ERR_INVALID_ARG;
  g_last_launches = 0;
  if (d->T == 0) return MOE_OK;
  return stage_combine(*d, y_perm, inv_perm, topk_w, gamma, u_out, n_out, reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_layer_forward(const moe_dims* d, const moe_weights* w, const void* x, void* y, const moe_aux* aux,
                             void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_dims(d);
  if (st != MOE_OK) return st;
  if (w == nullptr || x == nullptr || y == nullptr) return MOE_ERR_INVALID_ARG;
  const void* need[] = {w->Wr, w->bias, w->Wdown, w->Wup, w->gamma, w->Wg, w->Wv, w->Wo, x, y};
  for (const void* p : need)
    if (p == nullptr || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (d->S > 0 && (w->Wsg == nullptr || w->Wsv == nullptr || w->Wso == nullptr || !aligned16(w->Wsg) ||
                   !aligned16(w->Wsv) || !aligned16(w->Wso)))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_scales(*d, *w)) != MOE_OK) return st;
  moe_aux a{};
  if (aux != nullptr) a = *aux;
  const void* auxp[] = {a.scores, a.topk_idx, a.topk_w, a.expert_offsets, a.u, a.n, a.z};
  if (a.stage_events != nullptr)
    for (int i = 0; i < 2 * MOE_NUM_STAGES; ++i)
      if (a.stage_events[i] == nullptr) return MOE_ERR_INVALID_ARG;
  for (const void* p : auxp)
    if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (!ws_ok(*d, ws, ws_bytes)) return MOE_ERR_INVALID_ARG;
  g_last_launches = 0;
  if (d->T == 0) return MOE_OK;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(*d);
  float* scores = a.scores ? a.scores : at<float>(ws, L.scores);
  int32_t* idx = a.topk_idx ? a.topk_idx : at<int32_t>(ws, L.topk_idx);
  float* tw = a.topk_w ? a.topk_w : at<float>(ws, L.topk_w);
  int32_t* offsets = a.expert_offsets ? a.expert_offsets : at<int32_t>(ws, L.offsets);
  void* z = a.z ? a.z : at<void>(ws, L.z);
  void* n = a.n ? a.n : at<void>(ws, L.n);
  void* h_s = at<void>(ws, L.h_s);
  int32_t* perm_token = at<int32_t>(ws, L.perm_token);
  int32_t* inv_perm = at<int32_t>(ws, L.inv_perm);

  // Records event 2*stage (+1 after) when the caller asked for stage timing.
  auto mark = [&](int stage, int after) {
    if (a.stage_events != nullptr)
      cudaEventRecord(static_cast<cudaEvent_t>(a.stage_events[2 * stage + after]), s);
  };
  // x-side: router scores, latent projection, shared experts' gate/up
  mark(MOE_STAGE_ROUTER, 0);
  if ((st = stage_router(*d, x, w->Wr, scores, s)) != MOE_OK) return st;
  mark(MOE_STAGE_ROUTER, 1);
  mark(MOE_STAGE_TOPK, 0);
  if ((st = stage_topk(*d, scores, w->bias, idx, tw, s)) != MOE_OK) return st;
  mark(MOE_STAGE_TOPK, 1);
  mark(MOE_STAGE_LATENT_DOWN, 0);
  if ((st = stage_dense(*d, d->act == MOE_BF16 ? kEpiBF16 : kEpiF32, x, d->H, w->Wdown, d->L, d->H, z, d->L, 120,
                        s)) != MOE_OK)
    return st;
  mark(MOE_STAGE_LATENT_DOWN, 1);
  mark(MOE_STAGE_SHARED_GATE_UP, 0);
  if (d->S > 0 && (st = stage_shared_gate_up(*d, *w, x, h_s, s, at<int4>(ws, L.dense_tiles),
                                             at<int32_t>(ws, L.dense_num))) != MOE_OK)
    return st;
  mark(MOE_STAGE_SHARED_GATE_UP, 1);
  // dispatch
  mark(MOE_STAGE_PERMUTE, 0);
  if ((st = stage_permute(*d, idx, L, ws, offsets, nullptr, perm_token, inv_perm, s)) != MOE_OK) return st;
  mark(MOE_STAGE_PERMUTE, 1);
  // routed experts
  const int4* table = at<int4>(ws, L.tile_table);
  const int32_t* n_tiles = at<int32_t>(ws, L.num_m_tiles);
  if (routed_bs(*d)) {
    // block-scaled paths: the gather writes the MXFP8 / MXFP4 codes and
    // scales of the expert-major z rows; h is quantised in the down stage
    const long long R = d->T * d->k;
    const int max_tiles = static_cast<int>(cdiv(R, TC_BM) + d->E);
    const BsBufs b{at<uint8_t>(ws, L.z_perm), at<uint8_t>(ws, L.sf_z), at<void>(ws, L.h_perm), at<uint8_t>(ws, L.h_q),
                   at<uint8_t>(ws, L.sf_h)};
    mark(MOE_STAGE_GATHER, 0);
    if ((st = stage_quant_mx(*d, z, d->T, perm_token, table, n_tiles, max_tiles, d->L, b.xq, b.sfx, 180, s)) != MOE_OK)
      return st;
    mark(MOE_STAGE_GATHER, 1);
    if ((st = run_routed_bs_after_quant(*d, *w, b, R, table, n_tiles, max_tiles, at<float>(ws, L.y_perm), s, mark)) !=
        MOE_OK)
      return st;
  } else {
    mark(MOE_STAGE_GATHER, 0);
    if ((st = stage_gather(*d, z, at<void>(ws, L.z_perm), perm_token, offsets + d->E, s)) != MOE_OK) return st;
    mark(MOE_STAGE_GATHER, 1);
    mark(MOE_STAGE_EXPERT_GATE_UP, 0);
    if ((st = stage_expert_gate_up(*d, *w, at<void>(ws, L.z_perm), table, n_tiles, at<void>(ws, L.h_perm), s)) != MOE_OK)
      return st;
    mark(MOE_STAGE_EXPERT_GATE_UP, 1);
    mark(MOE_STAGE_EXPERT_DOWN, 0);
    if ((st = stage_expert_down(*d, *w, at<void>(ws, L.h_perm), table, n_tiles, at<float>(ws, L.y_perm), s)) != MOE_OK)
      return st;
    mark(MOE_STAGE_EXPERT_DOWN, 1);
  }
  // combine + RMSNorm, then [shared | W_up] output projection
  mark(MOE_STAGE_COMBINE, 0);
  if ((st = stage_combine(*d, at<float>(ws, L.y_perm), inv_perm, tw, w->gamma, a.u, n, s)) != MOE_OK) return st;
  mark(MOE_STAGE_COMBINE, 1);
  mark(MOE_STAGE_OUTPUT, 0);
  st = stage_output(*d, *w, h_s, n, y, s);
  mark(MOE_STAGE_OUTPUT, 1);
  return st;
}

moe_status moe_latent_shared(const moe_dims* d, const moe_weights* w, const void* x, void* z, void* h_s,
                             moe_stream_t stream) {
  moe_status st = check_dims(d);
  if (st != MOE_OK) return st;
  if (w == nullptr || x == nullptr || z == nullptr || !aligned16(x) || !aligned16(z) || w->Wdown == nullptr ||
      !aligned16(w->Wdown))
    return MOE_ERR_INVALID_ARG;
  if (d->S > 0 && (h_s == nullptr || !aligned16(h_s) || w->Wsg == nullptr || w->Wsv == nullptr ||
                   !aligned16(w->Wsg) || !aligned16(w->Wsv)))
    return MOE_ERR_INVALID_ARG;
  g_last_launches = 0;
  if (d->T == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = stage_dense(*d, d->act == MOE_BF16 ? kEpiBF16 : kEpiF32, x, d->H, w->Wdown, d->L, d->H, z, d->L, 120,
                        s)) != MOE_OK)
    return st;
  if (d->S > 0) st = stage_shared_gate_up(*d, *w, x, h_s, s);
  return st;
}

moe_status moe_output(const moe_dims* d, const moe_weights* w, const void* h_s, const void* n, void* y,
                      moe_stream_t stream) {
  moe_status st = check_dims(d);
  if (st != MOE_OK) return st;
  if (w == nullptr || n == nullptr || y == nullptr || !aligned16(n) || !aligned16(y) || w->Wup == nullptr ||
      !aligned16(w->Wup))
    return MOE_ERR_INVALID_ARG;
  if (d->S > 0 && (h_s == nullptr || !aligned16(h_s) || w->Wso == nullptr || !aligned16(w->Wso)))
    return MOE_ERR_INVALID_ARG;
  g_last_launches = 0;
  if (d->T == 0) return MOE_OK;
  return stage_output(*d, *w, h_s, n, y, reinterpret_cast<cudaStream_t>(stream));
}

size_t moe_expert_ffn_blocks_workspace_size(const moe_dims* d, int64_t n_rows, int32_t n_blocks) {
  if (!dims_ok(d) || n_rows < 0 || n_blocks < 1) return 0;
  return blocks_ws_layout(*d, n_rows, n_blocks).total;
}

moe_status moe_expert_ffn_blocks(const moe_dims* d, const moe_weights* w, const void* x_rows, int64_t n_rows,
                                 const int32_t* block_offsets, int32_t n_blocks, float* y_rows, void* ws,
                                 size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_dims(d);
  if (st != MOE_OK) return st;
  if (w == nullptr || x_rows == nullptr || block_offsets == nullptr || y_rows == nullptr || n_rows < 0 ||
      n_blocks < 1 || n_rows > 0x7fffffffLL)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(w->Wg) || !aligned16(w->Wv) || !aligned16(w->Wo) || w->Wg == nullptr || w->Wv == nullptr ||
      w->Wo == nullptr || !aligned16(x_rows) || !aligned16(y_rows))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_scales(*d, *w)) != MOE_OK) return st;
  const BlocksWsLayout L = blocks_ws_layout(*d, n_rows, n_blocks);
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 || ws_bytes < L.total)
    return MOE_ERR_INVALID_ARG;
  g_last_launches = 0;
  if (n_rows == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The stages size their row tensor maps from d->T * d->k: describe the rows as
  // n_rows single-slot tokens.
  moe_dims dr = *d;
  dr.T = n_rows;
  dr.k = 1;
  tile_table_blocks_kernel<<<1, 1024, 0, s>>>(block_offsets, n_blocks, d->E, n_rows, expert_tile_rows(dr),
                                              at<int4>(ws, L.tile_table), at<int32_t>(ws, L.num_tiles));
  ++g_last_launches;
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  const int4* table = at<int4>(ws, L.tile_table);
  const int32_t* n_tiles = at<int32_t>(ws, L.num_tiles);
  if (routed_bs(dr)) {
    const BsBufs b{at<uint8_t>(ws, L.xq), at<uint8_t>(ws, L.sfx), at<void>(ws, L.h), at<uint8_t>(ws, L.hq),
                   at<uint8_t>(ws, L.sfh)};
    if ((st = stage_quant_mx(dr, x_rows, n_rows, nullptr, table, n_tiles, L.max_tiles, d->L, b.xq, b.sfx, 180, s)) !=
        MOE_OK)
      return st;
    return run_routed_bs_after_quant(dr, *w, b, n_rows, table, n_tiles, L.max_tiles, y_rows, s, [](int, int) {});
  }
  st = stage_expert_gate_up(dr, *w, x_rows, table, n_tiles, at<void>(ws, L.h), s, L.max_tiles);
  if (st != MOE_OK) return st;
  return stage_expert_down(dr, *w, at<void>(ws, L.h), table, n_tiles, y_rows, s, L.max_tiles);
}

moe_status moe_mx8_quantize(const void* x, int64_t rows, int32_t K, uint8_t* codes, uint8_t* scales,
                            moe_stream_t stream) {
  return mx_quantize_rows(false, x, rows, K, codes, scales, stream, 182);
}

moe_status moe_mx4_quantize(const void* x, int64_t rows, int32_t K, uint8_t* codes, uint8_t* scales,
                            moe_stream_t stream) {
  return mx_quantize_rows(true, x, rows, K, codes, scales, stream, 183);
}

moe_status moe_gather_rows(const void* src, int64_t src_rows, int64_t row_bytes, const int32_t* idx, int64_t n,
                           void* dst, moe_stream_t stream) {
  if (src_rows < 0 || n < 0 || row_bytes <= 0 || row_bytes % 16 != 0 || row_bytes / 16 > 0x7fffffffLL)
    return MOE_ERR_INVALID_ARG;
  if (n > 0x7fffffffLL * GATHER_WARPS) return MOE_ERR_INVALID_ARG;
  g_last_launches = 0;
  if (n == 0) return MOE_OK;
  if (src == nullptr || idx == nullptr || dst == nullptr || !aligned16(src) || !aligned16(dst))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  gather_rows_idx_kernel<<<static_cast<unsigned>(cdiv(n, GATHER_WARPS)), GATHER_WARPS * 32, 0, s>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), idx, n, src_rows, static_cast<int>(row_bytes / 16));
  g_last_launches = 1;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_mx_tiled_scales_size(const moe_dims* d, size_t* gate_up_bytes, size_t* down_bytes) {
  if (!dims_ok(d) || gate_up_bytes == nullptr || down_bytes == nullptr) return MOE_ERR_INVALID_ARG;
  if (d->L % 512 != 0 || d->I % 512 != 0) return MOE_ERR_UNSUPPORTED;
  *gate_up_bytes = tiled_scales_gate_up(*d);
  *down_bytes = tiled_scales_down(*d);
  return MOE_OK;
}

moe_status moe_mx_tile_scales(const moe_dims* d, const uint8_t* Sg, const uint8_t* Sv, const uint8_t* So,
                              uint8_t* Sgv_tiled, uint8_t* So_tiled, moe_stream_t stream) {
  if (!dims_ok(d)) return MOE_ERR_INVALID_ARG;
  if (d->L % 512 != 0 || d->I % 512 != 0) return MOE_ERR_UNSUPPORTED;
  const void* ptrs[] = {Sg, Sv, So, Sgv_tiled, So_tiled};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  g_last_launches = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long n_gu = static_cast<long long>(tiled_scales_gate_up(*d));
  const long long n_dn = static_cast<long long>(tiled_scales_down(*d));
  const int grid = 4 * num_sms();
  mx_tile_weight_scales_kernel<<<grid, 256, 0, s>>>(Sg, Sv, d->I, d->L, 1, n_gu, Sgv_tiled);
  mx_tile_weight_scales_kernel<<<grid, 256, 0, s>>>(So, nullptr, d->L, d->I, 0, n_dn, So_tiled);
  g_last_launches = 2;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

size_t moe_backward_workspace_size(const moe_dims* d) {
  if (!dims_ok(d)) return 0;
  return bw_layout(*d).total;
}

moe_status moe_layer_backward(const moe_dims* d, const moe_weights* w, const void* x, const float* dy,
                              const int32_t* topk_idx, const moe_grads* g, void* ws, size_t ws_bytes,
                              moe_stream_t stream) {
  moe_status st = check_dims(d);
  if (st != MOE_OK) return st;
  if (d->routed != d->act) return MOE_ERR_UNSUPPORTED;
  if (w == nullptr || g == nullptr || x == nullptr || dy == nullptr || topk_idx == nullptr) return MOE_ERR_INVALID_ARG;
  const void* need[] = {w->Wr, w->Wdown, w->Wup, w->gamma, w->Wg, w->Wv, w->Wo, x, dy, topk_idx,
                        g->dx, g->dWr, g->dWdown, g->dWup, g->dgamma, g->dWg, g->dWv, g->dWo};
  for (const void* q : need)
    if (q == nullptr || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  if (d->S > 0) {
    const void* sh[] = {w->Wsg, w->Wsv, w->Wso, g->dWsg, g->dWsv, g->dWso};
    for (const void* q : sh)
      if (q == nullptr || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  }
  const BwLayout L = bw_layout(*d);
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 || ws_bytes < L.total)
    return MOE_ERR_INVALID_ARG;
  if (d->T > 0x7fffffffLL / (d->H > d->E ? d->H : d->E)) return MOE_ERR_UNSUPPORTED;
  g_last_launches = 0;
  if (d->T == 0) return MOE_OK;
  return run_backward(*d, *w, x, dy, topk_idx, *g, ws, reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_selftest_wait_timeout(int32_t limit_ms, unsigned long long* waited_ns, moe_stream_t stream) {
  if (limit_ms < 1 || limit_ms > 2000 || waited_ns == nullptr) return MOE_ERR_INVALID_ARG;
  wait_timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_ms) * 1000000ull, MOE_FAULT_SELFTEST_WAIT, waited_ns);
  g_last_launches = 1;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_device_error(int* code, moe_stream_t stream) {
  if (code == nullptr) return MOE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_moe_fault, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  *code = v;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_moe_fault, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_ERR_DEVICE;
  }
  return MOE_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------------
// Allocation-free dispatch: moe_permute_noalloc.
//
// Some callers cannot allocate device memory at the point where they route
// tokens: code running inside a custom allocator or memory-pool callback, a
// runtime that forbids cudaMalloc after start-up so its memory footprint stays
// fixed, or a host that hands this library its inputs and outputs but owns no
// allocator of its own.  This variant keeps its scratch (per-tile expert
// counts and in-tile ranks) in a file-scope device array instead of a caller
// workspace.  The array is part of the library image: every GPU that
// loads the library holds it until the process exits.
namespace moe {
namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(MOE_PERMUTE_NOALLOC_SCRATCH_BYTES);
static __device__ __align__(256) uint8_t g_permute_scratch[kNoAllocScratchBytes];

struct NoAllocLayout {
  size_t tile_base, rank, total;
};

NoAllocLayout noalloc_layout(const moe_dims& d) {
  NoAllocLayout l{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += round_up(bytes, kAlign);
    return o;
  };
  const size_t T = static_cast<size_t>(d.T), R = T * d.k;
  l.tile_base = take(static_cast<size_t>(cdiv(d.T, PERM_TILE)) * d.E * 4);
  l.rank = take(R * 4);
  l.total = off;
  return l;
}

// Device address of g_permute_scratch in the current context.  The host-side
// name of a __device__ array is only a stand-in, so the address is asked for
// with the device current and cached per device together with the context it
// belongs to; a different current context (after cudaDeviceReset, or a
// context the caller created) makes it ask again.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
  return fn;
}

struct NoAllocCache {
  CUcontext ctx;
  void* ptr;
};
std::mutex g_noalloc_mu;
NoAllocCache g_noalloc[128] = {};

moe_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return MOE_ERR_CUDA;
  CtxGetCurrentFn ctx_fn = ctx_get_current_fn();
  if (ctx_fn == nullptr) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  CUcontext ctx = nullptr;
  if (ctx_fn(&ctx) != CUDA_SUCCESS) return MOE_ERR_CUDA;
  NoAllocCache& c = g_noalloc[dev];
  if (c.ptr == nullptr || ctx == nullptr || c.ctx != ctx) {
    // The first runtime call with the device current creates its primary
    // context if needed; the context is read again after it.
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    if (ctx_fn(&ctx) != CUDA_SUCCESS || ctx == nullptr) return MOE_ERR_CUDA;
    c.ctx = ctx;
    c.ptr = p;
  }
  *out = c.ptr;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_permute_noalloc(const moe_dims* d, const int32_t* topk_idx, const void* z,
                                          int32_t* expert_offsets, int32_t* perm_token, int32_t* inv_perm,
                                          void* z_perm, moe_stream_t stream) {
  moe_status st = check_dims(d);
  if (st != MOE_OK) return st;
  if (topk_idx == nullptr || expert_offsets == nullptr || perm_token == nullptr || inv_perm == nullptr)
    return MOE_ERR_INVALID_ARG;
  if ((z == nullptr) != (z_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  if (z != nullptr && (!aligned16(z) || !aligned16(z_perm))) return MOE_ERR_INVALID_ARG;
  const NoAllocLayout L = noalloc_layout(*d);
  if (L.total > kNoAllocScratchBytes) return MOE_ERR_INVALID_ARG;  // more scratch than the fixed array holds
  g_last_launches = 0;
  if (d->T == 0) return MOE_OK;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // Every scratch word the kernels read is written earlier in the same call,
  // so nothing has to be cleared between calls.
  const long long ntiles = cdiv(d->T, PERM_TILE);
  int32_t* tile_base = at<int32_t>(scratch, L.tile_base);
  int32_t* rank = at<int32_t>(scratch, L.rank);
  perm_rank_kernel<<<static_cast<unsigned>(ntiles), PERM_TILE, static_cast<size_t>(d->E) * 16, s>>>(
      topk_idx, d->T, d->E, d->k, tile_base, rank);
  // no grouped GEMM follows, so no tile table is built
  perm_scan_kernel<<<1, 1024, 0, s>>>(tile_base, static_cast<int>(ntiles), d->E, nullptr, expert_offsets,
                                      expert_tile_rows(*d), nullptr, nullptr);
  const long long pairs = d->T * d->k;
  perm_scatter_kernel<<<static_cast<unsigned>(cdiv(pairs, 256)), 256, 0, s>>>(
      topk_idx, d->T, d->E, d->k, tile_base, rank, expert_offsets, perm_token, inv_perm);
  g_last_launches = 3;
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  if (z != nullptr) st = stage_gather(*d, z, z_perm, perm_token, expert_offsets + d->E, s);
  return st;
}

extern "C" moe_status moe_qb_bias_update(const moe_dims* d, const float* scores, const float* bias_in, float* bias_out,
                                         float* quantile_out, uint32_t* hist, int32_t nbins, float lo, float hi,
                                         moe_stream_t stream) {
  using namespace moe;
  if (d == nullptr || scores == nullptr || bias_in == nullptr || bias_out == nullptr || hist == nullptr)
    return MOE_ERR_INVALID_ARG;
  const long long T = d->T;
  const int E = d->E, k = d->k;
  if (T < 1 || E < 2 || E > 1024 || k < 1 || k >= E) return MOE_ERR_INVALID_ARG;
  const long long c = T * k / E;
  if (c < 1 || c >= T) return MOE_ERR_INVALID_ARG;
  if (nbins < 32 || nbins > 65536 || nbins % 32 != 0) return MOE_ERR_INVALID_ARG;
  if (!(lo < hi) || !std::isfinite(lo) || !std::isfinite(hi) || !std::isfinite(hi - lo)) return MOE_ERR_INVALID_ARG;
  auto al4 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; };
  if (!al4(scores) || !al4(bias_in) || !al4(bias_out) || !al4(hist) || (quantile_out && !al4(quantile_out)))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const double span = static_cast<double>(hi) - static_cast<double>(lo);
  const float inv_w = static_cast<float>(nbins / span);
  const float w = static_cast<float>(span / nbins);
  const long long n = static_cast<long long>(E) * nbins;
  qb_zero_kernel<<<static_cast<unsigned>(std::min<long long>(cdiv(n, 256), 1184)), 256, 0, s>>>(hist, n);
  qb_hist_kernel<<<static_cast<unsigned>(cdiv(T, QB_WARPS)), QB_WARPS * 32, 0, s>>>(scores, bias_in, T, E, k, nbins,
                                                                                      lo, inv_w, hist);
  qb_quantile_kernel<<<E, 32, 0, s>>>(hist, E, nbins, c, lo, w, bias_in, bias_out, quantile_out);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
