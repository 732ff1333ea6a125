// Block-scaled grouped routed-expert GEMM for sm_100a: MXFP4 weights times
// MXFP8 activations on tcgen05.mma kind::mxf8f6f4, or times MXFP4
// activations on kind::mxf4 (template flag A4); the tensor cores apply both
// operands' E8M0 block scales, no decode pass.
//
//   D[w, t] = sum_k (Wq[w, k] * 2^(sw[w, k/32] - 127)) * (Xq[t, k] * 2^(sx[t, k/32] - 127))
//
// Same work decomposition and operand swap as gemm_expert.cuh (weight rows are
// the MMA's M on a 2-CTA pair, M = 256; token rows its N), with these
// differences (as written for MXFP8 inputs; MXFP4 inputs below):
//  * a stage covers K = 256 (two 128-wide halves, 8 MMAs of K = 32).  The MMA
//    issue is single-threaded and each barrier wait costs it a few hundred
//    cycles (measured on B200: ~250 cycles per mbarrier check and ~50 per
//    tcgen05 instruction, against 64 cycles of tensor time for an N = 128
//    MMA at the fp8 rate), so one wait and one commit per 8 MMAs;
//  * the weight tile is loaded from the packed E2M1 codes with the TMA type
//    that spreads 16 codes over 16 bytes of shared memory (8 bytes of codes,
//    8 bytes of gap), the operand layout this MMA kind reads for 4-bit types;
//    its completion count is the packed size (64 bytes per row);
//  * the activation tile is E4M3 codes, one byte each;
//  * per stage both CTAs also load their weight rows' scale atoms (1 KB) and
//    the whole token tile's scale atoms (2 KB: each CTA's half of the
//    accumulator needs the scales of every token column).  A copier warp (warp
//    6 of the even CTA) moves them to tensor memory with tcgen05.cp
//    (cta_group::2: each CTA from its own shared memory) into one of three scale
//    buffers and commits to the stage's scale barrier, on which the MMA thread
//    waits instead of the data barrier; so the MMA thread issues MMAs only;
//  * token tiles hold at most 208 rows, so two accumulators (2 x 208 fp32
//    columns) and three scale buffers (3 x 24) fit the 512 columns of tensor
//    memory; with three, the copier can put stage g's scales in the tensor
//    pipe's queue ahead of stage g-1's MMAs.
// With A4 both operands are packed E2M1 codes (two per byte, the even
// element in the low nibble), which kind::mxf4 reads as they are: a 128-byte
// wide box (plain byte TMA, 128-byte swizzle) holds K = 256, and a stage
// covers K = 512 in two such slices, 8 MMAs of K = 64, each taking two scale
// bytes (j = 0 or 2) of one 128-wide K chunk's scale columns, so that a
// stage again carries 8 MMAs per wait and commit (measured on B200 at the K3
// shape, K = 256 and K = 512 stages gave the same time: the data path, not the
// single-thread roles, bounds this kernel).  Its token box is at most 104
// rows per CTA (the tile's half), so that three stages fit; its four chunks'
// scales take 48 tensor-memory columns per buffer, so two buffers.
// Warp roles: 0 TMA producer (both CTAs), 1 TMEM owner and MMA issuer (even
// CTA), 2-5 and 7-10 epilogue (both CTAs), 6 scale copier (even CTA).  The
// two epilogue sets of four warps (one per tensor-memory lane quarter each)
// drain alternate 32-token chunks of an accumulator: measured on B200, one set
// left the MMA waiting for accumulators (the SiTU epilogue's latency per chunk
// exceeded the next item's MMA and load time).  Every wait is bounded.
#pragma once

#include "gemm_expert.cuh"
#include "mx_quant.cuh"

namespace moe {

constexpr uint32_t BS_SLICE_BYTES = 128 * 128;    // 128 weight rows x one 128-byte wide slice of K
constexpr int BS_MAX_TILE_ROWS = 208;              // largest token tile (MMA N)
constexpr uint32_t BS_ACC_COLS = BS_MAX_TILE_ROWS;
constexpr uint32_t BS_SF_COL = 2 * BS_ACC_COLS;    // the scale buffers from here
constexpr int BS_THREADS = 352;
constexpr int BS_COPY_WARP = 6;
constexpr int BS_EPI_SET1_WARP = 7;                // warps 7-10: the second epilogue set

// Stage geometry.  A stage is two 128-byte wide K slices per operand (A8: K =
// 128 E4M3 codes, or E2M1 codes spread one per byte, per slice; A4: K = 256
// packed E2M1 codes per slice), four MMAs per slice, and the scales of its
// 128-wide K chunks (A8: 2, A4: 4): per chunk one 512-byte atom of the CTA's
// weight rows and two of the token tile's rows (0-127, 128-255).  In a scale
// buffer chunk q's weight scales sit at column +4q and its token scales at
// +SFB_COL + 8q (rows 128-255 at +4 more).
template <bool A4>
struct BsStage {
  static constexpr int K = A4 ? 512 : 256;                  // K elements per stage
  static constexpr int CHUNKS = K / 128;                    // 128-wide K chunks (scale atoms) per stage
  static constexpr uint32_t A_BYTES = 2 * BS_SLICE_BYTES;   // 128 weight rows
  static constexpr uint32_t A_TX = 128 * K / 2;             // bytes the A tile's TMA completes (packed codes)
  static constexpr int B_MAX_ROWS = A4 ? 104 : 128;         // token rows of this CTA's largest box
  static constexpr uint32_t B_SLICE = B_MAX_ROWS * 128;     // (a multiple of 1024: the swizzle atom)
  static constexpr uint32_t B_BYTES = 2 * B_SLICE;
  static constexpr uint32_t SFA_BYTES = CHUNKS * 512;
  static constexpr uint32_t SFB_BYTES = CHUNKS * 1024;
  static constexpr int STAGES = 3;
  static constexpr int SF_BUFS = A4 ? 2 : 3;
  static constexpr uint32_t SFB_COL = 4 * CHUNKS;
  static constexpr uint32_t SF_BUF_COLS = 12 * CHUNKS;
  static constexpr uint32_t BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(STAGES) * BYTES + EX_XCH_BYTES + 512;
  static_assert(SMEM <= 232448, "shared memory per CTA");
  static_assert(B_SLICE % 1024 == 0, "token slices start on a swizzle atom");
  static_assert(2 * B_MAX_ROWS >= BS_MAX_TILE_ROWS, "a CTA's box covers its half of the largest tile");
  static_assert(BS_SF_COL + SF_BUFS * SF_BUF_COLS <= 2 * EX_ACC_COLS, "tensor memory columns");
  static_assert(STAGES >= SF_BUFS, "the scale copier's reuse wait assumes a stage per scale buffer at least");
};

struct BsMaps {
  CUtensorMap a0;    // E2M1 codes (A8: 16 per 16-byte slot; A4: packed bytes, 128-byte wide boxes):
                     //   PAIRED W_g [E*I, L] (64-row boxes), else W_o [E*L, I] (128-row)
  CUtensorMap a1;    // PAIRED: W_v, as a0
  CUtensorMap sa;    // weight scale tiles as [n, 16] bytes, boxes of a stage's atoms (SFA_BYTES)
  CUtensorMap b[4];  // activation codes (A8: E4M3 [R, K]; A4: packed E2M1 [R, K/2] bytes): 128-byte
                     //   wide boxes of B_MAX_ROWS, 64, 32, 16 rows, 128-byte swizzle
  CUtensorMap sb;    // activation scale tiles as [n, 16] bytes, boxes of a stage's atoms (SFB_BYTES)
};

// Shared-memory descriptor of a scale atom for tcgen05.cp: 32 rows of 16
// bytes, no swizzle, i.e. core matrices of 8 rows x 16 bytes, 16 bytes apart
// along K (leading offset) and 128 bytes apart along the rows (stride
// offset); version 1 in bits [46, 48).
__device__ __forceinline__ uint64_t sf_atom_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(16u >> 4) << 16) |
         (static_cast<uint64_t>(128u >> 4) << 32) | (static_cast<uint64_t>(1u) << 46);
}

// Instruction descriptor of tcgen05.mma kind::mxf8f6f4 with A = E2M1 (format
// 5 in bits [7, 10)), B = E4M3 (0 in [10, 13)), both K-major, E8M0 scales
// (bit 23), N >> 3 in [17, 23), M >> 4 in [24, 29), and the byte j of the
// scale column that holds this K = 32 step's scales: A's in [29, 31), B's in
// [4, 6).
__host__ __device__ constexpr uint32_t idesc_mxf4_mxf8(int M, int N, int j) {
  return (static_cast<uint32_t>(j) << 4) | (5u << 7) | (0u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(M >> 4) << 24) | (static_cast<uint32_t>(j) << 29);
}

// kind::mxf4 with A = B = E2M1 (format 1 in [7, 10) and [10, 13)), E8M0
// scales, K = 64 per MMA: scale bytes j and j + 1 (j = 0 or 2) of the column.
__host__ __device__ constexpr uint32_t idesc_mxf4_mxf4(int M, int N, int j) {
  return (static_cast<uint32_t>(j) << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(M >> 4) << 24) | (static_cast<uint32_t>(j) << 29);
}

// 32 rows x 128 bits of shared memory -> tensor memory lanes 0-31 of every
// lane quarter (4 columns from taddr), in both CTAs of the pair.
__device__ __forceinline__ void bs_copy_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// D[tmem] (+)= (A . 2^sfa) (B . 2^sfb)^T, one 256 x N x 32 step on the pair.
__device__ __forceinline__ void bs_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                       uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// As bs_mma, one 256 x N x 64 step of kind::mxf4 (two 32-blocks per scale).
__device__ __forceinline__ void bs_mma4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                        uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane (32x32b shape, x16).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* r) {
  uint32_t* u = reinterpret_cast<uint32_t*>(r);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]), "=r"(u[8]),
        "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
      : "r"(taddr));
}

// Columns ch*32 .. ch*32+31 of the accumulator (only the first 16 when the
// tile ends within them, so that no load reaches past the tile's columns).
__device__ __forceinline__ void bs_load_chunk(uint32_t tbase, int ch, int ntok, float (&r)[32]) {
  if (ch * 32 + 16 >= ntok) {
    tmem_ld16(tbase + ch * 32, r);
#pragma unroll
    for (int i = 16; i < 32; ++i) r[i] = 0.f;
  } else {
    tmem_ld32(tbase + ch * 32, r);
  }
}

// A work item with the token tile clamped to BS_MAX_TILE_ROWS rows (a table
// built for larger tiles records `site` in the fault flag and is cut, so that
// no accumulator column outside the tile's 240 is written or read).  Every
// role decodes the same item, so all see the same clamp.
__device__ __forceinline__ ExTile bs_decode(int w, int num_tiles, int num_multi, const ExParams& p, bool report) {
  ExTile t = ex_decode(w, num_tiles, num_multi, p);
  if (t.ntok > BS_MAX_TILE_ROWS) {
    if (report) record_fault(p.fault_site + 9);
    t.ntok = BS_MAX_TILE_ROWS;
    t.n_mma = BS_MAX_TILE_ROWS;
  }
  return t;
}

template <int EPI, bool PAIRED, bool A4>
__global__ void __launch_bounds__(BS_THREADS, 1)
    tc_expert_bs_kernel(const __grid_constant__ BsMaps maps, const ExParams p) {
  constexpr int CG = 2;
  using G = BsStage<A4>;
  constexpr int kStages = G::STAGES;
  extern __shared__ uint8_t bs_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bs_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kStages * G::A_BYTES;
  uint8_t* sSA = sB + kStages * G::B_BYTES;
  uint8_t* sSB = sSA + kStages * G::SFA_BYTES;
  float* xch = reinterpret_cast<float*>(sSB + kStages * G::SFB_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(xch) + EX_XCH_BYTES);
  uint64_t* empty = full + kStages;
  uint64_t* sf_full = empty + kStages;  // the stage's scales are in tensor memory (even CTA)
  uint64_t* acc_full = sf_full + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint64_t* copy_drain = drain + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(copy_drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* epi_ok = abort + 1;  // [2]: accumulator-ready verdict of each epilogue set

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_full[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 8 * CG);  // both epilogue sets' warps, in both CTAs
    }
    mbar_init(drain, 1);
    mbar_init(copy_drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.a0);
    if (PAIRED) tma_prefetch_desc(&maps.a1);
    tma_prefetch_desc(&maps.sa);
    for (int i = 0; i < 4; ++i) tma_prefetch_desc(&maps.b[i]);
    tma_prefetch_desc(&maps.sb);
  }
  if (warp == 1) ex_tmem_alloc<CG>(tmem_holder);
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int num_tiles = p.num_tiles_dev[0];
  const int num_multi = p.num_tiles_dev[1];
  const int total = num_tiles * p.n_wtiles;
  const int n_stages = p.num_k_blocks;  // stages of K = 256 per item
  const int nkb128 = G::CHUNKS * p.num_k_blocks;  // 128-wide K chunks per row (scale-tile indexing)

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0u, issued_parity = 0u;
      bool ok = true;
      const uint64_t pol_w = l2_policy_evict_first(), pol_t = l2_policy_evict_last();
      for (int w = pair; w < total && ok; w += npairs) {
        const ExTile t = bs_decode(w, num_tiles, num_multi, p, true);
        const int rows_cta = t.n_mma / 2;  // token rows this CTA stages
        const int bsel = rows_cta > 64 ? 0 : rows_cta > 32 ? 1 : rows_cta > 16 ? 2 : 3;
        const int brows = bsel == 0 ? G::B_MAX_ROWS : 128 >> bsel;
        const int tok0 = t.row0 + static_cast<int>(rank) * rows_cta;
        const uint32_t bytes = static_cast<uint32_t>(CG) * (G::A_TX + 2u * static_cast<uint32_t>(brows) * 128u +
                                                            G::SFA_BYTES + G::SFB_BYTES);
        const int wrow = t.expert * p.w_rows_per_expert + (PAIRED ? t.wt * 128 : t.wt * 256) +
                         static_cast<int>(rank) * (PAIRED ? 64 : 128);
        // 16-byte rows of the scale tiles: 32 per atom
        const int sa_row0 = ((t.expert * p.n_wtiles + t.wt) * 2 + static_cast<int>(rank)) * nkb128 * 32;
        const int sb_row0 = t.tt * nkb128 * 64;
        for (int kb = 0; kb < n_stages; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort, p.fault_site + 1)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[stage], bytes);
          uint8_t* a_dst = sA + stage * G::A_BYTES;
          uint8_t* b_dst = sB + stage * G::B_BYTES;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            // slice h: x = 128 E4M3 codes / spread E2M1 codes (A8) or 128
            // bytes of packed E2M1 codes (A4), 256 per stage either way
            const int kc = kb * 256 + h * 128;
            uint8_t* ah = a_dst + h * BS_SLICE_BYTES;
            if (kExL2Hints && !t.multi) {
              ex_tma_load_hint<CG>(ah, &maps.a0, &full[stage], kc, wrow, pol_w);
              if (PAIRED) ex_tma_load_hint<CG>(ah + BS_SLICE_BYTES / 2, &maps.a1, &full[stage], kc, wrow, pol_w);
            } else {
              ex_tma_load<CG>(ah, &maps.a0, &full[stage], kc, wrow);
              if (PAIRED) ex_tma_load<CG>(ah + BS_SLICE_BYTES / 2, &maps.a1, &full[stage], kc, wrow);
            }
            ex_tma_load_hint<CG>(b_dst + h * G::B_SLICE, &maps.b[bsel], &full[stage], kc, tok0, pol_t);
          }
          ex_tma_load<CG>(sSA + stage * G::SFA_BYTES, &maps.sa, &full[stage], 0, sa_row0 + kb * (G::SFA_BYTES / 16));
          ex_tma_load<CG>(sSB + stage * G::SFB_BYTES, &maps.sb, &full[stage], 0, sb_row0 + kb * (G::SFB_BYTES / 16));
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // The even CTA's barriers count both CTAs' bytes: it waits for every
      // load of the pair to land before the pair may exit.
      if (leader) {
        volatile int never = 0;
        for (int s = 0; s < kStages; ++s)
          if ((issued >> s) & 1u) mbar_wait(&full[s], (issued_parity >> s) & 1u, &never, p.fault_site + 2);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t g = 0;  // stages consumed so far
      uint32_t sf_buf = 0;  // scale buffer of stage g (g mod SF_BUFS)
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int w = pair; w < total && ok; w += npairs) {
        const ExTile t = bs_decode(w, num_tiles, num_multi, p, false);
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort, p.fault_site + 3)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc) * BS_ACC_COLS;
        const uint32_t idesc0 = A4 ? idesc_mxf4_mxf4(256, t.n_mma, 0) : idesc_mxf4_mxf8(256, t.n_mma, 0);
        for (int kb = 0; kb < n_stages; ++kb, ++g) {
          if (!mbar_wait(&sf_full[stage], phase, abort, p.fault_site + 4)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sf = tmem_base + BS_SF_COL + sf_buf * G::SF_BUF_COLS;
          if (++sf_buf == G::SF_BUFS) sf_buf = 0;
          const uint32_t a_addr = smem_u32(sA + stage * G::A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * G::B_BYTES);
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              // MMA kk of slice h starts 32 bytes into the slice per step.  A8:
              // K = 32, the 32-block kk of chunk h (scale byte kk).  A4: K = 64,
              // 32-blocks 2 (kk % 2), +1 of chunk 2h + kk / 2 (bytes j, j + 1).
              const uint32_t q = A4 ? 2u * h + (kk >> 1) : static_cast<uint32_t>(h);
              const uint32_t j = A4 ? 2u * (kk & 1) : static_cast<uint32_t>(kk);
              const uint32_t id = idesc0 | (j << 4) | (j << 29);
              const uint64_t ad = sw128_kmajor_desc(a_addr + h * BS_SLICE_BYTES + kk * 32);
              const uint64_t bd = sw128_kmajor_desc(b_addr + h * G::B_SLICE + kk * 32);
              const uint32_t sfa = (sf + 4u * q) | (j << 30), sfb = (sf + G::SFB_COL + 8u * q) | (j << 30);
              const uint32_t accum = (kb | h | kk) != 0 ? 1u : 0u;
              if constexpr (A4)
                bs_mma4(d_tmem, ad, bd, id, sfa, sfb, accum);
              else
                bs_mma(d_tmem, ad, bd, id, sfa, sfb, accum);
            }
          ex_commit<CG>(&empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        ex_commit<CG>(&acc_full[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      ex_commit<CG>(drain);
    }
    // Both CTAs: every MMA touching this CTA's shared memory or TMEM is done.
    if (lane == 0) {
      volatile int never = 0;
      mbar_wait(drain, 0u, &never, p.fault_site + 5);
    }
    __syncwarp();
  } else if (warp == BS_COPY_WARP) {
    // ------------------------------------------------------------------ scale copier (even CTA)
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t g = 0;
      int prev2_stage = 0;        // stage of g - SF_BUFS (its MMAs used the same scale buffer)
      uint32_t prev2_phase = 0;
      uint32_t sf_buf = 0;
      bool ok = true;
      for (int w = pair; w < total && ok; w += npairs) {
        const ExTile t = bs_decode(w, num_tiles, num_multi, p, false);
        const bool two_atoms = t.n_mma > 128;
        for (int kb = 0; kb < n_stages; ++kb, ++g) {
          if (!mbar_wait(&full[stage], phase, abort, p.fault_site + 7)) {
            ok = false;
            break;
          }
          if (g >= static_cast<uint32_t>(G::SF_BUFS)) {
            if (!mbar_wait(&empty[prev2_stage], prev2_phase, abort, p.fault_site + 8)) {
              ok = false;
              break;
            }
            if (++prev2_stage == kStages) {
              prev2_stage = 0;
              prev2_phase ^= 1u;
            }
          }
          tc_fence_after();
          const uint32_t sf = tmem_base + BS_SF_COL + sf_buf * G::SF_BUF_COLS;
          if (++sf_buf == G::SF_BUFS) sf_buf = 0;
          const uint8_t* sa = sSA + stage * G::SFA_BYTES;
          const uint8_t* sb = sSB + stage * G::SFB_BYTES;
#pragma unroll
          for (int q = 0; q < G::CHUNKS; ++q) {
            bs_copy_sf(sf + 4u * q, sf_atom_desc(smem_u32(sa + q * 512)));
            bs_copy_sf(sf + G::SFB_COL + 8u * q, sf_atom_desc(smem_u32(sb + q * 1024)));
            if (two_atoms) bs_copy_sf(sf + G::SFB_COL + 4u + 8u * q, sf_atom_desc(smem_u32(sb + q * 1024 + 512)));
          }
          // the MMA thread waits on this instead of full[]: data and scales are in place
          asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                           smem_u32(&sf_full[stage]))
                       : "memory");
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                       smem_u32(copy_drain))
                   : "memory");
      volatile int never = 0;
      mbar_wait(copy_drain, 0u, &never, p.fault_site + 9);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;  // TMEM lane quarter of this warp
    const int es = warp >= BS_EPI_SET1_WARP ? 1 : 0;  // epilogue set: chunks es, es + 2, ...
    const uint32_t acc_empty_leader = map_to_rank(smem_u32(&acc_empty[0]), 0u);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int w = pair; w < total; w += npairs) {
      const ExTile t = bs_decode(w, num_tiles, num_multi, p, false);
      bool got;
      if constexpr (PAIRED) {
        // one thread of the set waits; the set's barrier before the write keeps
        // the previous verdict until every thread has read it
        epi_set_bar(es);
        if (lane == 0 && q == (es ? 3 : 2)) epi_ok[es] = mbar_wait(&acc_full[acc], acc_phase, abort, p.fault_site + 6) ? 1 : 0;
        epi_set_bar(es);
        got = epi_ok[es] != 0;
      } else {
        got = __all_sync(0xffffffffu, mbar_wait(&acc_full[acc], acc_phase, abort, p.fault_site + 6));
      }
      if (!got) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc) * BS_ACC_COLS;
      const int nch = (t.ntok + 31) >> 5;
      if constexpr (PAIRED) {
        // quarters 0,1 hold g and 2,3 hold v for intermediate columns
        // base + 32 * (q & 1) + lane; g warps form tokens 0-15 of a chunk,
        // v warps tokens 16-31, after swapping the other half through this
        // set's exchange buffer (the two warps of a column pair sync alone).
        const bool is_g = q < 2;
        const int col = t.wt * 128 + static_cast<int>(rank) * 64 + (q & 1) * 32 + lane;
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
        const float c = p.situ_c;
        const float inv_c = 1.0f / c;
        float* X = xch + es * EX_XCH_FLOATS + (q & 1) * 1024;
#pragma unroll 1
        for (int ch = es; ch < nch; ch += 2) {
          float r[32];
          bs_load_chunk(tbase, ch, t.ntok, r);
          epi_pair_bar(es, q & 1);  // the partner has read the previous chunk's half
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (is_g)
              X[i * 32 + lane] = r[16 + i];
            else
              X[512 + i * 32 + lane] = r[i];
          }
          epi_pair_bar(es, q & 1);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float g = is_g ? r[i] : X[i * 32 + lane];
            const float v = is_g ? X[512 + i * 32 + lane] : r[16 + i];
            const int tok = ch * 32 + (is_g ? 0 : 16) + i;
            if (tok < t.ntok && col < p.out_cols)
              out[static_cast<long long>(t.row0 + tok) * p.ldo + col] = __float2bfloat16_rn(situ_glu_fast(g, v, c, inv_c));
          }
        }
      } else {
        const int col = t.wt * 256 + static_cast<int>(rank) * 128 + q * 32 + lane;
        float* out = reinterpret_cast<float*>(p.out);
#pragma unroll 1
        for (int ch = es; ch < nch; ch += 2) {
          float r[32];
          bs_load_chunk(tbase, ch, t.ntok, r);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int tok = ch * 32 + i;
            if (tok < t.ntok && col < p.out_cols) out[static_cast<long long>(t.row0 + tok) * p.ldo + col] = r[i];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader + static_cast<uint32_t>(acc * sizeof(uint64_t)));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncwarp();  // reconverge lanes that skipped the single-thread roles
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    ex_tmem_dealloc<CG>(tmem_base);
  }
}

}  // namespace moe
