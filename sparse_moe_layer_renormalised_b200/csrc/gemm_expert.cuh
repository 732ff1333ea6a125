// Grouped routed-expert GEMM for sm_100a, operands swapped so that expert
// WEIGHT rows are the MMA's M dimension and TOKENS its N dimension:
//
//   D[w, t] = sum_k W_e[w, k] * X[row0 + t, k]      (accumulated in TMEM, fp32)
//
// One work item = (token tile, weight tile).  A token tile is at most 256
// consecutive rows of the expert-major activation buffer that belong to one
// expert; its MMA N is the row count rounded up to 16, so a tile wastes at
// most 15 rows (against up to 127 for 128-row M tiles over tokens).
//
// CG = 2 runs each item on a CTA pair (a 2-CTA cluster) with
// tcgen05.mma.cta_group::2 (M = 256): each CTA stages 128 weight rows and
// half of the token rows, so per SM the shared-memory traffic per MMA is two
// thirds of the 1-CTA 128x256 tile's.  Only the even CTA issues MMAs; TMA loads
// of both CTAs complete on its barrier; tcgen05.commit multicasts to both.
// CG = 1 is the same kernel on single CTAs (M = 128).
//
// PAIRED (gate/up): each CTA's 128 weight rows are 64 rows of W_g followed by
// the same 64 rows of W_v (two 64-row TMA boxes), so epilogue warps 0/1 hold g
// and warps 2/3 hold v for the same intermediate columns; per 32-token chunk
// the g and v warps of a column range swap half their values through shared
// memory and each forms SiTU-GLU for 16 of the tokens.  Otherwise (down
// projection) the 128 rows are consecutive rows of W_o and each lane stores
// one output column.
//
// MX (block-scaled weights): the weights arrive as OCP MXFP4 -- E2M1 codes,
// two per byte, and one E8M0 scale per 32 elements along K.  Each CTA loads
// its codes and scales by TMA into a local staging slot; eight converter
// warps decode them (E2M1 pair -> f16x2 in hardware, times 2^(scale-127) in
// fp32, packed to bf16, all exact) into the same 128-byte-swizzled bf16 A tile
// the tensor cores read, and the MMA is the ordinary bf16 kind::f16.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM owner and (on the even CTA)
// MMA issuer, warps 2-5 the first epilogue set, with MX warps 6-13
// converters, and the next four warps the second epilogue set (the two sets
// drain alternate 32-token chunks).  Every wait is bounded.
#pragma once

#include "activations.cuh"
#include "gemm_tc.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int EX_BK = 64;
constexpr uint32_t EX_A_BYTES = 128 * EX_BK * 2;      // 128 weight rows
constexpr uint32_t EX_B_BYTES = 128 * EX_BK * 2;      // up to 128 token rows per CTA
constexpr uint32_t EX_STAGE_BYTES = EX_A_BYTES + EX_B_BYTES;
constexpr uint32_t EX_ACC_COLS = 256;
constexpr uint32_t EX_XCH_FLOATS = 2 * 2 * 16 * 32;        // [pair][direction][token][lane]
constexpr uint32_t EX_XCH_BYTES = 2 * EX_XCH_FLOATS * 4;    // one buffer per epilogue set, 16 KB
constexpr uint32_t EX_CODES_BYTES = 128 * 32;               // MX: E2M1 codes of 128 rows x 64 K
constexpr uint32_t EX_SCALES_BYTES = 128 * 16;              // MX: E8M0 scales of 128 rows x 8 k-blocks
constexpr int EX_CONV_WARPS = 8;
// MX: converted k-blocks per proxy fence (and per release of decoded stages).
// It must divide the k-block count of every item (K is a multiple of 512, so
// any divisor of 8 does) and be below the MX stage count, so that decoding the
// batch's last k-block never waits on a stage the batch itself holds back.
constexpr int EX_CONV_BATCH = 4;

template <bool MX>
struct ExCfg {
  static constexpr int kStages = MX ? 5 : 6;
  static_assert(!MX || (kStages > EX_CONV_BATCH && 8 % EX_CONV_BATCH == 0), "MX fence batch");
  // warps: 0 producer, 1 MMA, 2-5 epilogue set 0, (MX) converters, then
  // epilogue set 1
  static constexpr int kEpi1Warp = 6 + (MX ? EX_CONV_WARPS : 0);
  static constexpr int kThreads = 32 * (kEpi1Warp + 4);
  static constexpr uint32_t kStageBytes = EX_STAGE_BYTES + (MX ? EX_CODES_BYTES + EX_SCALES_BYTES : 0u);
  static constexpr size_t kSmem = 1024 + static_cast<size_t>(kStages) * kStageBytes + EX_XCH_BYTES + 512;
};

struct ExMaps {
  CUtensorMap a0;      // PAIRED: W_g as [E*I, L], 64-row boxes; else W_o as [E*L, I], 128-row boxes
                       // (MX: the packed codes, [rows, K/2] bytes, 32-byte-wide boxes)
  CUtensorMap a1;      // PAIRED: W_v, as a0
  CUtensorMap s0;      // MX: E8M0 scales of a0's rows, [rows, K/32] bytes, 16-byte-wide boxes
  CUtensorMap s1;      // MX, PAIRED: scales of W_v
  CUtensorMap b[4];    // activations [R, K] with 128-, 64-, 32- and 16-row boxes
};

struct ExParams {
  const int4* tile_table;     // {expert, row0, ntok, 0} per token tile
  const int* num_tiles_dev;   // number of valid entries
  int n_wtiles;               // weight tiles per expert
  int w_rows_per_expert;      // I (PAIRED) or L
  int num_k_blocks;
  void* out;                  // PAIRED: bf16 h [R, I]; else fp32 y [R, L]
  long long ldo;
  int out_cols;               // I or L (output columns; bound for stores)
  float situ_c;
  int fault_site;
};

// ------------------------------------------------------------------------------ 2-CTA PTX
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

// Named barriers of the two epilogue sets (four warps each, one per
// tensor-memory lane quarter): ids 1-4 for the two warps of a column pair (g
// quarter q, v quarter q + 2) of set es, ids 5-6 for all four warps of a set
// (aligned barriers: the warp reconverges first).
__device__ __forceinline__ void epi_pair_bar(int es, int pair_q) {
  __syncwarp();
  asm volatile("bar.sync %0, 64;" ::"r"(1 + 2 * es + pair_q) : "memory");
}
__device__ __forceinline__ void epi_set_bar(int es) {
  __syncwarp();
  asm volatile("bar.sync %0, 128;" ::"r"(5 + es) : "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

template <int CG>
__device__ __forceinline__ void ex_tmem_alloc(uint32_t* holder) {
  if (CG == 2) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(holder)),
                 "r"(2 * EX_ACC_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  } else {
    tmem_alloc(holder, 2 * EX_ACC_COLS);
    tmem_relinquish();
  }
}

template <int CG>
__device__ __forceinline__ void ex_tmem_dealloc(uint32_t taddr) {
  if (CG == 2)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(2 * EX_ACC_COLS) : "memory");
  else
    tmem_dealloc(taddr, 2 * EX_ACC_COLS);
}

// TMA tile load that completes on the pair's even-CTA barrier (CG = 2) or the
// local one (CG = 1).  `bar` is the local barrier; for CG = 2 the pair bit of
// its address is cleared so both CTAs signal the even CTA's copy.
template <int CG>
__device__ __forceinline__ void ex_tma_load(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t c0, int32_t c1) {
  if (CG == 2) {
    const uint32_t mb = smem_u32(bar) & 0xFEFFFFFFu;
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
        "%3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(mb)
        : "memory");
  } else {
    tma_load_2d(dst, map, bar, c0, c1);
  }
}

// The same load with an L2 cache-eviction hint.
template <int CG>
__device__ __forceinline__ void ex_tma_load_hint(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t c0,
                                                 int32_t c1, uint64_t policy) {
  if (CG == 2) {
    const uint32_t mb = smem_u32(bar) & 0xFEFFFFFFu;
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], "
        "[%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(mb), "l"(policy)
        : "memory");
  } else {
    tma_load_2d_hint(dst, map, bar, c0, c1, policy);
  }
}

// L2 eviction hints on the expert kernels' loads: the weight rows of experts
// with a single token tile are read once and are marked evict-first, so that
// streaming them does not push out of L2 the token rows, which every weight
// tile of their group re-reads and which are marked evict-last; the weight
// rows of experts with several token tiles are re-read through L2 by each and
// keep the default policy.  (Evict-first on every weight row raised the
// gate/up kernel's DRAM reads from 60 to 65 GB at the K3 prefill shape.)
constexpr bool kExL2Hints = true;

template <int CG>
__device__ __forceinline__ void ex_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  if (CG == 2) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    tc_mma_bf16(d_tmem, adesc, bdesc, idesc, accumulate);
  }
}

// Arrive on `bar` (same offset in both CTAs of the pair for CG = 2) when the
// MMAs issued so far have completed.
template <int CG>
__device__ __forceinline__ void ex_commit(uint64_t* bar) {
  if (CG == 2) {
    const uint16_t mask = 0x3;
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::
                     "r"(smem_u32(bar)),
                 "h"(mask)
                 : "memory");
  } else {
    tc_commit(bar);
  }
}

// E8M0 scale byte -> 2^(s - 127) as fp32 (s = 0: 2^-127; s = 255: NaN).
__device__ __forceinline__ float e8m0_to_f32(uint32_t s) {
  if (s == 0u) return __int_as_float(0x00400000);
  if (s == 255u) return __int_as_float(0x7FC00000);
  return __int_as_float(static_cast<int>(s << 23));
}

// Two E2M1 codes (low nibble = element 0) times `scale`, as bf16x2.
__device__ __forceinline__ uint32_t e2m1x2_scaled_bf16x2(uint32_t byte, float scale) {
  uint32_t h2;
  asm("{\n\t.reg .b8 t;\n\tmov.b16 {t, _}, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(h2)
      : "h"(static_cast<unsigned short>(byte & 0xFFu)));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
  return pack_bf16x2(f.x * scale, f.y * scale);
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

struct ExTile {
  int expert, row0, ntok, n_mma, wt;
  int tt;      // index of the token tile in the tile table
  bool multi;  // the tile's expert has several token tiles (its weight tiles are re-read through L2)
};

// Work order: token tiles are taken in groups of EX_GROUP consecutive tiles;
// inside a group the weight tile is the outer index.  Consecutive work items
// then share a weight tile (its rows stream from HBM once per group, not once
// per token tile, when a large expert has many token tiles) while the
// group's token rows stay in L2 across the weight tiles.
#ifndef MOE_EX_GROUP
#define MOE_EX_GROUP 8
#endif
constexpr int EX_GROUP = MOE_EX_GROUP;

// Item i of a list of token tiles [t0, t0 + n) in the grouped order above.
__device__ __forceinline__ ExTile ex_decode_list(int i, int t0, int n, int num_multi, const ExParams& p) {
  const int gsize = EX_GROUP * p.n_wtiles;
  const int grp = i / gsize;
  const int r = i - grp * gsize;
  const int in_grp = min(EX_GROUP, n - grp * EX_GROUP);
  const int wt = r / in_grp;
  const int tt = t0 + grp * EX_GROUP + (r - wt * in_grp);
  ExTile t;
  t.wt = wt;
  t.tt = tt;
  t.multi = tt < num_multi;
  const int4 e = p.tile_table[tt];
  t.expert = e.x;
  t.row0 = e.y;
  t.ntok = e.z;
  t.n_mma = max(16, (t.ntok + 15) & ~15);
  return t;
}

// The tile table lists the tiles of experts with several tiles first
// (num_multi of them: their weight tiles are shared through L2 by the
// expert's token tiles) and then those of single-tile experts (weights
// streamed from DRAM once).  kExInterleave = true would interleave the two
// lists in proportion to their sizes so that items of both kinds run at the
// same time; measured at the K3 prefill shape it raised the gate/up kernel's
// DRAM reads from 58 to 68 GB and its time by 5%, so items run in list order.
constexpr bool kExInterleave = false;

__device__ __forceinline__ ExTile ex_decode(int w, int num_tiles, int num_multi, const ExParams& p) {
  if (!kExInterleave || num_multi <= 0 || num_multi >= num_tiles) return ex_decode_list(w, 0, num_tiles, num_multi, p);
  const long long total = static_cast<long long>(num_tiles) * p.n_wtiles;
  const long long n_multi = static_cast<long long>(num_multi) * p.n_wtiles;
  const int before = static_cast<int>(static_cast<long long>(w) * n_multi / total);  // multi items before w
  const bool multi = static_cast<int>((static_cast<long long>(w) + 1) * n_multi / total) > before;
  return multi ? ex_decode_list(before, 0, num_multi, num_multi, p)
               : ex_decode_list(w - before, num_multi, num_tiles - num_multi, num_multi, p);
}

template <int EPI, bool PAIRED, int CG, bool MX>
__global__ void __launch_bounds__(ExCfg<MX>::kThreads, 1)
    tc_expert_kernel(const __grid_constant__ ExMaps maps, const ExParams p) {
  constexpr int EX_STAGES = ExCfg<MX>::kStages;
  extern __shared__ uint8_t ex_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ex_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + EX_STAGES * EX_A_BYTES;
  uint8_t* sQ = sB + EX_STAGES * EX_B_BYTES;                       // MX codes
  uint8_t* sS = sQ + (MX ? EX_STAGES * EX_CODES_BYTES : 0u);       // MX scales
  float* xch = reinterpret_cast<float*>(sS + (MX ? EX_STAGES * EX_SCALES_BYTES : 0u));
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(xch) + EX_XCH_BYTES);
  uint64_t* empty = full + EX_STAGES;
  uint64_t* raw = empty + EX_STAGES;     // MX: local codes + scales landed
  uint64_t* conv = raw + EX_STAGES;      // MX: both CTAs' A tiles converted (even CTA's copy counts)
  uint64_t* acc_full = conv + EX_STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* epi_ok = abort + 1;  // [2]: accumulator-ready verdict of each epilogue set

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int pair = CG == 2 ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int npairs = CG == 2 ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < EX_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&raw[s], 1);
      mbar_init(&conv[s], CG * EX_CONV_WARPS);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 8 * CG);  // both epilogue sets' warps, in every CTA
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.a0);
    if (PAIRED) tma_prefetch_desc(&maps.a1);
    if (MX) {
      tma_prefetch_desc(&maps.s0);
      if (PAIRED) tma_prefetch_desc(&maps.s1);
    }
    for (int i = 0; i < 4; ++i) tma_prefetch_desc(&maps.b[i]);
  }
  if (warp == 1) ex_tmem_alloc<CG>(tmem_holder);
  tc_fence_before();
  if (CG == 2)
    cluster_sync_all();
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int num_tiles = p.num_tiles_dev[0];
  const int num_multi = p.num_tiles_dev[1];
  const int total = num_tiles * p.n_wtiles;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0u, issued_parity = 0u;
      bool ok = true;
      const uint64_t pol_w = l2_policy_evict_first(), pol_t = l2_policy_evict_last();
      // No separate L2 prefetch of the weight rows: on B200 the extra bulk
      // requests cost more than the latency they hide (measured, prefill
      // gate/up about 15% slower with a 12-k-block-ahead prefetch).
      auto weight_row = [&](const ExTile& t) {
        const int wrow_pair = PAIRED ? t.wt * (64 * CG) : t.wt * (128 * CG);
        return t.expert * p.w_rows_per_expert + wrow_pair + static_cast<int>(rank) * (PAIRED ? 64 : 128);
      };
      for (int w = pair; w < total && ok; w += npairs) {
        const ExTile t = ex_decode(w, num_tiles, num_multi, p);
        const int rows_cta = CG == 2 ? t.n_mma / 2 : t.n_mma;   // token rows this CTA stages
        // Staged as ONE box of 128, 64, 32 or 16 rows, the smallest that covers
        // the tile: measured on B200, a single TMA request per operand and
        // stage streams far better than several smaller ones, even though up
        // to half of the box may be rows of the next tile.
        const int bsel = rows_cta > 64 ? 0 : rows_cta > 32 ? 1 : rows_cta > 16 ? 2 : 3;
        const int brows = 128 >> bsel;
        const int tok0 = t.row0 + static_cast<int>(rank) * rows_cta;
        const uint32_t bytes = static_cast<uint32_t>(CG) * ((MX ? 0u : EX_A_BYTES) + brows * EX_BK * 2);
        const int wrow = weight_row(t);  // first weight row of this CTA
        for (int kb = 0; kb < p.num_k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort, p.fault_site + 1)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[stage], bytes);
          const int kc = kb * EX_BK;
          uint8_t* a_dst = sA + stage * EX_A_BYTES;
          uint8_t* b_dst = sB + stage * EX_B_BYTES;
          if constexpr (MX) {
            // codes and scales of this CTA's rows, to its own staging slot
            uint8_t* q_dst = sQ + stage * EX_CODES_BYTES;
            uint8_t* s_dst = sS + stage * EX_SCALES_BYTES;
            const int sc0 = (kb >> 3) * 16;  // 16 scale bytes = 8 k-blocks per box
            mbar_arrive_expect_tx(&raw[stage], EX_CODES_BYTES + EX_SCALES_BYTES);
            if (PAIRED) {
              tma_load_2d(q_dst, &maps.a0, &raw[stage], kb * 32, wrow);
              tma_load_2d(q_dst + EX_CODES_BYTES / 2, &maps.a1, &raw[stage], kb * 32, wrow);
              tma_load_2d(s_dst, &maps.s0, &raw[stage], sc0, wrow);
              tma_load_2d(s_dst + EX_SCALES_BYTES / 2, &maps.s1, &raw[stage], sc0, wrow);
            } else {
              tma_load_2d(q_dst, &maps.a0, &raw[stage], kb * 32, wrow);
              tma_load_2d(s_dst, &maps.s0, &raw[stage], sc0, wrow);
            }
          } else if (kExL2Hints && !t.multi) {
            ex_tma_load_hint<CG>(a_dst, &maps.a0, &full[stage], kc, wrow, pol_w);
            if (PAIRED) ex_tma_load_hint<CG>(a_dst + EX_A_BYTES / 2, &maps.a1, &full[stage], kc, wrow, pol_w);
          } else if (PAIRED) {
            ex_tma_load<CG>(a_dst, &maps.a0, &full[stage], kc, wrow);
            ex_tma_load<CG>(a_dst + EX_A_BYTES / 2, &maps.a1, &full[stage], kc, wrow);
          } else {
            ex_tma_load<CG>(a_dst, &maps.a0, &full[stage], kc, wrow);
          }
          if (kExL2Hints)
            ex_tma_load_hint<CG>(b_dst, &maps.b[bsel], &full[stage], kc, tok0, pol_t);
          else
            ex_tma_load<CG>(b_dst, &maps.b[bsel], &full[stage], kc, tok0);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == EX_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // The even CTA's barriers count both CTAs' bytes: it waits for every
      // load of the pair to land before the pair may exit.
      {
        volatile int never = 0;
        for (int s = 0; s < EX_STAGES; ++s) {
          if (!((issued >> s) & 1u)) continue;
          if (leader) mbar_wait(&full[s], (issued_parity >> s) & 1u, &never, p.fault_site + 2);
          if (MX) mbar_wait(&raw[s], (issued_parity >> s) & 1u, &never, p.fault_site + 2);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int w = pair; w < total && ok; w += npairs) {
        const ExTile t = ex_decode(w, num_tiles, num_multi, p);
        const uint32_t idesc = idesc_bf16_f32(128 * CG, t.n_mma);
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort, p.fault_site + 3)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * EX_ACC_COLS);
        for (int kb = 0; kb < p.num_k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort, p.fault_site + 4) ||
              (MX && !mbar_wait(&conv[stage], phase, abort, p.fault_site + 7))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * EX_A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * EX_B_BYTES);
#pragma unroll
          for (int kk = 0; kk < EX_BK / 16; ++kk)
            ex_mma<CG>(d_tmem, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32), idesc,
                       (kb | kk) != 0 ? 1u : 0u);
          ex_commit<CG>(&empty[stage]);
          if (++stage == EX_STAGES) {
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
  } else if (MX && warp >= 6 && warp < 6 + EX_CONV_WARPS) {
    // ------------------------------------------------------------------ MXFP4 converters (both CTAs)
    // thread = one 32-element MX block: row r of the A tile, K half h
    const int ct = threadIdx.x - 192;
    const int r = ct >> 1, h = ct & 1;
    const uint32_t conv_leader = CG == 2 ? map_to_rank(smem_u32(&conv[0]), 0u) : smem_u32(&conv[0]);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int w = pair; w < total && ok; w += npairs) {
      for (int kb = 0; kb < p.num_k_blocks; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(&raw[stage], phase, abort, p.fault_site + 8))) {
          ok = false;
          break;
        }
        const uint4 q = *reinterpret_cast<const uint4*>(sQ + stage * EX_CODES_BYTES + r * 32 + h * 16);
        const float sc = e8m0_to_f32(sS[stage * EX_SCALES_BYTES + r * 16 + (kb & 7) * 2 + h]);
        uint32_t o[16];
        const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) o[4 * i + j] = e2m1x2_scaled_bf16x2(words[i] >> (8 * j), sc);
        // 64 bytes = chunks 4h .. 4h+3 of row r, 128-byte swizzle
        uint8_t* arow = sA + stage * EX_A_BYTES + r * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int chunk = (4 * h + c) ^ (r & 7);
          *reinterpret_cast<uint4*>(arow + chunk * 16) = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
        }
        // The proxy fence that hands these generic-proxy writes to the tensor
        // cores is the converters' dominant stall (ncu: membar), so it is paid
        // once per EX_CONV_BATCH k-blocks, after which the batch's stages are
        // released together (measured: 1 -> 4 k-blocks per fence, MXFP4 layer
        // +19%).  The batch's last stage was freed by the MMA of a k-block of
        // an earlier batch, so holding this batch back cannot deadlock.
        if (kb % EX_CONV_BATCH == EX_CONV_BATCH - 1) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
#pragma unroll
            for (int d = EX_CONV_BATCH - 1; d >= 0; --d) {
              const int st = (stage - d + EX_STAGES) % EX_STAGES;
              if (CG == 2)
                mbar_arrive_cluster(conv_leader + static_cast<uint32_t>(st * sizeof(uint64_t)));
              else
                mbar_arrive(&conv[st]);
            }
          }
        }
        if (++stage == EX_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    // Two sets of four warps drain alternate 32-token chunks of an accumulator
    // (set es: chunks es, es + 2, ...).  Measured on B200 (prefill gate/up):
    // without the SiTU arithmetic and stores the kernel ran 13% faster, so one
    // set's drain was on the critical path.
    const int q = warp & 3;  // TMEM lane quarter of this warp
    const int es = warp >= ExCfg<MX>::kEpi1Warp ? 1 : 0;
    const uint32_t acc_empty_leader =
        CG == 2 ? map_to_rank(smem_u32(&acc_empty[0]), 0u) : smem_u32(&acc_empty[0]);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int w = pair; w < total; w += npairs) {
      const ExTile t = ex_decode(w, num_tiles, num_multi, p);
      bool got;
      if constexpr (PAIRED) {
        // One thread of the set waits; the verdict reaches the set's four warps
        // through its barrier, so they always run the same number of barriers
        // (the barrier before the write keeps the previous verdict until every
        // thread has read it).
        epi_set_bar(es);
        if (lane == 0 && q == 2) epi_ok[es] = mbar_wait(&acc_full[acc], acc_phase, abort, p.fault_site + 6) ? 1 : 0;
        epi_set_bar(es);
        got = epi_ok[es] != 0;
      } else {
        // warp-uniform decision: tcgen05.ld below needs the whole warp
        got = __all_sync(0xffffffffu, mbar_wait(&acc_full[acc], acc_phase, abort, p.fault_site + 6));
      }
      if (!got) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * EX_ACC_COLS);
      const int nch = (t.ntok + 31) >> 5;  // 32-token chunks (uniform over the epilogue warps)
      if constexpr (PAIRED) {
        // quarters 0,1 hold g and 2,3 hold v for intermediate columns
        // base + 32 * (q & 1) + lane; g warps form tokens 0-15 of a chunk,
        // v warps tokens 16-31, after swapping the other half through the
        // set's exchange buffer (the two warps of a column pair sync alone).
        const bool is_g = q < 2;
        const int col = t.wt * (64 * CG) + static_cast<int>(rank) * 64 + (q & 1) * 32 + lane;
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
        const float c = p.situ_c;
        const float inv_c = 1.0f / c;
        float* X = xch + es * EX_XCH_FLOATS + (q & 1) * 1024;
#pragma unroll 1
        for (int ch = es; ch < nch; ch += 2) {
          float r[32];
          tmem_ld32(tbase + ch * 32, r);
          epi_pair_bar(es, q & 1);  // the partner has read the previous chunk's half
          // direction 0 region carries g (tokens 16-31), direction 1 carries v (tokens 0-15)
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
        const int col = t.wt * (128 * CG) + static_cast<int>(rank) * 128 + q * 32 + lane;
        float* out = reinterpret_cast<float*>(p.out);
#pragma unroll 1
        for (int ch = es; ch < nch; ch += 2) {
          float r[32];
          tmem_ld32(tbase + ch * 32, r);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int tok = ch * 32 + i;
            if (tok < t.ntok && col < p.out_cols) out[static_cast<long long>(t.row0 + tok) * p.ldo + col] = r[i];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (CG == 2)
          mbar_arrive_cluster(acc_empty_leader + static_cast<uint32_t>(acc * sizeof(uint64_t)));
        else
          mbar_arrive(&acc_empty[acc]);
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncwarp();  // reconverge lanes that skipped the single-thread roles
  tc_fence_before();
  if (CG == 2)
    cluster_sync_all();
  else
    __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    ex_tmem_dealloc<CG>(tmem_base);
  }
}

}  // namespace moe
