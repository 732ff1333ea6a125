// Grouped routed-expert GEMM for sm_100a with TWO weight tiles per token tile
// (bf16 weights).  As in gemm_expert.cuh the operands are swapped -- expert
// weight rows are the MMA's M, tokens its N -- and one token tile is at most
// 128 * CG rows of one expert in the expert-major activation buffer.
//
// One work item = (token tile, weight-tile pair):
//   gate/up (PAIRED): the pair is the W_g rows and the W_v rows of the same
//     128 * CG intermediate columns, so TMEM lane l of accumulator 0 holds g
//     and lane l of accumulator 1 holds v for the same column: the SiTU-GLU
//     epilogue reads both with two TMEM loads and needs no exchange;
//   down projection: two consecutive 128 * CG-row tiles of W_o (the second
//     is absent when the expert's tile count is odd).
// Each stage holds both weight tiles and the token box once, so the token
// rows cross from L2 into shared memory once per weight-tile PAIR (half the
// token traffic of one tile per item), and two MMA-issuing threads (warps 1
// and 6, one accumulator each) issue the pair's MMAs side by side: one thread
// holds its MMA for ~150 cycles whatever its N, so two issuers keep the tensor
// cores busy at the token-tile heights a skewed expert load produces.
//
// CG = 2: tcgen05.mma.cta_group::2 with M = 256 (each CTA stages 128 rows of
// each weight tile and half the token rows; loads complete on the even CTA's
// barrier; commits multicast to both CTAs).  CG = 1: single CTAs, M = 128.
//
// Warp roles: 0 TMA producer; 1 TMEM owner and issuer of accumulator 0;
// 2-5 and 7-10 epilogue (two sets of four warps, one per TMEM lane quarter
// each, on alternate 32-token chunks); 6 issuer of accumulator 1.  TMEM:
// accumulator a is columns [256 a, 256 a + 256).  Both accumulators are
// single-buffered, so an item's MMAs start once the epilogue has drained the
// previous item's accumulator; the two epilogue sets halve that drain.
// Every wait is bounded.
#pragma once

#include "activations.cuh"
#include "gemm_expert.cuh"
#include "ptx.cuh"

namespace moe {

constexpr uint32_t X2_A_BYTES = 128 * EX_BK * 2;  // 128 weight rows x 64 k
constexpr uint32_t X2_B_BYTES = 128 * EX_BK * 2;  // up to 128 token rows per CTA
constexpr uint32_t X2_STAGE_BYTES = 2 * X2_A_BYTES + X2_B_BYTES;
constexpr int X2_STAGES = 4;
constexpr int X2_THREADS = 352;
constexpr int X2_EPI1_WARP = 7;  // warps 7-10: the second epilogue set
constexpr size_t X2_SMEM = 1024 + static_cast<size_t>(X2_STAGES) * X2_STAGE_BYTES + 256;

struct X2Maps {
  CUtensorMap a0;    // PAIRED: W_g as [E*I, L]; else W_o as [E*L, I]; 128-row boxes
  CUtensorMap a1;    // PAIRED: W_v as [E*I, L] (unused otherwise)
  CUtensorMap b[4];  // activations [R, K] with 128-, 64-, 32- and 16-row boxes
};

struct X2Params {
  const int4* tile_table;    // {expert, row0, ntok, 0} per token tile
  const int* num_tiles_dev;  // number of valid entries
  int n_items;               // weight-tile pairs per expert
  int n_wtiles;              // 128*CG-row weight tiles per expert (down: the second of a pair exists if < n_wtiles)
  int w_rows_per_expert;     // I (PAIRED) or L
  int num_k_blocks;
  void* out;                 // PAIRED: bf16 h [R, I]; else fp32 y [R, L]
  long long ldo;
  int out_cols;
  float situ_c;
  int fault_site;
};

struct X2Tile {
  int expert, row0, ntok, n_mma, j;
};

// Same grouped order as the one-tile kernel: groups of EX_GROUP token tiles,
// the weight-tile pair as the outer index inside a group.
__device__ __forceinline__ X2Tile x2_decode(int w, int num_tiles, const X2Params& p) {
  const int gsize = EX_GROUP * p.n_items;
  const int grp = w / gsize;
  const int r = w - grp * gsize;
  const int in_grp = min(EX_GROUP, num_tiles - grp * EX_GROUP);
  const int j = r / in_grp;
  const int tt = grp * EX_GROUP + (r - j * in_grp);
  X2Tile t;
  t.j = j;
  const int4 e = p.tile_table[tt];
  t.expert = e.x;
  t.row0 = e.y;
  t.ntok = e.z;
  t.n_mma = max(16, (t.ntok + 15) & ~15);
  return t;
}

template <int EPI, bool PAIRED, int CG>
__global__ void __launch_bounds__(X2_THREADS, 1) tc_expert2_kernel(const __grid_constant__ X2Maps maps,
                                                                   const X2Params p) {
  extern __shared__ uint8_t x2_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(x2_smem_raw) + 1023) & ~uintptr_t(1023));
  // stage s: [A0 | A1 | B]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + X2_STAGES * X2_STAGE_BYTES);
  uint64_t* empty = full + X2_STAGES;
  uint64_t* acc_full = empty + X2_STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int pair = CG == 2 ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int npairs = CG == 2 ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < X2_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 2);  // one commit from each issuer
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 8 * CG);  // both epilogue sets' warps, in every CTA
    }
    mbar_init(drain, 2);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.a0);
    if (PAIRED) tma_prefetch_desc(&maps.a1);
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

  const int num_tiles = *p.num_tiles_dev;
  const int total = num_tiles * p.n_items;
  // weight rows of this CTA for accumulator a of item j (expert-local)
  auto wrow_local = [&](int j, int a) {
    const int tile = PAIRED ? j : 2 * j + a;
    return tile * (128 * CG) + static_cast<int>(rank) * 128;
  };
  auto has_second = [&](int j) { return PAIRED || 2 * j + 1 < p.n_wtiles; };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0u, issued_parity = 0u;
      bool ok = true;
      for (int w = pair; w < total && ok; w += npairs) {
        const X2Tile t = x2_decode(w, num_tiles, p);
        const int rows_cta = CG == 2 ? t.n_mma / 2 : t.n_mma;
        const int bsel = rows_cta > 64 ? 0 : rows_cta > 32 ? 1 : rows_cta > 16 ? 2 : 3;
        const int brows = 128 >> bsel;
        const int tok0 = t.row0 + static_cast<int>(rank) * rows_cta;
        const bool two = has_second(t.j);
        const uint32_t bytes = static_cast<uint32_t>(CG) * ((two ? 2u : 1u) * X2_A_BYTES + brows * EX_BK * 2);
        const int base = t.expert * p.w_rows_per_expert;
        const int r0 = base + wrow_local(t.j, 0), r1 = base + wrow_local(t.j, 1);
        for (int kb = 0; kb < p.num_k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort, p.fault_site + 1)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[stage], bytes);
          const int kc = kb * EX_BK;
          uint8_t* st = smem + stage * X2_STAGE_BYTES;
          ex_tma_load<CG>(st, &maps.a0, &full[stage], kc, r0);
          if (PAIRED)
            ex_tma_load<CG>(st + X2_A_BYTES, &maps.a1, &full[stage], kc, r1);
          else if (two)
            ex_tma_load<CG>(st + X2_A_BYTES, &maps.a0, &full[stage], kc, r1);
          ex_tma_load<CG>(st + 2 * X2_A_BYTES, &maps.b[bsel], &full[stage], kc, tok0);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == X2_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every load of the pair lands before the pair may exit
      volatile int never = 0;
      for (int s = 0; s < X2_STAGES; ++s)
        if (leader && ((issued >> s) & 1u)) mbar_wait(&full[s], (issued_parity >> s) & 1u, &never, p.fault_site + 2);
    }
  } else if (warp == 1 || warp == 6) {
    // ------------------------------------------------------------------ MMA issuers (even CTA)
    const int a = warp == 1 ? 0 : 1;  // accumulator / weight tile of this issuer
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * EX_ACC_COLS);
      for (int w = pair; w < total && ok; w += npairs) {
        const X2Tile t = x2_decode(w, num_tiles, p);
        const bool active = a == 0 || has_second(t.j);
        const uint32_t idesc = idesc_bf16_f32(128 * CG, t.n_mma);
        if (!mbar_wait(&acc_empty[a], acc_phase ^ 1u, abort, p.fault_site + 3)) break;
        tc_fence_after();
        for (int kb = 0; kb < p.num_k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort, p.fault_site + 4)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (active) {
            const uint8_t* st = smem + stage * X2_STAGE_BYTES;
            const uint32_t a_addr = smem_u32(st + a * X2_A_BYTES);
            const uint32_t b_addr = smem_u32(st + 2 * X2_A_BYTES);
#pragma unroll
            for (int kk = 0; kk < EX_BK / 16; ++kk)
              ex_mma<CG>(d_tmem, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32), idesc,
                         (kb | kk) != 0 ? 1u : 0u);
          }
          ex_commit<CG>(&empty[stage]);  // counts even without MMAs of this issuer
          if (++stage == X2_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        ex_commit<CG>(&acc_full[a]);
        acc_phase ^= 1u;
      }
      ex_commit<CG>(drain);
    }
    // Both CTAs: every MMA touching this CTA's shared memory or TMEM is done.
    if (warp == 1 && lane == 0) {
      volatile int never = 0;
      mbar_wait(drain, 0u, &never, p.fault_site + 5);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2-5, 7-10, both CTAs)
    const int q = warp & 3;  // TMEM lane quarter of this warp
    const int es = warp >= X2_EPI1_WARP ? 1 : 0;  // epilogue set: chunks es, es + 2, ...
    const uint32_t acc_empty_leader =
        CG == 2 ? map_to_rank(smem_u32(&acc_empty[0]), 0u) : smem_u32(&acc_empty[0]);
    uint32_t acc_phase = 0;
    auto release = [&](int a) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (CG == 2)
          mbar_arrive_cluster(acc_empty_leader + static_cast<uint32_t>(a * sizeof(uint64_t)));
        else
          mbar_arrive(&acc_empty[a]);
      }
    };
    for (int w = pair; w < total; w += npairs) {
      const X2Tile t = x2_decode(w, num_tiles, p);
      const int nch = (t.ntok + 31) >> 5;  // 32-token chunks
      const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      if constexpr (PAIRED) {
        // warp-uniform decisions: tcgen05.ld below needs the whole warp
        if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[0], acc_phase, abort, p.fault_site + 6))) break;
        if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[1], acc_phase, abort, p.fault_site + 7))) break;
        tc_fence_after();
        const int col = wrow_local(t.j, 0) + q * 32 + lane;  // intermediate column of this lane
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
        const float c = p.situ_c;
        const float inv_c = 1.0f / c;
#pragma unroll 1
        for (int ch = es; ch < nch; ch += 2) {
          float g[32], v[32];
          tmem_ld32(lane_base + ch * 32, g);
          tmem_ld32(lane_base + EX_ACC_COLS + ch * 32, v);
          const long long r0 = static_cast<long long>(t.row0 + ch * 32);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (ch * 32 + i < t.ntok && col < p.out_cols)
              out[(r0 + i) * p.ldo + col] = __float2bfloat16_rn(situ_glu_fast(g[i], v[i], c, inv_c));
          }
        }
        release(0);
        release(1);
      } else {
        float* out = reinterpret_cast<float*>(p.out);
        bool ok = true;
        for (int a = 0; a < 2 && ok; ++a) {
          if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[a], acc_phase, abort, p.fault_site + 6 + a))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (a == 0 || has_second(t.j)) {
            const int col = wrow_local(t.j, a) + q * 32 + lane;
#pragma unroll 1
            for (int ch = es; ch < nch; ch += 2) {
              float r[32];
              tmem_ld32(lane_base + a * EX_ACC_COLS + ch * 32, r);
              const long long r0 = static_cast<long long>(t.row0 + ch * 32);
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (ch * 32 + i < t.ntok && col < p.out_cols) out[(r0 + i) * p.ldo + col] = r[i];
            }
          }
          release(a);
        }
        if (!ok) break;
      }
      acc_phase ^= 1u;
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
