/*
 * Host half of the seeded synthetic-input generator (C, pthreads).
 * Compiled with -ffp-contract=off so that value = centred * scale + offset
 * is one rounded multiply followed by one rounded add, exactly as on the
 * device half.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#include "gen_common.h"

void gen_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  gen_philox4x32_10_impl(ctr, key, out);
}

/* fp32 scale that maps a centred Irwin-Hall(8) sum of 16-bit uniforms to a
 * variate of standard deviation std.  Var of one 16-bit uniform integer is
 * (65536^2 - 1) / 12, so the sum of eight has standard deviation
 * 65536 * sqrt(2/3) * sqrt(1 - 2^-32). */
float gen_scale(double std) {
  double sd_sum = 65536.0 * sqrt(2.0 / 3.0) * sqrt(1.0 - 1.0 / 4294967296.0);
  return (float)(std / sd_sum);
}

static inline float gen_value(uint32_t seed, uint32_t tid, uint64_t index, float scale, float offset) {
  float c = (float)gen_ih8_centred(seed, tid, index);
  float v = c * scale;
  return v + offset;
}

typedef struct {
  uint32_t seed, tid;
  uint64_t start, count;
  float scale, offset;
  void* out;
  int kind; /* 0 = f32, 1 = bf16, 2 = mxfp4 rows */
  uint64_t K;  /* mxfp4: row length */
  uint8_t* scales;
} gen_job;

static void run_range(const gen_job* j, uint64_t lo, uint64_t hi) {
  if (j->kind == 0) {
    float* o = (float*)j->out;
    for (uint64_t i = lo; i < hi; ++i) o[i] = gen_value(j->seed, j->tid, j->start + i, j->scale, j->offset);
  } else if (j->kind == 1) {
    uint16_t* o = (uint16_t*)j->out;
    for (uint64_t i = lo; i < hi; ++i)
      o[i] = gen_f32_to_bf16_bits(gen_value(j->seed, j->tid, j->start + i, j->scale, j->offset));
  } else {
    /* rows [lo, hi) relative to row start; start is the first row */
    uint8_t* codes = (uint8_t*)j->out;
    uint64_t K = j->K;
    float blk[32];
    for (uint64_t r = lo; r < hi; ++r) {
      uint64_t row = j->start + r;
      for (uint64_t b = 0; b < K / 32; ++b) {
        for (int i = 0; i < 32; ++i) blk[i] = gen_value(j->seed, j->tid, row * K + b * 32 + (uint64_t)i, j->scale, 0.0f);
        j->scales[r * (K / 32) + b] = gen_mxfp4_block(blk, codes + r * (K / 2) + b * 16);
      }
    }
  }
}

typedef struct {
  const gen_job* job;
  uint64_t lo, hi;
} gen_slice;

static void* slice_main(void* p) {
  gen_slice* s = (gen_slice*)p;
  run_range(s->job, s->lo, s->hi);
  return NULL;
}

static void run_parallel(const gen_job* j, uint64_t n, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((uint64_t)nthreads > n) nthreads = (int)(n > 0 ? n : 1);
  if (nthreads == 1) {
    run_range(j, 0, n);
    return;
  }
  pthread_t th[256];
  gen_slice sl[256];
  uint64_t per = (n + (uint64_t)nthreads - 1) / (uint64_t)nthreads;
  int launched = 0;
  for (int t = 0; t < nthreads; ++t) {
    uint64_t lo = per * (uint64_t)t, hi = lo + per;
    if (lo >= n) break;
    if (hi > n) hi = n;
    sl[t].job = j;
    sl[t].lo = lo;
    sl[t].hi = hi;
    if (pthread_create(&th[t], NULL, slice_main, &sl[t]) != 0) {
      run_range(j, lo, hi);
      sl[t].job = NULL;
    }
    launched = t + 1;
  }
  for (int t = 0; t < launched; ++t)
    if (sl[t].job) pthread_join(th[t], NULL);
}

/* out[i] = offset + N(0, std) for element indices start .. start+count-1 */
void gen_fill_f32(uint32_t seed, uint32_t tid, uint64_t start, uint64_t count, float scale, float offset,
                  float* out, int nthreads) {
  gen_job j;
  memset(&j, 0, sizeof j);
  j.seed = seed;
  j.tid = tid;
  j.start = start;
  j.count = count;
  j.scale = scale;
  j.offset = offset;
  j.out = out;
  j.kind = 0;
  run_parallel(&j, count, nthreads);
}

/* Same values rounded to bf16 (RNE), written as raw 16-bit patterns. */
void gen_fill_bf16(uint32_t seed, uint32_t tid, uint64_t start, uint64_t count, float scale, float offset,
                   uint16_t* out, int nthreads) {
  gen_job j;
  memset(&j, 0, sizeof j);
  j.seed = seed;
  j.tid = tid;
  j.start = start;
  j.count = count;
  j.scale = scale;
  j.offset = offset;
  j.out = out;
  j.kind = 1;
  run_parallel(&j, count, nthreads);
}

/* MXFP4 rows row_start .. row_start+nrows-1 of a [rows, K] tensor whose
 * unquantised element (r, k) is the N(0, std) variate of index r*K + k.
 * codes: [nrows, K/2] bytes; scales: [nrows, K/32] E8M0 bytes. K % 32 == 0. */
void gen_fill_mxfp4(uint32_t seed, uint32_t tid, uint64_t row_start, uint64_t nrows, uint64_t K, float scale,
                    uint8_t* codes, uint8_t* scales, int nthreads) {
  gen_job j;
  memset(&j, 0, sizeof j);
  j.seed = seed;
  j.tid = tid;
  j.start = row_start;
  j.count = nrows;
  j.scale = scale;
  j.out = codes;
  j.kind = 2;
  j.K = K;
  j.scales = scales;
  run_parallel(&j, nrows, nthreads);
}

/* Seeded uniform 32-bit words (word 0 of Philox(index)), for permutations. */
void gen_fill_u32(uint32_t seed, uint32_t tid, uint64_t start, uint64_t count, uint32_t* out) {
  for (uint64_t i = 0; i < count; ++i) {
    uint64_t idx = start + i;
    uint32_t ctr[4] = {(uint32_t)idx, (uint32_t)(idx >> 32), 0u, 0u};
    uint32_t key[2] = {seed, tid};
    uint32_t w[4];
    gen_philox4x32_10_impl(ctr, key, w);
    out[i] = w[0];
  }
}
