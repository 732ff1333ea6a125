// fp64 CPU oracle of the Stable LatentMoE layer forward pass, in plain C++17
// with std::thread workers (TEST INFRASTRUCTURE ONLY: the tests, the smoke
// check and the bench's CPU-baseline / reference legs use it; the CUDA
// library never links or calls it, and it includes nothing of the library).
//
// Sources (web pages, cited by title and section):
//  [K3-896] "Kimi K3の896エキスパートを「896人の専門家」と呼ぶと何がズレるか、
//           ルーターは何を選んでいるのか"
//     - section "K3のエキスパートは896個の小型LLMではない": the dimension table
//       and the layer equations  z = W_down x;  u = sum_{i in Top16} p_i E_i(z);
//       y = E1_shared(x) + E2_shared(x) + W_up RMSNorm(u).
//     - section "ルーターは計算の割当器": s = Sigmoid(W_r x); a per-expert bias
//       is added to the scores to choose the experts; the mixture weights are
//       the original scores normalised over the chosen experts.
//  [K3-2axis] "Kimi K3の二軸スケーリング戦略とは何か", section "Stable
//     LatentMoE：条件付きの大容量を安定させる": inference keeps the expert
//     bias fixed and selects with ordinary top-k.
//  [K3-report] Kimi K3 tech-report summary, section "幅のスケーリング：Stable
//     LatentMoE": SiTU-GLU = SwiGLU with smooth caps on the linear and the up
//     branch.
//  [K3-QAT] ai-tech-express.jp article on K3, section "量子化を前提とした学習
//     「MXFP4 Quantization-Aware Training」": routed weights served in MXFP4
//     (format fixed by the OCP Microscaling Formats specification v1.0).
//     The pages give no activation format; where the routed experts take
//     MXFP8 or MXFP4 inputs (the block-scaled variants) the library's reading
//     is the same specification's formats with their shared-scale rule (below).
//
// Readings where the pages are silent (the same in the GPU library):
//  * SiTU-GLU(g, v) = sigmoid(g) * c*tanh(g/c) * c*tanh(v/c), c = 10;
//  * the shared experts use the same SiTU-GLU;
//  * RMSNorm(u) = gamma * u / sqrt(mean(u^2) + eps);
//  * equal selection keys go to the lower expert index; slots are listed in
//    descending key order; routing is dropless;
//  * storage-faithful rounding: where the device holds a tensor in the
//    activation type because it is a tensor-core operand (z, expert h, shared
//    h, n) the oracle rounds its fp64 value to that type; all else is fp64.
//
// Every sum is accumulated in fp64 in ascending index order (one running sum
// per output element); nothing is blocked, fused or reordered beyond that.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

// ------------------------------------------------------------------------------------------
// Worker threads: units of work handed out from an atomic counter.
// ------------------------------------------------------------------------------------------
int worker_count() {
  if (const char* env = std::getenv("MOE_ORACLE_THREADS")) {
    const int n = std::atoi(env);
    if (n > 0) return n;
  }
  const unsigned hc = std::thread::hardware_concurrency();
  return hc > 0 ? static_cast<int>(hc) : 1;
}

template <typename Fn>
void parallel_units(int64_t units, Fn fn) {
  if (units <= 0) return;
  const int nt = static_cast<int>(std::min<int64_t>(worker_count(), units));
  std::atomic<int64_t> next(0);
  auto work = [&](int tid) {
    for (int64_t u = next.fetch_add(1); u < units; u = next.fetch_add(1)) fn(u, tid);
  };
  if (nt == 1) {
    work(0);
    return;
  }
  std::vector<std::thread> pool;
  pool.reserve(nt);
  for (int t = 0; t < nt; ++t) pool.emplace_back(work, t);
  for (auto& th : pool) th.join();
}

// ------------------------------------------------------------------------------------------
// Number formats
// ------------------------------------------------------------------------------------------
// bf16 keeps 8 significant bits.  For x in [2^q, 2^(q+1)) the bf16 spacing is
// 2^(q-7) (2^-133 below the smallest normal, 2^-126); x / spacing is rounded
// to the nearest integer with ties to even (rint in the default rounding
// mode), then scaled back.  Both scalings are exact powers of two.
double round_to_bf16(double x) {
  if (x == 0.0 || !std::isfinite(x)) return x;
  int e = 0;
  std::frexp(x, &e);  // |x| = m * 2^e, m in [0.5, 1): |x| in [2^(e-1), 2^e)
  const int q = std::max(e - 1, -126);
  return std::ldexp(std::rint(std::ldexp(x, 7 - q)), q - 7);
}

double round_to_f32(double x) { return static_cast<double>(static_cast<float>(x)); }

enum RoundMode { kRoundNone = 0, kRoundBf16 = 1, kRoundF32 = 2 };

double store(double x, int mode) {
  return mode == kRoundBf16 ? round_to_bf16(x) : mode == kRoundF32 ? round_to_f32(x) : x;
}

double bf16_bits_value(uint16_t b) {
  // bf16 bits are the upper half of the fp32 with the same value
  const uint32_t w = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &w, sizeof f);
  return static_cast<double>(f);
}

// OCP MX v1.0 E2M1: sign bit 3, exponent bits 2-1 (bias 1), mantissa bit 0.
double e2m1_value(unsigned code) {
  const unsigned exp_bits = (code >> 1) & 3u, man = code & 1u;
  const double mag = exp_bits == 0 ? 0.5 * man                                    // subnormal: 0, 0.5
                                   : std::ldexp(1.0 + 0.5 * man, static_cast<int>(exp_bits) - 1);
  return (code & 8u) ? -mag : mag;
}

// OCP MX v1.0 E8M0 scale: 2^(s - 127), 0xFF = NaN.
double e8m0_value(uint8_t s) {
  if (s == 0xFF) return std::numeric_limits<double>::quiet_NaN();
  return std::ldexp(1.0, static_cast<int>(s) - 127);
}

// OCP FP8 E4M3 (OCP MX v1.0, FP8 E4M3): sign bit 7, exponent bits 6-3 (bias
// 7), mantissa bits 2-0; exponent field 0 is subnormal (m/8 * 2^-6); no
// infinities; S.1111.111 is NaN; largest finite 1.75 * 2^8 = 448.
double e4m3_value(uint8_t code) {
  const unsigned e = (code >> 3) & 15u, m = code & 7u;
  if (e == 15u && m == 7u) return std::numeric_limits<double>::quiet_NaN();
  const double mag = e == 0 ? std::ldexp(static_cast<double>(m), -9) : std::ldexp(8.0 + m, static_cast<int>(e) - 10);
  return (code & 0x80u) ? -mag : mag;
}

// Nearest E4M3 code to v, ties to the even code, magnitudes past 448
// saturated to 448 (the spec leaves overflow to the implementation; the
// library saturates).  The sign of v (of -0 too) is kept.
uint8_t e4m3_encode(double v) {
  const uint8_t sign = std::signbit(v) ? 0x80u : 0u;
  double a = std::fabs(v);
  if (a == 0.0) return sign;
  if (a >= 448.0) return sign | 0x7Eu;
  // spacing of E4M3 numbers around a: 2^(floor(log2 a) - 3), at least 2^-9
  int e2 = 0;
  std::frexp(a, &e2);  // a in [2^(e2-1), 2^e2)
  const int q = std::max(e2 - 1, -6);
  const double units = std::rint(std::ldexp(a, 3 - q));  // a / spacing, to nearest even integer
  // units in [8, 16] for q >= -6 normal numbers (16 carries into the next
  // exponent), in [0, 8] in the subnormal range
  if (q == -6 && units < 8.0) return sign | static_cast<uint8_t>(units);
  int exp_field = q + 7, mant = static_cast<int>(units) - 8;
  if (mant == 8) {
    ++exp_field;
    mant = 0;
  }
  if (exp_field > 15 || (exp_field == 15 && mant > 6)) return sign | 0x7Eu;
  return sign | static_cast<uint8_t>((exp_field << 3) | mant);
}

// OCP MX v1.0 shared scale of a block: s = floor(log2(max |v|)) - 8 (8 = the
// largest E4M3 exponent), clamped to the E8M0 range [-127, 127]; an all-zero
// block takes the lowest, -127.
int mx8_block_exponent(const double* v, int64_t n) {
  double amax = 0.0;
  for (int64_t i = 0; i < n; ++i) amax = std::max(amax, std::fabs(v[i]));
  if (amax == 0.0) return -127;
  int e2 = 0;
  std::frexp(amax, &e2);  // floor(log2 amax) = e2 - 1
  return std::max(-127, std::min(127, e2 - 1 - 8));
}

// One row of K values (K a multiple of 32) -> E4M3 codes [K] and E8M0 scale
// bytes [K/32]: block b's codes are e4m3_encode(v / 2^s_b), its scale byte
// s_b + 127.
void mx8_quantize_row(const double* v, int64_t K, uint8_t* codes, uint8_t* scales) {
  for (int64_t b = 0; b < K / 32; ++b) {
    const int s = mx8_block_exponent(v + 32 * b, 32);
    scales[b] = static_cast<uint8_t>(s + 127);
    for (int64_t i = 0; i < 32; ++i) codes[32 * b + i] = e4m3_encode(std::ldexp(v[32 * b + i], -s));
  }
}

// The values the MXFP8 encoding of a row stands for (quantise, then decode).
void mx8_round_row(const double* v, int64_t K, double* out) {
  std::vector<uint8_t> c(static_cast<size_t>(K)), sc(static_cast<size_t>(K / 32));
  mx8_quantize_row(v, K, c.data(), sc.data());
  for (int64_t k = 0; k < K; ++k) out[k] = e4m3_value(c[k]) * e8m0_value(sc[k / 32]);
}

// Nearest E2M1 code to v (OCP MX v1.0 FP4 E2M1: sign bit 3, exponent bits 2-1
// with bias 1, mantissa bit 0; values 0, 0.5, 1, 1.5, 2, 3, 4, 6), ties to the
// even code, magnitudes past 6 saturated to 6; the sign of v (of -0 too) kept.
// Between 2^q and 2^(q+1) (q >= 0) the E2M1 numbers are spaced 2^(q-1); below
// 2 the spacing is 0.5 (0.5 is the subnormal), so a / spacing is rounded to the
// nearest even integer (rint) and read back as exponent and mantissa.
uint8_t e2m1_encode(double v) {
  const uint8_t sign = std::signbit(v) ? 0x8u : 0u;
  const double a = std::fabs(v);
  if (a >= 6.0) return sign | 0x7u;
  if (a == 0.0) return sign;
  int e2 = 0;
  std::frexp(a, &e2);                        // a in [2^(e2-1), 2^e2)
  int q = std::max(e2 - 1, 0);
  int units = static_cast<int>(std::rint(std::ldexp(a, 1 - q)));  // a / 2^(q-1)
  if (q == 0) return sign | static_cast<uint8_t>(units);  // 0 .. 4: codes 0 .. 4 (4 = 2.0)
  if (units == 4) {                           // carry into the next binade
    ++q;
    units = 2;
  }
  return sign | static_cast<uint8_t>(((q + 1) << 1) | (units - 2));
}

// OCP MX v1.0 shared scale of an MXFP4 block: s = floor(log2(max |v|)) - 2 (2 =
// the largest E2M1 exponent), clamped to [-127, 127]; an all-zero block -127.
int mx4_block_exponent(const double* v, int64_t n) {
  double amax = 0.0;
  for (int64_t i = 0; i < n; ++i) amax = std::max(amax, std::fabs(v[i]));
  if (amax == 0.0) return -127;
  int e2 = 0;
  std::frexp(amax, &e2);
  return std::max(-127, std::min(127, e2 - 1 - 2));
}

// One row of K values -> packed E2M1 codes [K/2] (element 2i in the low
// nibble) and E8M0 scale bytes [K/32].
void mx4_quantize_row(const double* v, int64_t K, uint8_t* codes, uint8_t* scales) {
  for (int64_t b = 0; b < K / 32; ++b) {
    const int s = mx4_block_exponent(v + 32 * b, 32);
    scales[b] = static_cast<uint8_t>(s + 127);
    for (int64_t i = 0; i < 32; i += 2) {
      const uint8_t lo = e2m1_encode(std::ldexp(v[32 * b + i], -s));
      const uint8_t hi = e2m1_encode(std::ldexp(v[32 * b + i + 1], -s));
      codes[(32 * b + i) / 2] = static_cast<uint8_t>(lo | (hi << 4));
    }
  }
}

// The values the MXFP4 encoding of a row stands for.
void mx4_round_row(const double* v, int64_t K, double* out) {
  std::vector<uint8_t> c(static_cast<size_t>(K / 2)), sc(static_cast<size_t>(K / 32));
  mx4_quantize_row(v, K, c.data(), sc.data());
  for (int64_t k = 0; k < K; ++k) {
    const unsigned code = (k & 1) ? (c[k / 2] >> 4) : (c[k / 2] & 0xFu);
    out[k] = e2m1_value(code) * e8m0_value(sc[k / 32]);
  }
}

// Rounds a row of the expert's GEMM inputs to the activation format of the
// routed type: 0 none, 1 MXFP8, 2 MXFP4.
void act_round_row(int act, const double* v, int64_t K, double* out) {
  if (act == 1)
    mx8_round_row(v, K, out);
  else if (act == 2)
    mx4_round_row(v, K, out);
  else
    std::memcpy(out, v, sizeof(double) * K);
}

double sigmoid(double t) { return 1.0 / (1.0 + std::exp(-t)); }

double situ_glu(double g, double v, double c) {
  return sigmoid(g) * (c * std::tanh(g / c)) * (c * std::tanh(v / c));
}

}  // namespace

extern "C" {

// Element types of a weight matrix view.
enum { OC_F64 = 0, OC_F32 = 1, OC_BF16 = 2, OC_MXFP4 = 3 };

// A row-major [rows, cols] matrix.  F64 / F32: values.  BF16: raw uint16 bit
// patterns.  MXFP4: packed E2M1 codes [rows, cols/2] (even column in the low
// nibble) with E8M0 scales [rows, cols/32] in `scales`.
typedef struct {
  const void* data;
  const uint8_t* scales;
  int32_t type;
  int64_t rows, cols;
} oc_mat;

}  // extern "C"

namespace {

oc_mat row_view(const oc_mat& m, int64_t r0, int64_t nrows) {
  oc_mat v = m;
  v.rows = nrows;
  const uint8_t* base = static_cast<const uint8_t*>(m.data);
  switch (m.type) {
    case OC_F64:
      v.data = base + r0 * m.cols * 8;
      break;
    case OC_F32:
      v.data = base + r0 * m.cols * 4;
      break;
    case OC_BF16:
      v.data = base + r0 * m.cols * 2;
      break;
    default:
      v.data = base + r0 * (m.cols / 2);
      v.scales = m.scales + r0 * (m.cols / 32);
  }
  return v;
}

// Row r of m as fp64 values (exact for every supported type).
void decode_row(const oc_mat& m, int64_t r, double* out) {
  const int64_t K = m.cols;
  switch (m.type) {
    case OC_F64: {
      const double* p = static_cast<const double*>(m.data) + r * K;
      for (int64_t k = 0; k < K; ++k) out[k] = p[k];
      break;
    }
    case OC_F32: {
      const float* p = static_cast<const float*>(m.data) + r * K;
      for (int64_t k = 0; k < K; ++k) out[k] = static_cast<double>(p[k]);
      break;
    }
    case OC_BF16: {
      const uint16_t* p = static_cast<const uint16_t*>(m.data) + r * K;
      for (int64_t k = 0; k < K; ++k) out[k] = bf16_bits_value(p[k]);
      break;
    }
    default: {
      const uint8_t* q = static_cast<const uint8_t*>(m.data) + r * (K / 2);
      const uint8_t* s = m.scales + r * (K / 32);
      for (int64_t k = 0; k < K; ++k) {
        const unsigned code = (k & 1) ? (q[k / 2] >> 4) : (q[k / 2] & 0xFu);
        out[k] = e2m1_value(code) * e8m0_value(s[k / 32]);
      }
    }
  }
}

// out[r, n] = sum_k a[r, k] * W[n, k]   (a: [R, K] fp64; W: [N, K] view)
// Each output element is one fp64 running sum over k = 0 .. K-1 in order.
// Work is split into (8 columns of out) x (64 rows of a) units; a unit first
// decodes its 8 rows of W to fp64.
constexpr int64_t kColsPerUnit = 8;
constexpr int64_t kRowsPerUnit = 64;

void linear(const double* a, int64_t R, int64_t K, const oc_mat& W, double* out) {
  const int64_t N = W.rows;
  const int64_t col_units = (N + kColsPerUnit - 1) / kColsPerUnit;
  const int64_t row_units = (R + kRowsPerUnit - 1) / kRowsPerUnit;
  std::vector<std::vector<double>> buf(worker_count());
  parallel_units(col_units * row_units, [&](int64_t u, int tid) {
    const int64_t cu = u % col_units, ru = u / col_units;
    const int64_t n0 = cu * kColsPerUnit, n1 = std::min(N, n0 + kColsPerUnit);
    const int64_t r0 = ru * kRowsPerUnit, r1 = std::min(R, r0 + kRowsPerUnit);
    std::vector<double>& w = buf[tid];
    w.resize(static_cast<size_t>(kColsPerUnit * K));
    for (int64_t n = n0; n < n1; ++n) decode_row(W, n, &w[(n - n0) * K]);
    const int64_t nc = n1 - n0;
    for (int64_t r = r0; r < r1; ++r) {
      const double* ar = a + r * K;
      double acc[kColsPerUnit] = {0, 0, 0, 0, 0, 0, 0, 0};
      for (int64_t k = 0; k < K; ++k) {
        const double av = ar[k];
        for (int64_t j = 0; j < nc; ++j) acc[j] += av * w[j * K + k];
      }
      for (int64_t j = 0; j < nc; ++j) out[r * N + n0 + j] = acc[j];
    }
  });
}

// y[n, L] = W_o SiTU-GLU(W_g z, W_v z), h stored with `mode` ([K3-896]
// "K3のエキスパートは896個の小型LLMではない"; SiTU-GLU from [K3-report]).
// act (the routed experts' input format: 0 as stored, 1 MXFP8, 2 MXFP4): the
// expert's two GEMM inputs (the rows of z, and h after its storage rounding)
// are first replaced row by row by their values in that format.
void expert(const double* z, int64_t n, int64_t L, const oc_mat& Wg, const oc_mat& Wv, const oc_mat& Wo, double c,
            int mode, int act, double* y) {
  const int64_t I = Wg.rows;
  std::vector<double> zq;
  if (act != 0) {
    zq.resize(static_cast<size_t>(n * L));
    for (int64_t r = 0; r < n; ++r) act_round_row(act, z + r * L, L, &zq[r * L]);
    z = zq.data();
  }
  std::vector<double> g(static_cast<size_t>(n * I)), v(static_cast<size_t>(n * I));
  linear(z, n, L, Wg, g.data());
  linear(z, n, L, Wv, v.data());
  for (int64_t i = 0; i < n * I; ++i) g[i] = store(situ_glu(g[i], v[i], c), mode);
  if (act != 0)
    for (int64_t r = 0; r < n; ++r) {
      std::vector<double> row(g.begin() + r * I, g.begin() + (r + 1) * I);
      act_round_row(act, row.data(), I, &g[r * I]);
    }
  linear(g.data(), n, I, Wo, y);
}

}  // namespace

extern "C" {

int oc_num_threads(void) { return worker_count(); }

void oc_bf16_round(const double* x, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = round_to_bf16(x[i]);
}

void oc_f32_round(const double* x, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = round_to_f32(x[i]);
}

void oc_decode(const oc_mat* m, double* out) {
  for (int64_t r = 0; r < m->rows; ++r) decode_row(*m, r, out + r * m->cols);
}

void oc_sigmoid(const double* x, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = sigmoid(x[i]);
}

void oc_situ_glu(const double* g, const double* v, int64_t n, double c, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = situ_glu(g[i], v[i], c);
}

void oc_linear(const double* a, int64_t R, int64_t K, const oc_mat* W, double* out) { linear(a, R, K, *W, out); }

// s[t, e] = sigmoid(sum_h x[t, h] W_r[e, h])   ([K3-896] "ルーターは計算の割当器")
void oc_router_scores(const double* x, int64_t T, int64_t H, const oc_mat* Wr, double* s) {
  linear(x, T, H, *Wr, s);
  for (int64_t i = 0; i < T * Wr->rows; ++i) s[i] = sigmoid(s[i]);
}

// Selection with the frozen bias ([K3-896] "ルーターは計算の割当器"; [K3-2axis]):
// key = s + b, the k largest keys in descending order (equal keys: lower
// index first), p_j = s_{idx_j} / sum over the chosen experts of s (unbiased
// scores, summed in slot order), margin = key_(k) - key_(k+1) (+inf if k = E).
// bias is [E] (bias_per_token = 0) or [T, E].
void oc_select(const double* s, const double* bias, int bias_per_token, int64_t T, int64_t E, int64_t k,
               int64_t* idx, double* p, double* margin) {
  parallel_units(T, [&](int64_t t, int) {
    std::vector<double> key(static_cast<size_t>(E));
    std::vector<int64_t> order(static_cast<size_t>(E));
    const double* b = bias + (bias_per_token ? t * E : 0);
    for (int64_t e = 0; e < E; ++e) {
      key[e] = s[t * E + e] + b[e];
      order[e] = e;
    }
    std::sort(order.begin(), order.end(), [&](int64_t a, int64_t c) {
      return key[a] > key[c] || (key[a] == key[c] && a < c);
    });
    double sum = 0.0;
    for (int64_t j = 0; j < k; ++j) sum += s[t * E + order[j]];
    for (int64_t j = 0; j < k; ++j) {
      idx[t * k + j] = order[j];
      p[t * k + j] = s[t * E + order[j]] / sum;
    }
    margin[t] = k < E ? key[order[k - 1]] - key[order[k]] : std::numeric_limits<double>::infinity();
  });
}

// The same selection from fp32 scores with the key formed in fp32 (as the
// device forms it): key = fl32(s + b); p in fp64 from the fp32 scores.
void oc_select_f32(const float* s, const float* bias, int64_t T, int64_t E, int64_t k, int64_t* idx, double* p) {
  parallel_units(T, [&](int64_t t, int) {
    std::vector<float> key(static_cast<size_t>(E));
    std::vector<int64_t> order(static_cast<size_t>(E));
    for (int64_t e = 0; e < E; ++e) {
      const float kv = s[t * E + e] + bias[e];  // one fp32 addition, round to nearest
      key[e] = kv;
      order[e] = e;
    }
    std::sort(order.begin(), order.end(), [&](int64_t a, int64_t c) {
      return key[a] > key[c] || (key[a] == key[c] && a < c);
    });
    double sum = 0.0;
    for (int64_t j = 0; j < k; ++j) sum += static_cast<double>(s[t * E + order[j]]);
    for (int64_t j = 0; j < k; ++j) {
      idx[t * k + j] = order[j];
      p[t * k + j] = static_cast<double>(s[t * E + order[j]]) / sum;
    }
  });
}

// Expert-contiguous order of the (token, slot) pairs: pairs of expert e at
// positions offsets[e] .. offsets[e+1]-1 in ascending (token, slot) order.
// Returns -1 for an expert index outside [0, E).
int oc_permute(const int64_t* idx, int64_t T, int64_t k, int64_t E, int64_t* counts, int64_t* offsets,
               int64_t* perm_token, int64_t* inv_perm) {
  for (int64_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t i = 0; i < T * k; ++i) {
    if (idx[i] < 0 || idx[i] >= E) return -1;
    ++counts[idx[i]];
  }
  offsets[0] = 0;
  for (int64_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  std::vector<int64_t> fill(offsets, offsets + E);
  for (int64_t t = 0; t < T; ++t)
    for (int64_t j = 0; j < k; ++j) {
      const int64_t pos = fill[idx[t * k + j]]++;
      perm_token[pos] = t;
      inv_perm[t * k + j] = pos;
    }
  return 0;
}

void oc_expert_forward(const double* z, int64_t n, int64_t L, const oc_mat* Wg, const oc_mat* Wv, const oc_mat* Wo,
                       double c, int mode, int act, double* y) {
  expert(z, n, L, *Wg, *Wv, *Wo, c, mode, act, y);
}

// E2M1 codes (one per byte, low nibble) <-> values; rows of values -> packed
// MXFP4 codes [rows, K/2] and E8M0 scale bytes [rows, K/32].
void oc_e2m1_encode(const double* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e2m1_encode(v[i]);
}

void oc_mx4_quantize(const double* v, int64_t rows, int64_t K, uint8_t* codes, uint8_t* scales) {
  for (int64_t r = 0; r < rows; ++r) mx4_quantize_row(v + r * K, K, codes + r * (K / 2), scales + r * (K / 32));
}

// E4M3 codes -> values; values -> nearest E4M3 codes (ties to even,
// saturating); rows of values -> MXFP8 codes [rows, K] and E8M0 scale bytes
// [rows, K/32] (OCP MX v1.0; K a multiple of 32).
void oc_e4m3_decode(const uint8_t* codes, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_value(codes[i]);
}

void oc_e4m3_encode(const double* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_encode(v[i]);
}

void oc_mx8_quantize(const double* v, int64_t rows, int64_t K, uint8_t* codes, uint8_t* scales) {
  for (int64_t r = 0; r < rows; ++r) mx8_quantize_row(v + r * K, K, codes + r * K, scales + r * (K / 32));
}

// u[t] = sum_j p[t, j] y_slots[t, j]   (j ascending)
void oc_combine(const double* y_slots, const double* p, int64_t T, int64_t k, int64_t L, double* u) {
  for (int64_t t = 0; t < T; ++t)
    for (int64_t l = 0; l < L; ++l) {
      double acc = 0.0;
      for (int64_t j = 0; j < k; ++j) acc += p[t * k + j] * y_slots[(t * k + j) * L + l];
      u[t * L + l] = acc;
    }
}

// n[t] = gamma * u[t] / sqrt(mean_l u[t, l]^2 + eps)
void oc_rms_norm(const double* u, const double* gamma, int64_t T, int64_t L, double eps, double* n) {
  for (int64_t t = 0; t < T; ++t) {
    double ss = 0.0;
    for (int64_t l = 0; l < L; ++l) ss += u[t * L + l] * u[t * L + l];
    const double d = std::sqrt(ss / static_cast<double>(L) + eps);
    for (int64_t l = 0; l < L; ++l) n[t * L + l] = gamma[l] * u[t * L + l] / d;
  }
}

// y = sum_i W_so,i SiTU-GLU(W_sg,i x, W_sv,i x), each h_i stored with `mode`.
// Wsg / Wsv: [S*Is, H]; Wso: [S*H, Is].
void oc_shared_experts(const double* x, int64_t T, int64_t H, int64_t S, int64_t Is, const oc_mat* Wsg,
                       const oc_mat* Wsv, const oc_mat* Wso, double c, int mode, double* y) {
  std::vector<double> yi(static_cast<size_t>(T * H));
  for (int64_t i = 0; i < T * H; ++i) y[i] = 0.0;
  for (int64_t s = 0; s < S; ++s) {
    expert(x, T, H, row_view(*Wsg, s * Is, Is), row_view(*Wsv, s * Is, Is), row_view(*Wso, s * H, H), c, mode, 0,
           yi.data());
    for (int64_t i = 0; i < T * H; ++i) y[i] += yi[i];
  }
}

// ------------------------------------------------------------------------------------------
// The whole layer.
// ------------------------------------------------------------------------------------------
typedef struct {
  int64_t T;
  int32_t H, L, E, k, I, S, Is;
  double situ_c, rms_eps;
  int32_t mode;  // storage rounding of z, h, shared h, n
  int32_t routed_act;  // the routed experts' input format: 0 as stored, 1 MXFP8, 2 MXFP4 (block-scaled variants)
} oc_dims;

typedef struct {
  oc_mat Wr;          // [E, H]
  const double* bias; // [E]
  oc_mat Wdown;       // [L, H]
  oc_mat Wup;         // [H, L]
  const double* gamma;// [L]
  oc_mat Wg, Wv, Wo;  // in memory: [E*I, L], [E*I, L], [E*L, I]; unused (rows = 0) with a provider
  oc_mat Wsg, Wsv, Wso;
} oc_weights;

// Supplies expert e's (W_g [I, L], W_v [I, L], W_o [L, I]); nonzero = failure.
typedef int (*oc_expert_provider)(void* ctx, int32_t e, oc_mat* Wg, oc_mat* Wv, oc_mat* Wo);

typedef struct {
  double* s;        // [T, E]
  int64_t* idx;     // [T, k]
  double* p;        // [T, k]
  double* margin;   // [T]
  double* z;        // [T, L]
  double* u;        // [T, L]
  double* n;        // [T, L]
  double* y;        // [T, H]
  double* y_shared; // [T, H]
} oc_outputs;

// Steps in the order the pages give them ([K3-896]):
//   s = Sigmoid(W_r x); key = s + b; top-k; p = renormalised s      (router)
//   z = W_down x                                                    (latent)
//   u = sum_j p_j E_{idx_j}(z)                                      (routed experts)
//   y = sum_i E_shared,i(x) + W_up RMSNorm(u)                        (output)
// forced_idx (may be NULL) replaces the selection; p is then the unbiased
// scores renormalised over the forced experts.  Returns 0, or -1 if the
// provider failed or an index is out of range.
int oc_layer_forward(const oc_dims* d, const oc_weights* w, const double* x, const int64_t* forced_idx,
                     oc_expert_provider provider, void* ctx, const oc_outputs* o) {
  const int64_t T = d->T, H = d->H, L = d->L, E = d->E, k = d->k, I = d->I;
  oc_router_scores(x, T, H, &w->Wr, o->s);
  oc_select(o->s, w->bias, 0, T, E, k, o->idx, o->p, o->margin);
  if (forced_idx != nullptr) {
    for (int64_t t = 0; t < T; ++t) {
      double sum = 0.0;
      for (int64_t j = 0; j < k; ++j) {
        const int64_t e = forced_idx[t * k + j];
        if (e < 0 || e >= E) return -1;
        sum += o->s[t * E + e];
      }
      for (int64_t j = 0; j < k; ++j) {
        o->idx[t * k + j] = forced_idx[t * k + j];
        o->p[t * k + j] = o->s[t * E + forced_idx[t * k + j]] / sum;
      }
    }
  }
  linear(x, T, H, w->Wdown, o->z);
  for (int64_t i = 0; i < T * L; ++i) o->z[i] = store(o->z[i], d->mode);

  // routed experts, one expert at a time over its (token, slot) pairs
  std::vector<double> y_slots(static_cast<size_t>(T * k * L), 0.0);
  std::vector<std::vector<int64_t>> pairs(static_cast<size_t>(E));
  for (int64_t t = 0; t < T; ++t)
    for (int64_t j = 0; j < k; ++j) pairs[o->idx[t * k + j]].push_back(t * k + j);
  std::vector<double> zr, yr;
  for (int64_t e = 0; e < E; ++e) {
    const std::vector<int64_t>& pe = pairs[e];
    if (pe.empty()) continue;
    oc_mat Wg, Wv, Wo;
    if (provider != nullptr) {
      if (provider(ctx, static_cast<int32_t>(e), &Wg, &Wv, &Wo) != 0) return -1;
    } else {
      Wg = row_view(w->Wg, e * I, I);
      Wv = row_view(w->Wv, e * I, I);
      Wo = row_view(w->Wo, e * L, L);
    }
    const int64_t n = static_cast<int64_t>(pe.size());
    zr.assign(static_cast<size_t>(n * L), 0.0);
    yr.assign(static_cast<size_t>(n * L), 0.0);
    for (int64_t r = 0; r < n; ++r) std::memcpy(&zr[r * L], o->z + (pe[r] / k) * L, sizeof(double) * L);
    expert(zr.data(), n, L, Wg, Wv, Wo, d->situ_c, d->mode, d->routed_act, yr.data());
    for (int64_t r = 0; r < n; ++r) std::memcpy(&y_slots[pe[r] * L], &yr[r * L], sizeof(double) * L);
  }
  oc_combine(y_slots.data(), o->p, T, k, L, o->u);
  oc_rms_norm(o->u, w->gamma, T, L, d->rms_eps, o->n);
  for (int64_t i = 0; i < T * L; ++i) o->n[i] = store(o->n[i], d->mode);
  oc_shared_experts(x, T, H, d->S, d->Is, &w->Wsg, &w->Wsv, &w->Wso, d->situ_c, d->mode, o->y_shared);
  linear(o->n, T, L, w->Wup, o->y);
  for (int64_t i = 0; i < T * H; ++i) o->y[i] = o->y_shared[i] + o->y[i];
  return 0;
}

}  // extern "C"
