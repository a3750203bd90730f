// Plain, slow, obviously correct CPU oracle of the fused top-k MoE layer.
//
// TEST INFRASTRUCTURE ONLY: loaded (through oracle/moe_oracle.py) by tests/,
// by __graft_entry__.smoke() and by the CPU-baseline legs of bench.py; never
// by the product path.  It shares no code, header, table or constant
// generator with the CUDA library; it includes no CUDA header.
//
// C++17, double precision except where the method fixes a narrower format;
// every rounding point the method names is applied explicitly, so each
// function can be read against its source passage.  Loops are written in the
// order of the definitions they restate: no blocking, no fusion beyond the
// method's own.  The only parallelism is independent rows (OpenMP), which
// does not change any result.
//
// Sources (web pages the method is taken from):
//  [AWS]  "AWS erklärt zwei Kernel-Optimierungen, die den Durchsatz von
//         SageMaker AI auf H200 steigern" (kinachrichten.com).
//  [PR]   the analysis of vLLM PR #64760, "vLLM, H200 GPU를 위한 FP8 MoE 다운
//         프로젝션 최적화" (blog.secrett2633.cloud).
//  [PPLX] "Hosting von Qwen auf Blackwell" (perplexity.ai).
//
// Readings where the pages are silent (each is pinned in tests/test_oracle_*):
//  * route: experts chosen on the raw logits (softmax is monotone), equal
//    logits to the lower index; weights = softmax over all experts,
//    renormalised over the chosen ones.
//  * align: flat ids t*topk+j keep ascending order inside an expert; padding
//    holds the sentinel T*topk; empty experts own no block; unused blocks -1.
//  * the GEMM1 input x is quantised by the same per-(row,128) power-of-two
//    rule the fused kernel of [PR] §1.2 applies to the intermediate.
//  * weight block scale: max(blockmax, 1e-10) / 448 in fp32, code =
//    e4m3(fp32(w / scale)).
//  * combine: out[t] = sum_j w[t,j] * y[t,j] exactly (double), one bf16
//    rounding; duplicate ids in a row are independent assignments.
//  * MXFP8: one E8M0 scale per 32 elements of a row, by the same power-of-two
//    rule.
//  * expert parallelism: rank r of N holds experts [floor(rE/N),
//    floor((r+1)E/N)); a rank's output is the bf16 rounding of its own
//    assignments' sum; the all-reduce is the exact sum of the bf16 partials,
//    rounded once.
//
// Every entry point returns 0 on success and -1 on a caller error (the text
// is in orc_last_error()).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <string>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_API extern "C" __attribute__((visibility("default")))

namespace {

thread_local std::string g_err;

int fail(const std::string& m) {
  g_err = m;
  return -1;
}

// ---------------------------------------------------------------- number formats
// bfloat16: 1 sign, 8 exponent, 7 stored mantissa bits (8 significant bits).
const double kBf16Max = (2.0 - std::ldexp(1.0, -7)) * std::ldexp(1.0, 127);
// OCP 8-bit floating point E4M3 ("fn": no infinities; S.1111.111 is NaN).
constexpr double kE4m3Max = 448.0;
constexpr int kMxGroup = 32;     // elements per MXFP8 scale
constexpr int kE8m0Bias = 127;   // E8M0 byte of the scale 2**0

// Nearest bfloat16 value, ties to even.  bf16 keeps 8 significant bits over
// the binary32 exponent range: values whose leading bit weighs 2**(e-1) are
// spaced 2**(e-8); below the smallest normal 2**-126 the spacing is 2**-133.
// Values that round past the largest finite bf16 become infinite.
double round_bf16(double x) {
  if (!std::isfinite(x) || x == 0.0) return x;
  int e = 0;
  std::frexp(x, &e);                       // x = m * 2**e, 0.5 <= |m| < 1
  const int q = std::max(e - 8, -133);     // exponent of one unit in the last place
  const double r = std::ldexp(std::nearbyint(std::ldexp(x, -q)), q);
  if (std::fabs(r) > kBf16Max) return std::copysign(INFINITY, r);
  return r;
}

// bf16 bit pattern -> its value (the upper half of a binary32).
double bf16_bits_value(uint16_t b) {
  const uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  static_assert(sizeof f == sizeof u, "binary32");
  __builtin_memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

// Nearest E4M3 value, ties to even, saturating at +-448 (the clamp of [PR]
// §1.2).  4 significant bits, exponent bias 7, smallest normal 2**-6,
// subnormal spacing 2**-9.  The sign of a result that rounds to zero is kept.
double e4m3_round(double x) {
  if (std::isnan(x)) return x;
  if (std::isinf(x)) return std::copysign(kE4m3Max, x);
  if (x == 0.0) return x;
  int e = 0;
  std::frexp(x, &e);
  const int q = std::max(e - 4, -9);
  double r = std::ldexp(std::nearbyint(std::ldexp(x, -q)), q);
  r = std::min(std::max(r, -kE4m3Max), kE4m3Max);
  return r == 0.0 ? std::copysign(0.0, x) : r;
}

// Value of an E4M3 code, from the format definition.
double e4m3_value(uint8_t code) {
  const double sign = (code & 0x80) ? -1.0 : 1.0;
  const int exp_field = (code >> 3) & 0xF;
  const int mant = code & 0x7;
  if (exp_field == 0xF && mant == 0x7) return NAN;
  if (exp_field == 0) return sign * mant * std::ldexp(1.0, -9);
  return sign * (1.0 + mant / 8.0) * std::ldexp(1.0, exp_field - 7);
}

struct E4m3Table {
  double v[256];
  E4m3Table() {
    for (int c = 0; c < 256; ++c) v[c] = e4m3_value(static_cast<uint8_t>(c));
  }
};
const E4m3Table kE4m3;

// Round with e4m3_round, then write the code: sign, 4 exponent bits, 3
// mantissa bits (NaN -> S.1111.111).
uint8_t e4m3_encode(double x) {
  const double v = e4m3_round(x);
  const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  if (std::isnan(v)) return sign | 0x7F;
  const double a = std::fabs(v);
  if (a >= std::ldexp(1.0, -6)) {
    int e = 0;
    std::frexp(a, &e);                                     // leading bit weight 2**(e-1)
    const int exp_field = e - 1 + 7;
    const int mant = static_cast<int>(std::nearbyint((std::ldexp(a, -(e - 1)) - 1.0) * 8.0));
    return sign | static_cast<uint8_t>((exp_field << 3) | mant);
  }
  return sign | static_cast<uint8_t>(std::nearbyint(std::ldexp(a, 9)));   // subnormal or zero
}

// Smallest power of two >= s (s > 0), taken from the binary exponent so that
// exact powers of two map to themselves ([PR] §1.2 writes exp2(ceil(log2 s))).
double pow2_ceil(double s) {
  int e = 0;
  const double m = std::frexp(s, &e);                      // s = m * 2**e, 0.5 <= m < 1
  return m == 0.5 ? std::ldexp(1.0, e - 1) : std::ldexp(1.0, e);
}

// [PR] §1.2: raw scale max(amax, 1e-10) * (1/448), one fp32 rounding, then
// the power of two at or above it.  Shared by the per-(row,128) rule and the
// per-32 MX rule (the same rule on another group size).
double pow2_group_scale(double amax) {
  const float amax_f = static_cast<float>(amax);          // exact: the values are fp32
  const float floor_f = static_cast<float>(1e-10);
  const float inv448_f = static_cast<float>(1.0 / 448.0);
  const float raw = std::max(amax_f, floor_f) * inv448_f;  // fp32 product
  return pow2_ceil(static_cast<double>(raw));
}

// Quantise one group of n values with a power-of-two scale: codes and scale.
double quantize_group_pow2(const double* v, int n, uint8_t* codes) {
  double amax = 0.0;
  for (int i = 0; i < n; ++i) amax = std::max(amax, std::fabs(v[i]));
  const double scale = pow2_group_scale(amax);
  for (int i = 0; i < n; ++i) {
    const double q = std::min(std::max(v[i] / scale, -kE4m3Max), kE4m3Max);   // exact: scale is 2**n
    codes[i] = e4m3_encode(q);
  }
  return scale;
}

int e8m0_of_pow2(double scale) {
  int e = 0;
  std::frexp(scale, &e);                                   // scale = 0.5 * 2**e
  return e - 1 + kE8m0Bias;
}

// ---------------------------------------------------------------- weights
// Read access to one expert's [N, K] weight matrix in its stored format; the
// dequantised value w_hat = decode(code) * scale is formed when it is read
// (exactly the product a dequantised copy would hold: a 4-bit by 24-bit
// significand product is exact in double).
enum WeightType { W_F64 = 0, W_BF16 = 1, W_FP8_BLOCK128 = 2, W_MXFP8 = 3 };

struct Weights {
  int type;
  const void* data;
  const void* scale;
  int64_t N, K;
  double at(int64_t n, int64_t k) const {
    switch (type) {
      case W_F64:
        return static_cast<const double*>(data)[n * K + k];
      case W_BF16:
        return bf16_bits_value(static_cast<const uint16_t*>(data)[n * K + k]);
      case W_FP8_BLOCK128: {
        const uint8_t c = static_cast<const uint8_t*>(data)[n * K + k];
        const float s = static_cast<const float*>(scale)[(n / 128) * (K / 128) + k / 128];
        return kE4m3.v[c] * static_cast<double>(s);
      }
      default: {
        const uint8_t c = static_cast<const uint8_t*>(data)[n * K + k];
        const uint8_t e = static_cast<const uint8_t*>(scale)[n * (K / kMxGroup) + k / kMxGroup];
        return kE4m3.v[c] * std::ldexp(1.0, static_cast<int>(e) - kE8m0Bias);
      }
    }
  }
};

// sum_k w_hat[n, k] * v[k]: the dot product of weight row n with v, in double.
// The terms are those of the definition; the order of the additions is left
// to the compiler's vector lanes (any order of a double sum is a valid
// evaluation of it, and the results feed bf16 roundings).
double dot_row(const Weights& w, int64_t n, const double* v) {
  const int64_t K = w.K;
  double acc = 0.0;
  switch (w.type) {
    case W_F64: {
      const double* r = static_cast<const double*>(w.data) + n * K;
#pragma omp simd reduction(+ : acc)
      for (int64_t k = 0; k < K; ++k) acc += r[k] * v[k];
      break;
    }
    case W_BF16: {
      const uint16_t* r = static_cast<const uint16_t*>(w.data) + n * K;
#pragma omp simd reduction(+ : acc)
      for (int64_t k = 0; k < K; ++k) acc += bf16_bits_value(r[k]) * v[k];
      break;
    }
    case W_FP8_BLOCK128: {
      const uint8_t* r = static_cast<const uint8_t*>(w.data) + n * K;
      const float* s = static_cast<const float*>(w.scale) + (n / 128) * (K / 128);
#pragma omp simd reduction(+ : acc)
      for (int64_t k = 0; k < K; ++k) acc += (kE4m3.v[r[k]] * static_cast<double>(s[k / 128])) * v[k];
      break;
    }
    default: {
      const uint8_t* r = static_cast<const uint8_t*>(w.data) + n * K;
      const uint8_t* e = static_cast<const uint8_t*>(w.scale) + n * (K / kMxGroup);
#pragma omp simd reduction(+ : acc)
      for (int64_t k = 0; k < K; ++k)
        acc += (kE4m3.v[r[k]] * std::ldexp(1.0, static_cast<int>(e[k / kMxGroup]) - kE8m0Bias)) * v[k];
      break;
    }
  }
  return acc;
}

// ---------------------------------------------------------------- expert MLP
enum Requant { RQ_NONE = 0, RQ_BLOCK128 = 1, RQ_MX = 2 };

struct MlpScratch {
  std::vector<double> h, p, p_hat;
  std::vector<uint8_t> codes;
  std::vector<double> scales;
};

// One expert's SiLU-gated MLP on one row ([PR] §1.1 / §1.2):
//   h = x_hat . w13^T rounded to bf16 (intermediate_cache1 is bf16);
//   gate = h[0, I), up = h[I, 2I);
//   optional SwiGLU limit L (reading): gate = min(gate, L), up = clamp(up, -L, L);
//   act = bf16(gate / (1 + exp(-gate)));  p = bf16(act * up);
//   p_hat = p (bf16 path) or the per-(row,128) / per-32 MX requantisation of p;
//   y = p_hat . w2^T (double).
void expert_mlp_row(const double* x_hat, const Weights& w13, const Weights& w2, int64_t H, int64_t I,
                    int requant, bool has_limit, double limit_in, double* y, MlpScratch& s) {
  const double limit = static_cast<double>(static_cast<float>(limit_in));   // the limit is an fp32 value
  s.h.resize(2 * I);
  s.p.resize(I);
  s.p_hat.resize(I);
  s.codes.resize(I);
  for (int64_t n = 0; n < 2 * I; ++n) {
    s.h[n] = round_bf16(dot_row(w13, n, x_hat));
  }
  for (int64_t i = 0; i < I; ++i) {
    double gate = s.h[i];
    double up = s.h[I + i];
    if (has_limit) {
      gate = std::min(gate, limit);
      up = std::min(std::max(up, -limit), limit);
    }
    const double act = round_bf16(gate / (1.0 + std::exp(-gate)));
    s.p[i] = round_bf16(act * up);
  }
  if (requant == RQ_NONE) {
    for (int64_t i = 0; i < I; ++i) s.p_hat[i] = s.p[i];
  } else {
    const int group = requant == RQ_MX ? kMxGroup : 128;
    s.scales.resize(I / group);
    for (int64_t g = 0; g < I / group; ++g) {
      const double scale = quantize_group_pow2(&s.p[g * group], group, &s.codes[g * group]);
      s.scales[g] = scale;
      for (int j = 0; j < group; ++j) s.p_hat[g * group + j] = kE4m3.v[s.codes[g * group + j]] * scale;
    }
  }
  for (int64_t n = 0; n < H; ++n) {
    y[n] = dot_row(w2, n, s.p_hat.data());
  }
}

int threads_or_default(int nt) {
#ifdef _OPENMP
  return nt > 0 ? nt : omp_get_max_threads();
#else
  (void)nt;
  return 1;
#endif
}

}  // namespace

// ============================================================================ C ABI
ORC_API const char* orc_last_error(void) { return g_err.c_str(); }
ORC_API double orc_bf16_max(void) { return kBf16Max; }
ORC_API double orc_e4m3_max(void) { return kE4m3Max; }

ORC_API int orc_max_threads(void) { return threads_or_default(0); }

ORC_API void orc_round_bf16(const double* x, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = round_bf16(x[i]);
}

ORC_API void orc_e4m3_round(const double* x, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_round(x[i]);
}

ORC_API void orc_e4m3_encode(const double* x, uint8_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_encode(x[i]);
}

ORC_API void orc_e4m3_decode(const uint8_t* c, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = kE4m3.v[c[i]];
}

ORC_API void orc_pow2_ceil(const double* s, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = pow2_ceil(s[i]);
}

ORC_API void orc_mx_scale(const uint8_t* e8m0, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = std::ldexp(1.0, static_cast<int>(e8m0[i]) - kE8m0Bias);
}

// [PR] §1.2 per (row, 128 consecutive columns); the same rule quantises the
// GEMM1 input x (reading).  v [rows, K] (fp32-representable values), K % 128 == 0.
ORC_API int orc_quantize_act_group128(const double* v, int64_t rows, int64_t K, uint8_t* codes, float* scales) {
  if (K % 128) return fail("K must be a multiple of 128");
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t g = 0; g < K / 128; ++g)
      scales[r * (K / 128) + g] = static_cast<float>(quantize_group_pow2(&v[r * K + g * 128], 128,
                                                                          &codes[r * K + g * 128]));
  return 0;
}

ORC_API void orc_dequantize_act_group128(const uint8_t* codes, const float* scales, int64_t rows, int64_t K,
                                         double* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k)
      out[r * K + k] = kE4m3.v[codes[r * K + k]] * static_cast<double>(scales[r * (K / 128) + k / 128]);
}

// Workload definition: per 128x128 block scale = max(blockmax, 1e-10) / 448
// (fp32 division; the floor is a reading), code = e4m3(fp32(w / scale)) (fp32
// division).  w [batches, N, K] (bf16 values).
ORC_API int orc_quantize_weight_block128(const void* w_in, int32_t in_bf16, int64_t batches, int64_t N, int64_t K,
                                         uint8_t* codes, float* scales, int32_t num_threads) {
  if (N % 128 || K % 128) return fail("N and K must be multiples of 128");
  const int64_t nb = N / 128, kb = K / 128;
  // the input as values: double, or bf16 bit patterns
  auto w = [&](int64_t i) {
    return in_bf16 ? bf16_bits_value(static_cast<const uint16_t*>(w_in)[i]) : static_cast<const double*>(w_in)[i];
  };
#pragma omp parallel for collapse(2) schedule(static) num_threads(threads_or_default(num_threads))
  for (int64_t b = 0; b < batches; ++b)
    for (int64_t bn = 0; bn < nb; ++bn)
      for (int64_t bk = 0; bk < kb; ++bk) {
        double bmax = 0.0;
        for (int64_t n = bn * 128; n < bn * 128 + 128; ++n)
          for (int64_t k = bk * 128; k < bk * 128 + 128; ++k) bmax = std::max(bmax, std::fabs(w((b * N + n) * K + k)));
        const float scale = std::max(static_cast<float>(bmax), static_cast<float>(1e-10)) / 448.0f;
        scales[(b * nb + bn) * kb + bk] = scale;
        for (int64_t n = bn * 128; n < bn * 128 + 128; ++n)
          for (int64_t k = bk * 128; k < bk * 128 + 128; ++k) {
            const float ratio = static_cast<float>(w((b * N + n) * K + k)) / scale;
            codes[(b * N + n) * K + k] = e4m3_encode(static_cast<double>(ratio));
          }
      }
  return 0;
}

ORC_API void orc_dequantize_weight_block128(const uint8_t* codes, const float* scales, int64_t batches, int64_t N,
                                            int64_t K, double* out) {
  for (int64_t b = 0; b < batches; ++b) {
    const Weights w{W_FP8_BLOCK128, codes + b * N * K, scales + b * (N / 128) * (K / 128), N, K};
    for (int64_t n = 0; n < N; ++n)
      for (int64_t k = 0; k < K; ++k) out[(b * N + n) * K + k] = w.at(n, k);
  }
}

// [PPLX] "Quantisierung" (MXFP8): one E8M0 scale per 32 consecutive elements
// of a row, by the power-of-two rule above (reading).  v [rows, K], K % 32 == 0.
ORC_API int orc_quantize_mx_group32(const void* v_in, int32_t in_bf16, int64_t rows, int64_t K, uint8_t* codes,
                                    uint8_t* e8m0, int32_t num_threads) {
  if (K % kMxGroup) return fail("K must be a multiple of 32");
#pragma omp parallel for schedule(static) num_threads(threads_or_default(num_threads))
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t g = 0; g < K / kMxGroup; ++g) {
      double v[kMxGroup];                                  // the group's values (double, or bf16 bit patterns)
      for (int j = 0; j < kMxGroup; ++j) {
        const int64_t i = r * K + g * kMxGroup + j;
        v[j] = in_bf16 ? bf16_bits_value(static_cast<const uint16_t*>(v_in)[i]) : static_cast<const double*>(v_in)[i];
      }
      const double scale = quantize_group_pow2(v, kMxGroup, &codes[r * K + g * kMxGroup]);
      e8m0[r * (K / kMxGroup) + g] = static_cast<uint8_t>(e8m0_of_pow2(scale));
    }
  return 0;
}

ORC_API void orc_dequantize_mx_group32(const uint8_t* codes, const uint8_t* e8m0, int64_t rows, int64_t K,
                                       double* out) {
  const Weights w{W_MXFP8, codes, e8m0, rows, K};
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k) out[r * K + k] = w.at(r, k);
}

// Top-k softmax router ([AWS] "Warum MoE-Kernel so wichtig sind" and the
// workload recipe): experts picked on the raw logits in descending order,
// equal logits by the lower index; weights = softmax over all E experts
// (double), the chosen ones renormalised to sum to one when asked.
ORC_API int orc_route(const float* logits, int64_t T, int32_t E, int32_t topk, int32_t renormalize, int32_t* ids,
                      float* weights) {
  if (topk < 1 || topk > E) return fail("need 1 <= topk <= E");
  for (int64_t i = 0; i < T * E; ++i)
    if (std::isnan(logits[i])) return fail("NaN logit");
  std::vector<char> taken(E);
  std::vector<double> p(E);
  for (int64_t t = 0; t < T; ++t) {
    const float* l = logits + t * E;
    std::fill(taken.begin(), taken.end(), 0);
    for (int32_t j = 0; j < topk; ++j) {
      int32_t best = -1;
      for (int32_t e = 0; e < E; ++e)
        if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;     // strict: ties keep the lower index
      taken[best] = 1;
      ids[t * topk + j] = best;
    }
    double m = -INFINITY;
    for (int32_t e = 0; e < E; ++e) m = std::max(m, static_cast<double>(l[e]));
    double sum = 0.0;
    for (int32_t e = 0; e < E; ++e) {
      p[e] = std::exp(static_cast<double>(l[e]) - m);
      sum += p[e];
    }
    for (int32_t e = 0; e < E; ++e) p[e] /= sum;
    double chosen_sum = 0.0;
    for (int32_t j = 0; j < topk; ++j) chosen_sum += p[ids[t * topk + j]];
    for (int32_t j = 0; j < topk; ++j) {
      const double w = p[ids[t * topk + j]];
      weights[t * topk + j] = static_cast<float>(renormalize ? w / chosen_sum : w);
    }
  }
  return 0;
}

// Length of sorted_token_ids: every non-empty expert pads its count up to a
// multiple of block_m (at most block_m - 1 extra slots) and at most
// min(E, T*topk) experts are non-empty; rounded up to whole blocks.
ORC_API int64_t orc_align_capacity(int64_t T, int32_t topk, int32_t E, int32_t block_m) {
  const int64_t n = T * topk;
  if (n == 0) return 0;
  const int64_t bound = n + std::min<int64_t>(E, n) * (block_m - 1);
  return (bound + block_m - 1) / block_m * block_m;
}

// [PR] §1.1: the expert-sorted, block-padded permutation of the flat
// assignments t*topk + j.  Expert parallelism ([PPLX] "Experten-Parallel":
// the dispatch keeps the tokens of this rank's experts): ids are global in
// [0, num_global); only [first, first + E) are kept, as local id - first.
ORC_API int orc_align(const int32_t* topk_ids, int64_t T, int32_t topk, int32_t E, int32_t block_m,
                      int32_t first_expert, int32_t num_global, int32_t* sorted_ids, int32_t* expert_ids,
                      int32_t* ntpp, int32_t* counts, int32_t* offsets) {
  if (block_m < 1 || E < 1) return fail("need E >= 1 and block_m >= 1");
  const int64_t n = T * topk;
  for (int64_t f = 0; f < n; ++f)
    if (topk_ids[f] < 0 || topk_ids[f] >= num_global) return fail("expert id out of range");
  const int64_t cap = orc_align_capacity(T, topk, E, block_m);
  for (int32_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t f = 0; f < n; ++f) {
    const int32_t e = topk_ids[f] - first_expert;
    if (e >= 0 && e < E) counts[e] += 1;
  }
  offsets[0] = 0;
  for (int32_t e = 0; e < E; ++e)
    offsets[e + 1] = offsets[e] + (counts[e] + block_m - 1) / block_m * block_m;
  for (int64_t r = 0; r < cap; ++r) sorted_ids[r] = static_cast<int32_t>(n);
  for (int64_t b = 0; b < cap / block_m; ++b) expert_ids[b] = -1;
  for (int32_t e = 0; e < E; ++e) {
    int64_t slot = offsets[e];
    for (int64_t f = 0; f < n; ++f)                        // ascending flat order
      if (topk_ids[f] - first_expert == e) sorted_ids[slot++] = static_cast<int32_t>(f);
    for (int64_t b = offsets[e] / block_m; b < offsets[e + 1] / block_m; ++b) expert_ids[b] = e;
  }
  *ntpp = offsets[E];
  return 0;
}

// One expert's MLP on rows of x_hat (double weights), with the intermediates:
// h [rows, 2I], p [rows, I], codes [rows, I] and scales [rows, I/group]
// (requant 1: per-(row,128) power-of-two fp32 scales; 2: MX E8M0 bytes).
// Each intermediate pointer may be NULL.
ORC_API int orc_expert_mlp(const double* x_hat, int64_t rows, int64_t H, int64_t I, const double* w13,
                           const double* w2, int32_t requant, int32_t has_limit, double limit, double* y,
                           double* h_out, double* p_out, uint8_t* codes_out, void* scales_out, int32_t num_threads) {
  if (requant == RQ_BLOCK128 && I % 128) return fail("I must be a multiple of 128 for the FP8 requantisation");
  if (requant == RQ_MX && I % kMxGroup) return fail("I must be a multiple of 32 for MXFP8");
  const Weights W13{W_F64, w13, nullptr, 2 * I, H};
  const Weights W2{W_F64, w2, nullptr, H, I};
  const int nt = threads_or_default(num_threads);
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
  for (int64_t r = 0; r < rows; ++r) {
    MlpScratch s;
    expert_mlp_row(x_hat + r * H, W13, W2, H, I, requant, has_limit != 0, limit, y + r * H, s);
    if (h_out) std::copy(s.h.begin(), s.h.end(), h_out + r * 2 * I);
    if (p_out) std::copy(s.p.begin(), s.p.end(), p_out + r * I);
    if (codes_out && requant != RQ_NONE) std::copy(s.codes.begin(), s.codes.end(), codes_out + r * I);
    if (scales_out && requant == RQ_BLOCK128)
      for (int64_t g = 0; g < I / 128; ++g) static_cast<float*>(scales_out)[r * (I / 128) + g] = static_cast<float>(s.scales[g]);
    if (scales_out && requant == RQ_MX)
      for (int64_t g = 0; g < I / kMxGroup; ++g)
        static_cast<uint8_t*>(scales_out)[r * (I / kMxGroup) + g] = static_cast<uint8_t>(e8m0_of_pow2(s.scales[g]));
  }
  return 0;
}

namespace {

// The arguments every layer evaluation shares (see orc_moe_forward).
struct Layer {
  const double* x;
  int64_t n, H, I;
  int32_t topk;
  const int32_t* ids;
  const float* wts;
  int32_t wtype;
  const void* const* w13;
  const void* const* w13_scale;
  const void* const* w2;
  const void* const* w2_scale;
  int32_t first, count, router_weight_on_input, has_limit;
  double limit;
  int nt;
  int requant() const { return wtype == W_FP8_BLOCK128 ? RQ_BLOCK128 : wtype == W_MXFP8 ? RQ_MX : RQ_NONE; }
};

int check_layer(const Layer& L) {
  if (L.wtype < W_F64 || L.wtype > W_MXFP8) return fail("unknown weight type");
  if (L.router_weight_on_input && L.topk != 1) return fail("router_weight_on_input needs topk == 1");
  if (L.wtype == W_FP8_BLOCK128 && (L.H % 128 || L.I % 128)) return fail("H and I must be multiples of 128");
  if (L.wtype == W_MXFP8 && (L.H % kMxGroup || L.I % kMxGroup)) return fail("H and I must be multiples of 32");
  return 0;
}

int check_assignment(const Layer& L, int64_t a) {
  const int32_t e = L.ids[a] - L.first;
  if (!L.w13[e] || !L.w2[e] || (L.wtype >= W_FP8_BLOCK128 && (!L.w13_scale[e] || !L.w2_scale[e])))
    return fail("weights of expert " + std::to_string(L.ids[a]) + " not given");
  return 0;
}

// Each row's expert input x_hat: x itself, (the router weight on the input),
// then the activation quantisation of the FP8 paths (the GEMM1 input reading).
std::vector<double> expert_inputs(const Layer& L) {
  std::vector<double> x_hat(static_cast<size_t>(L.n * L.H));
  const int rq = L.requant();
#pragma omp parallel for schedule(static) num_threads(L.nt)
  for (int64_t t = 0; t < L.n; ++t) {
    std::vector<double> row(L.x + t * L.H, L.x + (t + 1) * L.H);
    if (L.router_weight_on_input) {
      const float w = L.wts[t];
      for (int64_t k = 0; k < L.H; ++k)
        row[k] = round_bf16(static_cast<double>(static_cast<float>(row[k]) * w));   // one fp32 product
    }
    double* xh = &x_hat[t * L.H];
    if (rq == RQ_NONE) {
      std::copy(row.begin(), row.end(), xh);
    } else {
      const int group = rq == RQ_MX ? kMxGroup : 128;
      std::vector<uint8_t> codes(group);
      for (int64_t g = 0; g < L.H / group; ++g) {
        const double scale = quantize_group_pow2(&row[g * group], group, codes.data());
        for (int j = 0; j < group; ++j) xh[g * group + j] = kE4m3.v[codes[j]] * scale;
      }
    }
  }
  return x_hat;
}

// The unweighted expert output of every listed assignment (flat index
// row * topk + slot), rows in list order.
std::vector<double> expert_outputs(const Layer& L, const std::vector<double>& x_hat, const std::vector<int64_t>& todo) {
  std::vector<double> y(todo.size() * static_cast<size_t>(L.H));
  const int rq = L.requant();
#pragma omp parallel for schedule(dynamic, 1) num_threads(L.nt)
  for (int64_t i = 0; i < static_cast<int64_t>(todo.size()); ++i) {
    const int64_t a = todo[i];
    const int32_t e = L.ids[a] - L.first;
    const bool scaled = L.wtype >= W_FP8_BLOCK128;
    const Weights W13{L.wtype, L.w13[e], scaled ? L.w13_scale[e] : nullptr, 2 * L.I, L.H};
    const Weights W2{L.wtype, L.w2[e], scaled ? L.w2_scale[e] : nullptr, L.H, L.I};
    MlpScratch s;
    expert_mlp_row(&x_hat[(a / L.topk) * L.H], W13, W2, L.H, L.I, rq, L.has_limit != 0, L.limit, &y[i * L.H], s);
  }
  return y;
}

}  // namespace

// The fused MoE layer on a set of token rows ([AWS] "Warum MoE-Kernel so
// wichtig sind": route, run the chosen experts, combine; [PPLX] "MoE
// Dispatch - Combine": the combine is a weighted accumulation).
//
//  x [n, H]: the token rows to evaluate (bf16 values); ids / wts [n, topk]:
//  their routing (global expert ids, fp32 weights).
//  wtype: 0 double values, 1 bf16 bit patterns, 2 E4M3 codes with fp32
//  128x128 block scales (x and the intermediate quantised per (row,128)),
//  3 MXFP8 codes with E8M0 per-32 scales (x and the intermediate MX-quantised).
//  w13[e] [2I, H], w2[e] [H, I] (and their scales) for e in [0, count): the
//  experts [first, first + count) of the layer; a pointer may be NULL for an
//  expert no row uses.
//  router_weight_on_input (reading; top-1 only): each row becomes
//  bf16(fp32(x) * fp32(w)) before the expert, whose output is not weighted.
//  out [n, H]: bf16 rounding of sum_j w[t,j] * y[t,j] over the assignments to
//  experts in the range (zero without any); y [n, topk, H] (may be NULL): each
//  assignment's unweighted expert output (zero for other ranks' experts).
ORC_API int orc_moe_forward(const double* x, int64_t n, int64_t H, int64_t I, int32_t topk, const int32_t* ids,
                            const float* wts, int32_t wtype, const void* const* w13, const void* const* w13_scale,
                            const void* const* w2, const void* const* w2_scale, int32_t first, int32_t count,
                            int32_t router_weight_on_input, int32_t has_limit, double limit, int32_t num_threads,
                            double* out, double* y_out) {
  const Layer L{x, n, H, I, topk, ids, wts, wtype, w13, w13_scale, w2, w2_scale, first, count,
                router_weight_on_input, has_limit, limit, threads_or_default(num_threads)};
  if (check_layer(L)) return -1;
  std::vector<int64_t> todo;                               // in (row, slot) order
  for (int64_t a = 0; a < n * topk; ++a) {
    const int32_t e = ids[a] - first;
    if (e < 0 || e >= count) continue;                     // another rank's expert
    if (check_assignment(L, a)) return -1;
    todo.push_back(a);
  }
  const std::vector<double> y = expert_outputs(L, expert_inputs(L), todo);
  // combine: out[t] = sum over slots j in order of w[t,j] * y[t,j], rounded once
  std::vector<int64_t> where(static_cast<size_t>(n * topk), -1);
  for (size_t i = 0; i < todo.size(); ++i) where[todo[i]] = static_cast<int64_t>(i);
#pragma omp parallel for schedule(static) num_threads(L.nt)
  for (int64_t t = 0; t < n; ++t) {
    for (int64_t k = 0; k < H; ++k) {
      double acc = 0.0;
      for (int32_t j = 0; j < topk; ++j) {
        const int64_t i = where[t * topk + j];
        if (i < 0) continue;
        const double w = router_weight_on_input ? 1.0 : static_cast<double>(wts[t * topk + j]);
        acc += w * y[i * H + k];
      }
      out[t * H + k] = round_bf16(acc);
    }
    if (y_out)
      for (int32_t j = 0; j < topk; ++j) {
        const int64_t i = where[t * topk + j];
        for (int64_t k = 0; k < H; ++k) y_out[(t * topk + j) * H + k] = i < 0 ? 0.0 : y[i * H + k];
      }
  }
  return 0;
}

// The unweighted expert output of chosen assignments only: the same layer
// arguments as orc_moe_forward, plus the list of flat assignment indices
// (row * topk + slot) to evaluate; y_rows [n_sel, H] in list order.  (Each
// expert output depends only on its own token row, its expert and the
// weights, so one expert's rows can be checked without the others.)
ORC_API int orc_assignment_outputs(const double* x, int64_t n, int64_t H, int64_t I, int32_t topk,
                                   const int32_t* ids, const float* wts, int32_t wtype, const void* const* w13,
                                   const void* const* w13_scale, const void* const* w2,
                                   const void* const* w2_scale, int32_t first, int32_t count,
                                   int32_t router_weight_on_input, int32_t has_limit, double limit,
                                   int32_t num_threads, int64_t n_sel, const int64_t* sel, double* y_rows) {
  const Layer L{x, n, H, I, topk, ids, wts, wtype, w13, w13_scale, w2, w2_scale, first, count,
                router_weight_on_input, has_limit, limit, threads_or_default(num_threads)};
  if (check_layer(L)) return -1;
  std::vector<int64_t> todo(sel, sel + n_sel);
  for (int64_t a : todo) {
    if (a < 0 || a >= n * topk) return fail("assignment index out of range");
    const int32_t e = ids[a] - first;
    if (e < 0 || e >= count) return fail("assignment of an expert outside the range");
    if (check_assignment(L, a)) return -1;
  }
  const std::vector<double> y = expert_outputs(L, expert_inputs(L), todo);
  std::copy(y.begin(), y.end(), y_rows);
  return 0;
}

// [PPLX] shards 128 experts over EP=4/8/16 ranks without saying how.
// Reading: rank r holds [floor(rE/N), floor((r+1)E/N)).
ORC_API int orc_expert_shards(int32_t E, int32_t world, int32_t* first, int32_t* count) {
  if (world < 1 || world > E) return fail("need 1 <= world_size <= E");
  for (int32_t r = 0; r < world; ++r) {
    first[r] = static_cast<int32_t>((static_cast<int64_t>(r) * E) / world);
    count[r] = static_cast<int32_t>((static_cast<int64_t>(r + 1) * E) / world) - first[r];
  }
  return 0;
}

// The all-reduce of the expert-parallel reading: the exact sum of the ranks'
// bf16 partials (double), rounded once to bf16.
ORC_API void orc_sum_round_bf16(const double* const* parts, int32_t nparts, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) {
    double acc = 0.0;
    for (int32_t r = 0; r < nparts; ++r) acc += parts[r][i];
    out[i] = round_bf16(acc);
  }
}
