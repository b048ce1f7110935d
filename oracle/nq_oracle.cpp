// nq_oracle.cpp — plain, slow, single-threaded CPU oracle of the fused
// residual-add + RMSNorm / LayerNorm + activation-quantization path.
//
// TEST INFRASTRUCTURE.  Only the tests, the package smoke check and the
// benchmark's CPU-baseline / reference arm may load this library.  It shares no
// code, header, table or constant with the CUDA path; both sides are fed the
// same seeded inputs and compared.
//
// Build: g++ -O2 -ffp-contract=off -fno-fast-math -fPIC -shared (x86-64: SSE
// float arithmetic, so every float operation below is one IEEE binary32
// operation rounded to nearest even; std::fma is the fused multiply-add).
//
// Sources followed (web pages, by title and section):
//  [P1] "Fusing RMSNorm and FP8 Quantization Under torch.compile" (netraruntime
//       blog): "Where norm+quant sits" (per-token e4m3 scale, single rounding
//       from fp32 registers vs double rounding through bf16), FAQ (residual
//       update is exact, bf16 normed output written identically).
//  [P2] FlashInfer PR #3962 "fused FP8 quantization output for LayerNorm":
//       Description (LayerNorm, scale applied as division out = normed/scale).
//  [P3] TensorRT-LLM PR #14848 "RMSNorm nvfp4 quant fusion for DS V3.2 /
//       Kimi-K2.5": Description (RMSNorm in registers -> packed E2M1 +
//       per-16-element E4M3 block scale), commit notes (row-strided input,
//       hidden % 16 == 0, static input_scale).
//  [P4] vLLM PR #61343 "per_token_group_quant_8bit: multiply by reciprocal
//       instead of dividing per element": Overview/Details (group of 128,
//       s = absmax/448, one reciprocal per group, UE8M0 power-of-two scales).
//  [P5] FlashInfer PR #2459 "RMSNorm/FusedRMSNorm + Quant kernels cuda graph
//       fixes": Changes table (scale is a one-element device tensor,
//       scale_inv = 1/scale[0]); review (raw input, not an fp8 value, is added
//       to the residual; 1/0 when scale is zero).
//
// Readings where the pages are silent (each is a choice of this oracle, and
// the CUDA path is held to it):
//  * the norm input is the fp32 sum r = RN(x + residual) (P1: values are held
//    in fp32 registers through both phases);
//  * rstd = RN(1 / RN(sqrt(RN(mean_sq + eps)))) with correctly rounded sqrt
//    and reciprocal; eps inside the square root; mean divides by d;
//  * y = RN(RN(r * rstd) * gamma) for RMSNorm and
//    y = fma(RN((r - mean) * rstd), gamma, beta) for LayerNorm;
//  * canonical sum order (see canonical_sum) so that a parallel reduction with
//    packed two-lane arithmetic can reproduce it exactly; OR_SUM_PLAIN
//    switches to float64 sequential sums;
//  * e4m3 / e5m2 / e2m1 encoders round to nearest, ties to even, and saturate
//    to the largest finite magnitude (448 / 57344 / 6); with e5m2 output the
//    dynamic and group scales divide absmax by 57344;
//  * NVFP4 global scale g is a dequantization multiplier (x ~ q * sf * g),
//    block scale sf = e4m3(RN(RN(amax / 6) / g)), element multiplier
//    m = RN(1 / RN(dec(sf) * g));
//  * UE8M0 scale = 2^ceil(log2 s) clamped to [2^-127, 2^127], zero -> 2^-127.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

// ---- flags of this oracle (its own values; not shared with the library) ----
constexpr uint32_t OR_DIV = 1u;             // quantize as RN(y / s)
constexpr uint32_t OR_RECIP = 2u;           // quantize as RN(y * RN(1 / s))
constexpr uint32_t OR_UE8M0 = 4u;           // power-of-two group scales
constexpr uint32_t OR_NORM_BF16_ROUND = 8u; // round y to bf16 before quantizing
constexpr uint32_t OR_SUM_PLAIN = 16u;      // float64 sequential sums
constexpr uint32_t OR_E5M2 = 32u;           // FP8 outputs in e5m2 instead of e4m3

constexpr float kE4M3Max = 448.0f;  // largest finite e4m3 magnitude (1.75 * 2^8)
constexpr float kE2M1Max = 6.0f;    // largest e2m1 magnitude (1.5 * 2^2)

inline uint32_t f2u(float f) { uint32_t u; std::memcpy(&u, &f, 4); return u; }
inline float u2f(uint32_t u) { float f; std::memcpy(&f, &u, 4); return f; }

// bf16 bit pattern -> float: exact (bf16 is the top half of binary32).
inline float bf16_to_f32(uint16_t b) { return u2f(uint32_t(b) << 16); }

// float -> bf16, round to nearest even on the 16 discarded bits; NaN stays NaN.
inline uint16_t f32_to_bf16(float f) {
  uint32_t u = f2u(f);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu))
    return uint16_t((u >> 16) | 0x0040u);
  uint32_t lsb = (u >> 16) & 1u;
  return uint16_t((u + 0x7FFFu + lsb) >> 16);
}

// ---- e4m3 (OCP FP8 E4M3FN): bias 7, 3 mantissa bits, no infinities, NaN
// only at S.1111.111, largest finite 448, smallest subnormal 2^-9. [P1] FAQ
// names the format; encoding rule: round to nearest even, saturate. ----
uint8_t e4m3_encode(float v) {
  const uint8_t sign = (f2u(v) >> 31) ? 0x80 : 0x00;
  if (std::isnan(v)) return uint8_t(sign | 0x7F);
  float a = std::fabs(v);
  if (a >= kE4M3Max) return uint8_t(sign | 0x7E);  // satfinite (inf included)
  int e;
  std::frexp(a, &e);          // a = f * 2^e, f in [0.5, 1)  =>  floor(log2 a) = e - 1
  int E = e - 1;
  if (a == 0.0f || E < -6) E = -6;  // subnormal range shares the quantum 2^-9
  // quantum (spacing) at a is 2^(E-3); scaling by a power of two is exact.
  float n = std::nearbyint(std::ldexp(a, 3 - E));  // default mode: ties to even
  if (E == -6 && n < 8.0f) return uint8_t(sign | uint8_t(n));  // subnormal or zero
  if (n == 16.0f) { n = 8.0f; E += 1; }
  // E <= 8 here; E == 8 with n == 15 would be 480, impossible since a < 448
  // rounds to at most 448 (ties at 464 would need a >= 448).
  return uint8_t(sign | uint8_t(((E + 7) << 3) | (int(n) - 8)));
}

float e4m3_decode(uint8_t c) {
  const float s = (c & 0x80) ? -1.0f : 1.0f;
  const int ex = (c >> 3) & 0xF, m = c & 7;
  if (ex == 15 && m == 7) return std::nanf("");
  if (ex == 0) return s * std::ldexp(float(m), -9);
  return s * std::ldexp(float(8 + m), ex - 10);
}

// ---- e5m2 (OCP FP8 E5M2): bias 15, 2 mantissa bits, largest finite 57344,
// smallest subnormal 2^-16; infinities and NaNs exist but a saturating
// conversion never produces an infinity.  [P2] Description: the output dtype
// may be e5m2.  Round to nearest even, saturate. ----
constexpr float kE5M2Max = 57344.0f;  // 1.75 * 2^15

uint8_t e5m2_encode(float v) {
  const uint8_t sign = (f2u(v) >> 31) ? 0x80 : 0x00;
  if (std::isnan(v)) return uint8_t(sign | 0x7F);
  float a = std::fabs(v);
  if (a >= kE5M2Max) return uint8_t(sign | 0x7B);  // satfinite (inf included)
  int e;
  std::frexp(a, &e);
  int E = e - 1;
  if (a == 0.0f || E < -14) E = -14;  // subnormal range: quantum 2^-16
  float n = std::nearbyint(std::ldexp(a, 2 - E));  // quantum 2^(E-2); ties to even
  if (E == -14 && n < 4.0f) return uint8_t(sign | uint8_t(n));
  if (n == 8.0f) { n = 4.0f; E += 1; }
  return uint8_t(sign | uint8_t(((E + 15) << 2) | (int(n) - 4)));
}

float e5m2_decode(uint8_t c) {
  const float s = (c & 0x80) ? -1.0f : 1.0f;
  const int ex = (c >> 2) & 0x1F, m = c & 3;
  if (ex == 31) return m ? std::nanf("") : s * INFINITY;
  if (ex == 0) return s * std::ldexp(float(m), -16);
  return s * std::ldexp(float(4 + m), ex - 17);
}

// The FP8 output format of a call: e4m3 by default, e5m2 with OR_E5M2.
struct Fp8Out {
  bool e5m2;
  float max() const { return e5m2 ? kE5M2Max : kE4M3Max; }
  uint8_t encode(float v) const { return e5m2 ? e5m2_encode(v) : e4m3_encode(v); }
};

// ---- e2m1 (FP4): bias 1, 1 mantissa bit; magnitudes {0,.5,1,1.5,2,3,4,6}.
// [P3] Description: packed E2M1 elements. Round to nearest even, saturate. ----
uint8_t e2m1_encode(float v) {
  const uint8_t sign = (f2u(v) >> 31) ? 0x8 : 0x0;
  if (std::isnan(v)) return uint8_t(sign | 0x7);  // no NaN in e2m1: saturate
  float a = std::fabs(v);
  if (a >= kE2M1Max) return uint8_t(sign | 0x7);
  if (a < 2.0f) {  // quantum 0.5: codes 0..3 are 0, .5, 1, 1.5; n == 4 is 2.0 (code 4)
    float n = std::nearbyint(a * 2.0f);
    return uint8_t(sign | uint8_t(n));
  }
  if (a < 4.0f) {  // quantum 1: 2 -> code 4, 3 -> code 5, 4 -> code 6
    float n = std::nearbyint(a);
    return uint8_t(sign | uint8_t(int(n) + 2));
  }
  float n = std::nearbyint(a * 0.5f);  // quantum 2: 4 -> code 6, 6 -> code 7
  return uint8_t(sign | uint8_t(int(n) + 4));
}

float e2m1_decode(uint8_t c) {
  static const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  return ((c & 0x8) ? -1.0f : 1.0f) * mag[c & 7];
}

// ---- UE8M0: the smallest power of two >= s ([P4] Details: with such a scale
// the reciprocal is exact, so division and multiplication agree); zero maps
// to 2^-127. ----
float ue8m0_ceil(float s) {
  if (!(s > 0.0f)) return std::ldexp(1.0f, -127);
  int e;
  float f = std::frexp(s, &e);  // s = f * 2^e, f in [0.5, 1)
  int p = (f == 0.5f) ? e - 1 : e;
  if (p < -127) p = -127;
  if (p > 127) p = 127;
  return std::ldexp(1.0f, p);
}

// ---- canonical sum of a row ----
// The pages fix no summation order.  The oracle fixes one that a parallel
// reduction with packed two-lane float arithmetic can reproduce bit for bit:
// elements are cut into chunks of 8 consecutive values (the last one padded
// with +0); inside a chunk two accumulators, one for the even positions
// (0, 2, 4, 6) and one for the odd positions (1, 3, 5, 7), start at +0 and take
// their four values in order (acc = RN(acc + v) for a sum, acc = fma(v, v, acc)
// for a sum of squares); the chunk partial is RN(even + odd).  Chunk count is
// padded with +0 partials to a power of two P; then for half = P/2, P/4, ...,
// 1: p[c] = RN(p[c] + p[c + half]) for every c < half.  No partial is ever -0
// (they start at +0), so extra +0 padding never changes the result.
float canonical_sum(const float* v, int64_t n, bool squares) {
  const int64_t C = (n + 7) / 8;
  int64_t P = 1;
  while (P < C) P *= 2;
  std::vector<float> p(size_t(P), 0.0f);
  for (int64_t c = 0; c < C; ++c) {
    float acc[2] = {0.0f, 0.0f};
    for (int64_t i = 8 * c; i < 8 * c + 8 && i < n; ++i) {
      float& a = acc[(i - 8 * c) & 1];
      a = squares ? std::fma(v[i], v[i], a) : a + v[i];
    }
    p[size_t(c)] = acc[0] + acc[1];
  }
  for (int64_t half = P / 2; half >= 1; half /= 2)
    for (int64_t c = 0; c < half; ++c) p[size_t(c)] = p[size_t(c)] + p[size_t(c + half)];
  return p[0];
}

// float64 sequential sum rounded once to float: the plain definition.
float plain_sum(const float* v, int64_t n, bool squares) {
  double acc = 0.0;
  for (int64_t i = 0; i < n; ++i) acc += squares ? double(v[i]) * double(v[i]) : double(v[i]);
  return float(acc);
}

inline float row_sum(const float* v, int64_t n, bool squares, uint32_t flags) {
  return (flags & OR_SUM_PLAIN) ? plain_sum(v, n, squares) : canonical_sum(v, n, squares);
}

// rstd from a mean square (or variance): RN(1 / RN(sqrt(RN(ms + eps)))).
inline float rstd_of(float ms, float eps) {
  float t = ms + eps;
  float sq = std::sqrt(t);
  return 1.0f / sq;
}

// Residual add ([P1] TL;DR and FAQ; [P5] review: the raw input is added):
// r = RN(x + residual) in fp32; residual_out = bf16(r).  Without a residual
// r = x.  Then RMSNorm: y = RN(RN(r * rstd) * gamma), rstd from the mean of r^2.
void rms_row(const uint16_t* x, const uint16_t* res_in, uint16_t* res_out,
             const uint16_t* gamma, int64_t d, float eps, uint32_t flags,
             std::vector<float>& r, std::vector<float>& y) {
  r.resize(size_t(d));
  y.resize(size_t(d));
  for (int64_t i = 0; i < d; ++i) {
    float xv = bf16_to_f32(x[i]);
    r[size_t(i)] = res_in ? xv + bf16_to_f32(res_in[i]) : xv;
  }
  if (res_out)
    for (int64_t i = 0; i < d; ++i) res_out[i] = f32_to_bf16(r[size_t(i)]);
  float ss = row_sum(r.data(), d, true, flags);
  float ms = ss / float(d);
  float rstd = rstd_of(ms, eps);
  for (int64_t i = 0; i < d; ++i) y[size_t(i)] = (r[size_t(i)] * rstd) * bf16_to_f32(gamma[i]);
  if (flags & OR_NORM_BF16_ROUND)  // the unfused pipeline's first rounding ([P1])
    for (int64_t i = 0; i < d; ++i) y[size_t(i)] = bf16_to_f32(f32_to_bf16(y[size_t(i)]));
}

// LayerNorm ([P2] Description): mean, biased variance of the centred values,
// y = fma(RN((r - mean) * rstd), gamma, beta) with fp32 gamma and beta.
void ln_row(const uint16_t* x, const float* gamma, const float* beta, int64_t d, float eps,
            uint32_t flags, std::vector<float>& c, std::vector<float>& y) {
  c.resize(size_t(d));
  y.resize(size_t(d));
  for (int64_t i = 0; i < d; ++i) c[size_t(i)] = bf16_to_f32(x[i]);
  float mean = row_sum(c.data(), d, false, flags) / float(d);
  for (int64_t i = 0; i < d; ++i) c[size_t(i)] = c[size_t(i)] - mean;
  float var = row_sum(c.data(), d, true, flags) / float(d);
  float rstd = rstd_of(var, eps);
  for (int64_t i = 0; i < d; ++i) y[size_t(i)] = std::fma(c[size_t(i)] * rstd, gamma[i], beta[i]);
  if (flags & OR_NORM_BF16_ROUND)
    for (int64_t i = 0; i < d; ++i) y[size_t(i)] = bf16_to_f32(f32_to_bf16(y[size_t(i)]));
}

inline bool use_div(uint32_t flags, bool default_div) {
  if (flags & OR_DIV) return true;
  if (flags & OR_RECIP) return false;
  return default_div;
}

}  // namespace

extern "C" {

int oracle_version(void) { return 1; }

void oracle_bf16_from_f32(const float* in, uint16_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16(in[i]);
}
void oracle_e4m3_encode(const float* in, uint8_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_encode(in[i]);
}
void oracle_e4m3_decode(const uint8_t* in, float* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_decode(in[i]);
}
void oracle_e5m2_encode(const float* in, uint8_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = e5m2_encode(in[i]);
}
void oracle_e5m2_decode(const uint8_t* in, float* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = e5m2_decode(in[i]);
}
void oracle_e2m1_encode(const float* in, uint8_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = e2m1_encode(in[i]);
}
void oracle_e2m1_decode(const uint8_t* in, float* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = e2m1_decode(in[i]);
}
void oracle_ue8m0_ceil(const float* in, float* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = ue8m0_ceil(in[i]);
}
float oracle_canonical_sum(const float* v, int64_t n, int squares) {
  return canonical_sum(v, n, squares != 0);
}

// The fp32 normalized rows y [M, d] (RMSNorm, optional residual), before any
// quantization.  Used to derive an NVFP4 global scale and by the numerics pins.
void oracle_rms_y(const uint16_t* x, int64_t ld_x, const uint16_t* res_in, int64_t ld_res,
                  const uint16_t* gamma, float* y_out, int64_t ld_y, int64_t M, int64_t d,
                  float eps, uint32_t flags) {
  std::vector<float> r, y;
  for (int64_t m = 0; m < M; ++m) {
    rms_row(x + m * ld_x, res_in ? res_in + m * ld_res : nullptr, nullptr, gamma, d, eps,
            flags, r, y);
    std::memcpy(y_out + m * ld_y, y.data(), size_t(d) * 4);
  }
}

void oracle_ln_y(const uint16_t* x, int64_t ld_x, const float* gamma, const float* beta,
                 float* y_out, int64_t ld_y, int64_t M, int64_t d, float eps, uint32_t flags) {
  std::vector<float> c, y;
  for (int64_t m = 0; m < M; ++m) {
    ln_row(x + m * ld_x, gamma, beta, d, eps, flags, c, y);
    std::memcpy(y_out + m * ld_y, y.data(), size_t(d) * 4);
  }
}

// Fused residual-add + RMSNorm + dynamic per-token e4m3 ([P1]; per-token
// scale s = absmax(y) / 448).  Default quantizes by exact division RN(y / s)
// ([P4] Details: per-token FP8 keeps per-element division); OR_RECIP
// multiplies by RN(1 / s).  A zero row (s == 0) yields the signed zeros of y.
int oracle_fused_add_rmsnorm_quant_fp8(const uint16_t* x, int64_t ld_x, const uint16_t* res_in,
                                       uint16_t* res_out, int64_t ld_res, const uint16_t* gamma,
                                       uint8_t* q, int64_t ld_q, float* scale_out,
                                       uint16_t* norm_out, int64_t ld_norm, int64_t M, int64_t d,
                                       float eps, uint32_t flags) {
  const bool div = use_div(flags, true);
  const Fp8Out fmt{(flags & OR_E5M2) != 0};
  std::vector<float> r, y;
  for (int64_t m = 0; m < M; ++m) {
    rms_row(x + m * ld_x, res_in ? res_in + m * ld_res : nullptr,
            res_out ? res_out + m * ld_res : nullptr, gamma, d, eps, flags, r, y);
    if (norm_out)
      for (int64_t i = 0; i < d; ++i) norm_out[m * ld_norm + i] = f32_to_bf16(y[size_t(i)]);
    float amax = 0.0f;
    for (int64_t i = 0; i < d; ++i) amax = std::fmax(amax, std::fabs(y[size_t(i)]));
    const float s = amax / fmt.max();
    scale_out[m] = s;
    const float inv = 1.0f / s;
    for (int64_t i = 0; i < d; ++i) {
      float t = (s == 0.0f) ? y[size_t(i)] : (div ? y[size_t(i)] / s : y[size_t(i)] * inv);
      q[m * ld_q + i] = fmt.encode(t);
    }
  }
  return 0;
}

// RMSNorm (optional residual) + e4m3 with a static scale read from device
// memory ([P5] Changes: scale is a one-element tensor, the kernel uses
// scale_inv = 1 / scale[0]).  Default multiplies by RN(1 / scale); OR_DIV
// divides.  scale == 0 follows IEEE (inf / NaN then saturate / NaN code).
int oracle_rmsnorm_quant_fp8_static(const uint16_t* x, int64_t ld_x, const uint16_t* res_in,
                                    uint16_t* res_out, int64_t ld_res, const uint16_t* gamma,
                                    float scale, uint8_t* q, int64_t ld_q, uint16_t* norm_out,
                                    int64_t ld_norm, int64_t M, int64_t d, float eps,
                                    uint32_t flags) {
  const bool div = use_div(flags, false);
  const Fp8Out fmt{(flags & OR_E5M2) != 0};
  const float inv = 1.0f / scale;
  std::vector<float> r, y;
  for (int64_t m = 0; m < M; ++m) {
    rms_row(x + m * ld_x, res_in ? res_in + m * ld_res : nullptr,
            res_out ? res_out + m * ld_res : nullptr, gamma, d, eps, flags, r, y);
    if (norm_out)
      for (int64_t i = 0; i < d; ++i) norm_out[m * ld_norm + i] = f32_to_bf16(y[size_t(i)]);
    for (int64_t i = 0; i < d; ++i)
      q[m * ld_q + i] = fmt.encode(div ? y[size_t(i)] / scale : y[size_t(i)] * inv);
  }
  return 0;
}

// LayerNorm + e4m3 static scale ([P2] Description: out = normed / scale).
// Same scale convention and defaults as the RMSNorm static path.
int oracle_layernorm_quant_fp8(const uint16_t* x, int64_t ld_x, const float* gamma,
                               const float* beta, float scale, uint8_t* q, int64_t ld_q,
                               int64_t M, int64_t d, float eps, uint32_t flags) {
  const bool div = use_div(flags, false);
  const Fp8Out fmt{(flags & OR_E5M2) != 0};
  const float inv = 1.0f / scale;
  std::vector<float> c, y;
  for (int64_t m = 0; m < M; ++m) {
    ln_row(x + m * ld_x, gamma, beta, d, eps, flags, c, y);
    for (int64_t i = 0; i < d; ++i)
      q[m * ld_q + i] = fmt.encode(div ? y[size_t(i)] / scale : y[size_t(i)] * inv);
  }
  return 0;
}

// Per-token-group e4m3 ([P4] Overview/Details): for each group of `group`
// consecutive elements of a row, s = RN(absmax / 448) (UE8M0: the next power
// of two); default quantizes as RN(x * RN(1 / s)); OR_DIV divides.  A zero
// group in fp32 mode writes s = 0 and the signed zeros of x.
int oracle_per_token_group_quant_fp8(const uint16_t* x, int64_t ld_x, uint8_t* q, int64_t ld_q,
                                     float* scales, int64_t ld_s, int64_t M, int64_t K,
                                     int32_t group, uint32_t flags) {
  if (group <= 0 || K % group) return 1;
  const bool div = use_div(flags, false);
  const bool ue8m0 = (flags & OR_UE8M0) != 0;
  const Fp8Out fmt{(flags & OR_E5M2) != 0};
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t g = 0; g < K / group; ++g) {
      const uint16_t* xs = x + m * ld_x + g * group;
      float amax = 0.0f;
      for (int32_t i = 0; i < group; ++i) amax = std::fmax(amax, std::fabs(bf16_to_f32(xs[i])));
      float s = amax / fmt.max();
      if (ue8m0) s = ue8m0_ceil(s);
      scales[m * ld_s + g] = s;
      const float inv = (s == 0.0f) ? 0.0f : 1.0f / s;
      for (int32_t i = 0; i < group; ++i) {
        float v = bf16_to_f32(xs[i]);
        float t = (s == 0.0f) ? v : (div ? v / s : v * inv);
        q[m * ld_q + g * group + i] = fmt.encode(t);
      }
    }
  }
  return 0;
}

// RMSNorm (optional residual) + per-token-group e4m3 ([P4] Details: the fused
// RMSNorm + group-quant path multiplies by the group scale's reciprocal, the
// same numerics as the standalone group quantizer): y as in the other RMSNorm
// calls, then per group of `group` consecutive y values s = RN(absmax / 448)
// (UE8M0: next power of two), q = e4m3(RN(y * RN(1 / s))) (OR_DIV: RN(y / s));
// a zero fp32 group scale stores the signed zeros of y.
int oracle_rmsnorm_quant_fp8_group(const uint16_t* x, int64_t ld_x, const uint16_t* res_in,
                                   uint16_t* res_out, int64_t ld_res, const uint16_t* gamma,
                                   uint8_t* q, int64_t ld_q, float* scales, int64_t ld_s,
                                   uint16_t* norm_out, int64_t ld_norm, int64_t M, int64_t d,
                                   int32_t group, float eps, uint32_t flags) {
  if (group <= 0 || d % group) return 1;
  const bool div = use_div(flags, false);
  const bool ue8m0 = (flags & OR_UE8M0) != 0;
  const Fp8Out fmt{(flags & OR_E5M2) != 0};
  std::vector<float> r, y;
  for (int64_t m = 0; m < M; ++m) {
    rms_row(x + m * ld_x, res_in ? res_in + m * ld_res : nullptr,
            res_out ? res_out + m * ld_res : nullptr, gamma, d, eps, flags, r, y);
    if (norm_out)
      for (int64_t i = 0; i < d; ++i) norm_out[m * ld_norm + i] = f32_to_bf16(y[size_t(i)]);
    for (int64_t g = 0; g < d / group; ++g) {
      const float* ys = y.data() + g * group;
      float amax = 0.0f;
      for (int32_t i = 0; i < group; ++i) amax = std::fmax(amax, std::fabs(ys[i]));
      float s = amax / fmt.max();
      if (ue8m0) s = ue8m0_ceil(s);
      scales[m * ld_s + g] = s;
      const float inv = (s == 0.0f) ? 0.0f : 1.0f / s;
      for (int32_t i = 0; i < group; ++i) {
        float t = (s == 0.0f) ? ys[i] : (div ? ys[i] / s : ys[i] * inv);
        q[m * ld_q + g * group + i] = fmt.encode(t);
      }
    }
  }
  return 0;
}

// RMSNorm (optional residual) + NVFP4 ([P3] Description and commit notes):
// per block of 16 consecutive elements, sf = e4m3(RN(RN(amax / 6) / g)),
// element multiplier m = RN(1 / RN(dec(sf) * g)) (0 when that product is 0),
// code = e2m1(RN(y * m)); element 2i goes to the low nibble of byte i.
// Default scale handling is by reciprocal; OR_DIV quantizes as RN(y / S).
int oracle_rmsnorm_quant_nvfp4(const uint16_t* x, int64_t ld_x, const uint16_t* res_in,
                               uint16_t* res_out, int64_t ld_res, const uint16_t* gamma,
                               float g, uint8_t* q, int64_t ld_q, uint8_t* sf, int64_t ld_sf,
                               uint16_t* norm_out, int64_t ld_norm, int64_t M, int64_t d,
                               float eps, uint32_t flags) {
  if (d % 16) return 1;
  const bool div = use_div(flags, false);
  std::vector<float> r, y;
  for (int64_t m = 0; m < M; ++m) {
    rms_row(x + m * ld_x, res_in ? res_in + m * ld_res : nullptr,
            res_out ? res_out + m * ld_res : nullptr, gamma, d, eps, flags, r, y);
    if (norm_out)
      for (int64_t i = 0; i < d; ++i) norm_out[m * ld_norm + i] = f32_to_bf16(y[size_t(i)]);
    for (int64_t b = 0; b < d / 16; ++b) {
      float amax = 0.0f;
      for (int i = 0; i < 16; ++i) amax = std::fmax(amax, std::fabs(y[size_t(16 * b + i)]));
      const uint8_t code = e4m3_encode((amax / kE2M1Max) / g);
      sf[m * ld_sf + b] = code;
      const float S = e4m3_decode(code) * g;
      const float mult = (S == 0.0f) ? 0.0f : 1.0f / S;  // a zero block scale zeroes the block
      for (int i = 0; i < 16; i += 2) {
        float v0 = y[size_t(16 * b + i)], v1 = y[size_t(16 * b + i + 1)];
        float t0 = (div && S != 0.0f) ? v0 / S : v0 * mult;
        float t1 = (div && S != 0.0f) ? v1 / S : v1 * mult;
        q[m * ld_q + (16 * b + i) / 2] = uint8_t(e2m1_encode(t0) | (e2m1_encode(t1) << 4));
      }
    }
  }
  return 0;
}

// ---- GEMM-ready scale layouts ([P3] Description and commit notes: the
// production NVFP4 quantizer writes its block scales in the swizzled layout
// that block-scaled GEMMs read, with padding left uninitialized) ----
//
// Swizzled layout (the 128 x 4 scale-factor tile of block-scaled tensor-core
// MMA in NVIDIA's public PTX ISA and cuBLAS documentation): the scale matrix
// [rows, n] is cut into tiles of 128 rows x 4 columns, each stored whole as
// 512 bytes; tiles are ordered by row tile, and within a row tile by column
// tile.  Inside a tile, row r (0..127) and column c (0..3) sit at byte
// 16 * (r % 32) + 4 * (r / 32) + c.  Rows pad to a multiple of 128 and columns
// to a multiple of 4; padding bytes are zero here (a defined value).
int64_t oracle_sf_swizzled_size(int64_t rows, int64_t n) {
  return ((rows + 127) / 128 * 128) * ((n + 3) / 4 * 4);
}

void oracle_sf_swizzle(const uint8_t* sf, int64_t ld_sf, int64_t rows, int64_t n, uint8_t* out) {
  const int64_t col_tiles = (n + 3) / 4;
  std::memset(out, 0, size_t(oracle_sf_swizzled_size(rows, n)));
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < n; ++c) {
      const int64_t tile = (r / 128) * col_tiles + c / 4;
      const int64_t rr = r % 128, cc = c % 4;
      out[tile * 512 + 16 * (rr % 32) + 4 * (rr / 32) + cc] = sf[r * ld_sf + c];
    }
}

// Group-scale layouts for per-token-group FP8 GEMMs.  s is the row-major
// [M, G] float32 result.  col_major: element (m, g) at g * ld + m (M-major, as
// a GEMM reading one k-block's scales for many tokens wants).  packed (UE8M0
// scales only): the exponent byte e + 127 of s = 2^e, four consecutive groups
// of a row per 32-bit word (group 4j + b in byte b, bytes past G zero); word
// (m, j) at m * ld + j, or at j * ld + m when col_major.  Returns 0, or -1 if
// packed and a scale is not a power of two in [2^-127, 2^127].
int oracle_group_scales_layout(const float* s, int64_t M, int64_t G, int col_major, int packed, int64_t ld,
                               void* out) {
  if (!packed) {
    float* o = static_cast<float*>(out);
    for (int64_t m = 0; m < M; ++m)
      for (int64_t g = 0; g < G; ++g) o[col_major ? g * ld + m : m * ld + g] = s[m * G + g];
    return 0;
  }
  uint32_t* o = static_cast<uint32_t*>(out);
  const int64_t W = (G + 3) / 4;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t j = 0; j < W; ++j) {
      uint32_t word = 0;
      for (int64_t b = 0; b < 4 && 4 * j + b < G; ++b) {
        const float v = s[m * G + 4 * j + b];
        int e2 = 0;
        const float f = std::frexp(v, &e2);  // v = f * 2^e2, f in [0.5, 1)
        const int e = e2 - 1;
        if (!(f == 0.5f) || e < -127 || e > 127) return -1;
        word |= uint32_t(e + 127) << (8 * b);
      }
      o[col_major ? j * ld + m : m * ld + j] = word;
    }
  return 0;
}

}  // extern "C"
