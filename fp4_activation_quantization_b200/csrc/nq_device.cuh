// nq_device.cuh — device helpers shared by the sm_100a kernels of libnq.
//
// Format conversions use the hardware's packed converters
// (cvt.rn.satfinite.{e4m3x2,e5m2x2,e2m1x2}.f32, cvt.rn.bf16x2.f32):
// round to nearest even, saturate to the largest finite value.  Every other
// float operation is written with an explicit IEEE intrinsic (__fadd_rn,
// __fmul_rn, __fmaf_rn, __fdiv_rn, __frcp_rn, __fsqrt_rn) so that contraction
// or approximation can never change a rounding: results are identical on
// every schedule and reproducible on the CPU.
#pragma once

#include <cooperative_groups.h>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace nq {

constexpr unsigned kFull = 0xffffffffu;

// A compile-time bool passed to generic lambdas (decltype(tag)::value).
template <bool B>
struct BoolTag {
  static constexpr bool value = B;
};
constexpr float kE4M3Max = 448.0f;
constexpr float kE5M2Max = 57344.0f;
constexpr float kE2M1Max = 6.0f;

// ---------------------------------------------------------------- PDL -----
// Programmatic dependent launch: both are no-ops when the grid was launched
// without the programmatic-serialization attribute.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- bf16 ----
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }

__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float (&v)[8]) {
  v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x);
  v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
  v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z);
  v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}

// Two floats -> two bf16 (round to nearest even), `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<const uint16_t*>(&h);
}
__device__ __forceinline__ uint4 pack_bf16x8(const float (&v)[8]) {
  return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                    pack_bf16x2(v[6], v[7]));
}
__device__ __forceinline__ float round_bf16(float f) { return bf16_to_f32(f32_to_bf16(f)); }

// ---------------------------------------------------------------- e4m3 ----
// Four floats -> four e4m3 bytes, a0 in the lowest byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a0, float a1, float a2, float a3) {
  uint32_t out;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(out)
      : "f"(a0), "f"(a1), "f"(a2), "f"(a3));
  return out;
}
// One float -> its e4m3 code (one converter instruction; the pair's other
// half is e4m3(+0) = 0x00).
__device__ __forceinline__ uint32_t f32_to_e4m3(float a) {
  uint16_t h;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(h) : "f"(a), "f"(0.0f));
  return h;
}

// ------------------------------------------------------------ absmax -----
// max(m, |v_0|, ..., |v_7|) with three-input max.f32 (sm_100), half the
// instructions of a two-input chain; exact, and the same result.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float absmax8(const float2 (&v)[4], float m) {
#pragma unroll
  for (int i = 0; i < 4; ++i) m = fmax3(m, fabsf(v[i].x), fabsf(v[i].y));
  return m;
}

// ------------------------------------------------ bounded division ------
// RN(a / b) for one divisor b shared by many quotients, from r = RN(1 / b)
// (correctly rounded).  q0 = RN(a r) is within 1.5 ulp of a / b; each step
// t = q b - a (fma), q' = q + t (-r) (fma) is the FMA remainder correction of
// Markstein (IBM J. Res. Dev. 34(1), 1990; Muller et al., "Handbook of
// Floating-Point Arithmetic", FMA-based division).  The first step brings q
// within one ulp, and the second then rounds correctly while the remainders
// are normal.  Contract, for b in [2^-60, 2^100] and |a / b| <= 2^17 (the
// callers guarantee both): the result is RN(a / b) bit for bit when
// |a / b| >= 2^-24; smaller quotients keep the sign of a / b and stay below
// 2^-20, so their e4m3 / e5m2 code is the same signed zero.  The remainder is
// taken as q b - a (not a - q b) so that a zero quotient keeps the sign of a.
// nq_selftest_division checks this over every float32 dividend.
constexpr float kFastDivMinDivisor = 8.6736173798840355e-19f;  // 2^-60
constexpr float kFastDivMaxDivisor = 1.2676506002282294e30f;   // 2^100
__device__ __forceinline__ bool fast_div_ok(float b) { return b >= kFastDivMinDivisor && b <= kFastDivMaxDivisor; }
__device__ __forceinline__ float div_rn_by(float a, float b, float nr) {
  const float q0 = __fmul_rn(a, -nr);
  const float q1 = __fmaf_rn(__fmaf_rn(q0, b, -a), nr, q0);
  return __fmaf_rn(__fmaf_rn(q1, b, -a), nr, q1);
}
// Two lanes at once (packed fp32x2, each lane rounding as its scalar form).
__device__ __forceinline__ float2 div2_rn_by(float2 a, float2 b2, float2 nr2) {
  const float2 na = make_float2(-a.x, -a.y);
  const float2 q0 = __fmul2_rn(a, make_float2(-nr2.x, -nr2.y));
  const float2 q1 = __ffma2_rn(__ffma2_rn(q0, b2, na), nr2, q0);
  return __ffma2_rn(__ffma2_rn(q1, b2, na), nr2, q1);
}

// s = RN(amax / max) for the FP8 format's largest value (448 or 57344):
// the bounded division where its quotient lies in [2^-24, 2^17], else the
// library division; always the correctly rounded quotient.
template <bool E5>
__device__ __forceinline__ float fp8_scale_of(float amax) {
  constexpr float kMax = E5 ? 57344.0f : 448.0f;
  constexpr float kNegRcp = -(1.0f / kMax);
  constexpr float kLo = 5.9604645e-08f, kHi = 131072.0f;  // 2^-24, 2^17
  return (amax >= kMax * kLo && amax <= kMax * kHi) ? div_rn_by(amax, kMax, kNegRcp) : __fdiv_rn(amax, kMax);
}

// ------------------------------------------------------ group scales -----
// Store the scale s of group g (of n_groups) of a row.  Float layout: element
// row * rs + g * cs (row-major: rs = ld, cs = 1; column-major: rs = 1, cs =
// ld).  Packed UE8M0 (s a power of two in [2^-127, 2^127]): its biased exponent
// byte (the float's exponent field, 0 for the subnormal 2^-127) goes to byte
// g % 4 of the 32-bit word at byte offset row * rs + (g / 4) * cs; the group
// that ends a row also zeroes the word's unused bytes.
__device__ __forceinline__ void store_group_scale(float* base, int64_t rs, int64_t cs, bool packed, int64_t row,
                                                  int64_t g, int64_t n_groups, float s) {
  if (!packed) {
    base[row * rs + g * cs] = s;
    return;
  }
  uint8_t* w = reinterpret_cast<uint8_t*>(base) + row * rs + (g >> 2) * cs;
  w[g & 3] = uint8_t(__float_as_uint(s) >> 23);
  if (g == n_groups - 1)
    for (int j = int(g & 3) + 1; j < 4; ++j) w[j] = 0;
}

// ---------------------------------------------------------------- e5m2 ----
__device__ __forceinline__ uint32_t pack_e5m2x4(float a0, float a1, float a2, float a3) {
  uint32_t out;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e5m2x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e5m2x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(out)
      : "f"(a0), "f"(a1), "f"(a2), "f"(a3));
  return out;
}

// The FP8 output format as a compile-time choice (E5: e5m2, else e4m3).
template <bool E5>
__device__ __forceinline__ uint32_t pack_fp8x4(float a0, float a1, float a2, float a3) {
  if constexpr (E5) return pack_e5m2x4(a0, a1, a2, a3);
  else return pack_e4m3x4(a0, a1, a2, a3);
}
template <bool E5>
constexpr float fp8_max() { return E5 ? kE5M2Max : kE4M3Max; }

// e4m3 code (low byte of c) -> float, exact: the hardware converter widens
// e4m3 to f16 (every e4m3 value, NaN included, is an f16 value), then f16 ->
// f32.
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
  float f;
  asm("{\n\t.reg .b16 c8, lo, hi;\n\t.reg .b32 h2;\n\t"
      "cvt.u16.u32 c8, %1;\n\t"
      "cvt.rn.f16x2.e4m3x2 h2, c8;\n\t"
      "mov.b32 {lo, hi}, h2;\n\t"
      "cvt.f32.f16 %0, lo;\n\t}"
      : "=f"(f)
      : "r"(c & 0xFFu));
  return f;
}

// ---------------------------------------------------------------- e2m1 ----
// Eight floats -> eight e2m1 nibbles packed in 4 bytes; element 2i in the low
// nibble of byte i.
__device__ __forceinline__ uint32_t pack_e2m1x8(const float (&v)[8]) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

// --------------------------------------------------------------- UE8M0 ----
// Smallest power of two >= s, clamped to [2^-127, 2^127]; s <= 0 -> 2^-127.
__device__ __forceinline__ float ue8m0_ceil(float s) {
  if (!(s > 0.0f)) return __uint_as_float(0x00400000u);
  const uint32_t b = __float_as_uint(s);
  const int e = int((b >> 23) & 0xFFu);
  const uint32_t m = b & 0x7FFFFFu;
  int p;
  if (e == 0) p = -149 + (m == 1u ? 0 : 32 - __clz(int(m - 1u)));  // subnormal input
  else p = e - 127 + (m ? 1 : 0);
  p = p < -127 ? -127 : (p > 127 ? 127 : p);
  return p >= -126 ? __uint_as_float(uint32_t(p + 127) << 23) : __uint_as_float(1u << (p + 149));
}

// ---------------------------------------------------------- reductions ----
// Canonical row sum.  Thread t of a row group of T threads holds chunk
// partials for chunks t, t+T, t+2T, ... already combined (highest index bit
// first) into `v`.  The remaining levels of the pairwise tree over the chunk
// index are: across warps (warp w absorbs warp w + W/2, lane by lane, highest
// bit first), then inside the warp (xor butterfly 16, 8, 4, 2, 1; IEEE
// addition is commutative, so lane l and l^o compute the same value).  Every
// thread returns the row total.  `red` holds W*32 floats (unused for T == 32).
// For T > 32 the row is the whole CTA and this contains one __syncthreads().
template <int T>
__device__ __forceinline__ float row_sum(float v, float* red, int tid) {
  if constexpr (T > 32) {
    constexpr int W = T / 32;
    const int lane = tid & 31, w = tid >> 5;
    red[w * 32 + lane] = v;
    __syncthreads();
    float p[W];
#pragma unroll
    for (int i = 0; i < W; ++i) p[i] = red[i * 32 + lane];
#pragma unroll
    for (int h = W / 2; h >= 1; h >>= 1)
#pragma unroll
      for (int i = 0; i < h; ++i) p[i] = __fadd_rn(p[i], p[i + h]);
    v = p[0];
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

// Row maximum of non-negative floats (order-free; exact).  `red` holds W words.
template <int T>
__device__ __forceinline__ float row_max_nonneg(float v, uint32_t* red, int tid) {
  uint32_t u = __reduce_max_sync(kFull, __float_as_uint(v));
  if constexpr (T > 32) {
    constexpr int W = T / 32;
    if ((tid & 31) == 0) red[tid >> 5] = u;
    __syncthreads();
    u = 0;
#pragma unroll
    for (int i = 0; i < W; ++i) u = max(u, red[i]);
  }
  return __uint_as_float(u);
}

// ------------------------------------------------- rows over a cluster ----
// A row wider than one CTA can hold in registers is split over a cluster of NC
// CTAs (thread-block cluster; each CTA on its own SM).  CTA rank j of the
// cluster owns, in thread t, the chunks k * NC * T + j * T + t, so the chunk
// index's bits are, from the top: k (the thread's own slots), j (the CTA),
// the warp, the lane.  The canonical tree combines them in that order; the
// level over j runs here, through distributed shared memory: each CTA writes
// its partial into slot `rank` of every CTA's xred (NC x T floats), and after
// the cluster barrier combines the NC partials of its thread index from its
// own buffer (CTA j absorbs CTA j + NC/2, ..., highest bit first), so every
// CTA holds the same values afterwards.  Nothing remote is touched after the
// barrier.  The remote buffers must exist before the first remote write,
// which the kernel ensures (every CTA arrives on the cluster barrier at entry
// and waits on it before its first reduction).  Each xred is used by one
// reduction only (no reuse, so no barrier is needed before it is written).
// The cluster barrier is a hardware barrier that every thread of the cluster
// reaches on the same path; nothing here spins.
template <int T, int NC>
__device__ __forceinline__ float cluster_tree_sum(float v, float* xred, int tid) {
  if constexpr (NC == 1) {
    return v;
  } else {
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    const int rank = int(cl.block_rank());
#pragma unroll
    for (int j = 0; j < NC; ++j) *cl.map_shared_rank(xred + rank * T + tid, j) = v;
    cl.sync();
    float p[NC];
#pragma unroll
    for (int j = 0; j < NC; ++j) p[j] = xred[j * T + tid];
#pragma unroll
    for (int h = NC / 2; h >= 1; h >>= 1)
#pragma unroll
      for (int i = 0; i < h; ++i) p[i] = __fadd_rn(p[i], p[i + h]);
    return p[0];
  }
}

// Largest of the cluster's per-CTA values (non-negative floats as bits;
// order-free).  Pull form: each CTA publishes its value in its own xred[0]
// and after the barrier reads the NC values from the CTAs' buffers, so a
// kernel that calls it ends with one more cluster barrier before any CTA
// exits.  (Measured on B200 for the dynamic path, 2048 x 65536 ... 8192 x
// 20480: pushing the absmax into every CTA as well and leaving without that
// barrier was 5-7 % slower.)
template <int NC>
__device__ __forceinline__ uint32_t cluster_max_u32(uint32_t u, uint32_t* xred, int tid) {
  if constexpr (NC == 1) {
    return u;
  } else {
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    if (tid == 0) xred[0] = u;
    cl.sync();
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < NC; ++j) m = max(m, *cl.map_shared_rank(xred, j));
    return m;
  }
}

// Rank of this CTA in its cluster (0 without a cluster).
template <int NC>
__device__ __forceinline__ int cluster_rank() {
  if constexpr (NC == 1) return 0;
  else return int(cooperative_groups::this_cluster().block_rank());
}

}  // namespace nq
