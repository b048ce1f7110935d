// nq_group.cu — per-token-group FP8 quantization of raw bf16 activations
// (vLLM PR #61343 "per_token_group_quant_8bit: multiply by reciprocal instead
// of dividing per element": Overview and Details).
//
// Per group of GROUP consecutive elements of a row: s = RN(absmax / max)
// (max = 448 for e4m3, 57344 for e5m2 (E5); UE8M0: the smallest power of two
// >= s), one correctly rounded reciprocal per group,
// q = fp8(RN(x * RN(1 / s))) (NQ_FLAG_SCALE_DIV: RN(x / s)).
//
// Mapping: the activations are a flat list of G = M * K / GROUP groups.  A
// group (GROUP / 8 chunks of 16 bytes) is owned by a team of TPG lanes; lane j
// of the team takes chunks j, j + TPG, j + 2 TPG, ..., so at each load step a
// team reads TPG consecutive chunks (TPG * 16 contiguous bytes, whole 32-byte
// sectors for TPG >= 2) and a warp reads 32 / TPG such runs.  The group's
// scale (a correctly rounded division and reciprocal) is paid once per lane
// for GROUP / TPG elements, so small teams amortize it; the absmax is a max
// over the lane's elements, then an xor-butterfly inside the team.  Each
// thread handles U groups, all loads issued first.
#include "nq_device.cuh"
#include "nq_internal.h"

namespace nq {

// Register budget: the lane's raw chunks (4 registers each, U groups) plus 32
// working registers, at least 48, so that ptxas fits more CTAs per SM (the
// kernel waits on its loads).  Measured on B200 for the default schedule
// (teams of four lanes, one group per thread: 48 registers, 5 CTAs per SM,
// was 56 and 4): 32768 x 4096 70.5 -> 65.6 us, 65536 x 2816 95.1 -> 88.7 us,
// UE8M0 and e5m2 alike; the copies with strided scale layouts spill a few
// words and still gain 2-3 %.
template <int GROUP, int TPG, int U>
constexpr int group_min_blocks() {
  constexpr int cap = 4 * (GROUP / 8 / TPG) * U + 32;
  constexpr int blocks = 65536 / (kGroupThreads * (cap < 48 ? 48 : cap));
  return blocks < 1 ? 1 : blocks;
}

template <int GROUP, int TPG, int U, bool VEC, bool E5, bool LAYOUT>
__global__ void __launch_bounds__(kGroupThreads, (group_min_blocks<GROUP, TPG, U>())) group_kernel(const GroupArgs a) {
  constexpr int CPG = GROUP / 8;             // chunks per group
  constexpr int CPL = CPG / TPG;             // chunks per lane
  constexpr int SLOT = kGroupThreads / TPG;  // groups per CTA per unit
  static_assert(CPG % TPG == 0, "team size divides the group's chunks");
  const int lane_g = int(threadIdx.x) % TPG;
  const int slot = int(threadIdx.x) / TPG;
  const int64_t base = int64_t(blockIdx.x) * SLOT * U;
  const bool div = (a.flags & kFlagDiv) != 0;
  const bool ue8m0 = (a.flags & kFlagUe8m0) != 0;

  griddep_wait();

  uint4 raw[U][CPL];
  int64_t row[U], cg[U];
  bool ok[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int64_t g = base + int64_t(u) * SLOT + slot;
    ok[u] = g < a.G;
    row[u] = !ok[u] ? 0
             : a.row_magic ? int64_t((uint64_t(uint32_t(g)) * a.row_magic) >> a.row_shift)
                           : g / a.groups_per_row;
    cg[u] = ok[u] ? g - row[u] * a.groups_per_row : 0;
    const uint16_t* src = a.x + row[u] * a.ld_x + cg[u] * GROUP;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
      const int c = lane_g + j * TPG;
      if constexpr (VEC) {
        raw[u][j] = ok[u] ? __ldcs(reinterpret_cast<const uint4*>(src + 8 * c)) : make_uint4(0u, 0u, 0u, 0u);
      } else {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          w[e] = ok[u] ? (uint32_t(src[8 * c + 2 * e]) | (uint32_t(src[8 * c + 2 * e + 1]) << 16)) : 0u;
        raw[u][j] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  griddep_launch_dependents();

#pragma unroll
  for (int u = 0; u < U; ++u) {
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
      const uint4 w = raw[u][j];
      const float2 v[4] = {make_float2(bf16_lo(w.x), bf16_hi(w.x)), make_float2(bf16_lo(w.y), bf16_hi(w.y)),
                           make_float2(bf16_lo(w.z), bf16_hi(w.z)), make_float2(bf16_lo(w.w), bf16_hi(w.w))};
      m = absmax8(v, m);
    }
#pragma unroll
    for (int o = TPG / 2; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    float s = fp8_scale_of<E5>(m);
    if (ue8m0) s = ue8m0_ceil(s);
    const float inv = (s == 0.0f) ? 0.0f : __frcp_rn(s);
    const float2 inv2 = make_float2(inv, inv);
    uint8_t* dst = a.q + row[u] * a.ld_q + cg[u] * GROUP;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
      const int c = lane_g + j * TPG;
      const uint4 w = raw[u][j];
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
      float t[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 x2 = make_float2(bf16_lo(ww[e]), bf16_hi(ww[e]));
        if (div && s != 0.0f) {
          t[2 * e] = __fdiv_rn(x2.x, s);
          t[2 * e + 1] = __fdiv_rn(x2.y, s);
        } else {
          const float2 q2 = __fmul2_rn(x2, inv2);
          t[2 * e] = q2.x;
          t[2 * e + 1] = q2.y;
        }
      }
      const uint32_t lo = pack_fp8x4<E5>(t[0], t[1], t[2], t[3]);
      const uint32_t hi = pack_fp8x4<E5>(t[4], t[5], t[6], t[7]);
      if (ok[u]) {
        if constexpr (VEC) {
          *reinterpret_cast<uint2*>(dst + 8 * c) = make_uint2(lo, hi);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) dst[8 * c + e] = uint8_t((e < 4 ? lo : hi) >> (8 * (e & 3)));
        }
      }
    }
    if (ok[u] && lane_g == 0) {
      if constexpr (LAYOUT)  // column-major or packed UE8M0
        store_group_scale(a.s, a.ld_s, a.cs_s, (a.flags & kFlagScalesPacked) != 0, row[u], cg[u], a.groups_per_row,
                          s);
      else
        a.s[row[u] * a.ld_s + cg[u]] = s;
    }
  }
}

namespace {
struct GroupTableHolder {
  GroupTable t;
  GroupTableHolder() {
    for (auto& f : t)
      for (auto& l : f)
        for (auto& x : l)
          for (auto& y : x)
            for (auto& z : y)
              for (auto& w : z) w = nullptr;
#define NQ_GROUP_FL(F, L, GI, G, TI, TPG, UI, U)                                                 \
  t[F][L][GI][TI][UI][0] = reinterpret_cast<const void*>(&group_kernel<G, TPG, U, false, F, L>); \
  t[F][L][GI][TI][UI][1] = reinterpret_cast<const void*>(&group_kernel<G, TPG, U, true, F, L>);
#define NQ_GROUP(GI, G, TI, TPG, UI, U)                                                          \
  NQ_GROUP_FL(false, false, GI, G, TI, TPG, UI, U) NQ_GROUP_FL(true, false, GI, G, TI, TPG, UI, U) \
  NQ_GROUP_FL(false, true, GI, G, TI, TPG, UI, U) NQ_GROUP_FL(true, true, GI, G, TI, TPG, UI, U)
    // group 64 (8 chunks): teams of 2, 4, 8 lanes; group 128 (16 chunks): 2, 4, 8, 16
    NQ_GROUP(0, 64, 0, 2, 0, 1) NQ_GROUP(0, 64, 0, 2, 1, 2) NQ_GROUP(0, 64, 0, 2, 2, 4)
    NQ_GROUP(0, 64, 1, 4, 0, 1) NQ_GROUP(0, 64, 1, 4, 1, 2) NQ_GROUP(0, 64, 1, 4, 2, 4)
    NQ_GROUP(0, 64, 2, 8, 0, 1) NQ_GROUP(0, 64, 2, 8, 1, 2) NQ_GROUP(0, 64, 2, 8, 2, 4)
    NQ_GROUP(1, 128, 0, 2, 0, 1) NQ_GROUP(1, 128, 0, 2, 1, 2) NQ_GROUP(1, 128, 0, 2, 2, 4)
    NQ_GROUP(1, 128, 1, 4, 0, 1) NQ_GROUP(1, 128, 1, 4, 1, 2) NQ_GROUP(1, 128, 1, 4, 2, 4)
    NQ_GROUP(1, 128, 2, 8, 0, 1) NQ_GROUP(1, 128, 2, 8, 1, 2) NQ_GROUP(1, 128, 2, 8, 2, 4)
    NQ_GROUP(1, 128, 3, 16, 0, 1) NQ_GROUP(1, 128, 3, 16, 1, 2) NQ_GROUP(1, 128, 3, 16, 2, 4)
#undef NQ_GROUP
#undef NQ_GROUP_FL
  }
};
}  // namespace

const GroupTable& group_kernels() {
  static const GroupTableHolder h;
  return h.t;
}

}  // namespace nq
