// nq_group.cu — per-token-group e4m3 quantization of raw bf16 activations
// (vLLM PR #61343 "per_token_group_quant_8bit: multiply by reciprocal instead
// of dividing per element": Overview and Details).
//
// Per group of GROUP consecutive elements of a row: s = RN(absmax / 448)
// (UE8M0: the smallest power of two >= s), one correctly rounded reciprocal
// per group, q = e4m3(RN(x * RN(1 / s))) (NQ_FLAG_SCALE_DIV: RN(x / s)).
//
// Mapping: the activations are a flat list of G = M * K / GROUP groups.  A
// group is owned by GROUP / 8 consecutive lanes, one 16-byte chunk each, so a
// warp reads two (GROUP = 128) or four (GROUP = 64) neighbouring groups as one
// contiguous 512-byte span.  Each thread keeps U groups in flight; the group
// absmax is an xor-butterfly max inside the lane group (exact, order-free).
#include "nq_device.cuh"
#include "nq_internal.h"

namespace nq {

template <int GROUP, int U, bool VEC>
__global__ void __launch_bounds__(kGroupThreads) group_kernel(const GroupArgs a) {
  constexpr int TPG = GROUP / 8;                 // lanes per group
  constexpr int SLOT = kGroupThreads / TPG;      // groups per CTA per unit
  const int lane_g = int(threadIdx.x) % TPG;
  const int slot = int(threadIdx.x) / TPG;
  const int64_t base = int64_t(blockIdx.x) * SLOT * U;
  const bool div = (a.flags & kFlagDiv) != 0;
  const bool ue8m0 = (a.flags & kFlagUe8m0) != 0;

  griddep_wait();

  float v[U][8];
  int64_t row[U], cg[U];
  bool ok[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int64_t g = base + int64_t(u) * SLOT + slot;
    ok[u] = g < a.G;
    row[u] = ok[u] ? g / a.groups_per_row : 0;
    cg[u] = ok[u] ? g - row[u] * a.groups_per_row : 0;
    const uint16_t* src = a.x + row[u] * a.ld_x + cg[u] * GROUP + 8 * lane_g;
    if constexpr (VEC) {
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (ok[u]) w = __ldcs(reinterpret_cast<const uint4*>(src));
      unpack_bf16x8(w, v[u]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[u][j] = ok[u] ? bf16_to_f32(src[j]) : 0.0f;
    }
  }
  griddep_launch_dependents();

#pragma unroll
  for (int u = 0; u < U; ++u) {
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[u][j]));
#pragma unroll
    for (int o = TPG / 2; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    float s = __fdiv_rn(m, kE4M3Max);
    if (ue8m0) s = ue8m0_ceil(s);
    const float inv = (s == 0.0f) ? 0.0f : __frcp_rn(s);
    float t[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) t[j] = (div && s != 0.0f) ? __fdiv_rn(v[u][j], s) : __fmul_rn(v[u][j], inv);
    const uint32_t lo = pack_e4m3x4(t[0], t[1], t[2], t[3]);
    const uint32_t hi = pack_e4m3x4(t[4], t[5], t[6], t[7]);
    if (ok[u]) {
      uint8_t* dst = a.q + row[u] * a.ld_q + cg[u] * GROUP + 8 * lane_g;
      if constexpr (VEC) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[j] = uint8_t((j < 4 ? lo : hi) >> (8 * (j & 3)));
      }
      if (lane_g == 0) a.s[row[u] * a.ld_s + cg[u]] = s;
    }
  }
}

namespace {
struct GroupTableHolder {
  GroupTable t;
  GroupTableHolder() {
    t[0][0][0] = reinterpret_cast<const void*>(&group_kernel<64, 1, false>);
    t[0][0][1] = reinterpret_cast<const void*>(&group_kernel<64, 1, true>);
    t[0][1][0] = reinterpret_cast<const void*>(&group_kernel<64, 4, false>);
    t[0][1][1] = reinterpret_cast<const void*>(&group_kernel<64, 4, true>);
    t[1][0][0] = reinterpret_cast<const void*>(&group_kernel<128, 1, false>);
    t[1][0][1] = reinterpret_cast<const void*>(&group_kernel<128, 1, true>);
    t[1][1][0] = reinterpret_cast<const void*>(&group_kernel<128, 4, false>);
    t[1][1][1] = reinterpret_cast<const void*>(&group_kernel<128, 4, true>);
  }
};
}  // namespace

const GroupTable& group_kernels() {
  static const GroupTableHolder h;
  return h.t;
}

}  // namespace nq
