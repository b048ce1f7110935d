// nq_row_kernel.cuh — the fused residual-add + norm + quantize row kernel.
//
// One row (token) is owned by a group of T threads: a single warp (T = 32,
// eight rows per CTA), the whole CTA (T = 64..1024), or, for rows wider than
// 16384 elements, a thread-block cluster of NC CTAs (row_kernel_cluster).
// Thread t of the group owns the 16-byte chunks c = t + k*T, k = 0..K-1, of
// the row (8 bf16 values each; c = t + j*T + k*T*NC in CTA j of a cluster), so
// every load and store instruction of a warp touches one contiguous 512-byte
// span.  The row stays in float32 registers from load to quantized
// store: the row is read once, and each output is written once.
//
// Steps, per row (netraruntime blog "Fusing RMSNorm and FP8 Quantization
// Under torch.compile", TL;DR and FAQ; FlashInfer PR #3962 Description;
// TensorRT-LLM PR #14848 Description; FlashInfer PR #2459 Changes):
//   a1 load x (and residual) as bf16, widen to float32 (exact);
//   a2 r = RN(x + residual); residual_out = RN_bf16(r);
//   a3 row sums in the canonical chunked pairwise order (nq::row_sum);
//      rstd = RN(1 / RN(sqrt(RN(RN(sum / d) + eps))));
//   a4 y = RN(RN(r * rstd) * gamma)  (LayerNorm: fma(RN((r - mean) * rstd), gamma, beta));
//      optional bf16 norm_out;
//   a5 scale: dynamic s = RN(max|y| / 448), static RN(1 / scale[0]), or the
//      NVFP4 per-16 block scale e4m3(RN(RN(amax / 6) / g));
//   a6 quantize, pack (cvt.rn.satfinite e4m3x2 / e5m2x2 / e2m1x2) and store.
//   With e5m2 output the largest code is 57344 instead of 448.
//
// The kernel is bound by instruction issue as much as by HBM, so every
// per-element float operation is a packed two-lane one (add / mul / fma
// .f32x2: each lane rounds exactly like its scalar form), the chunk sums use
// an even and an odd accumulator so that they too run two lanes wide, and
// gamma / beta are fetched only after the row's reductions.
#pragma once

#include "nq_device.cuh"
#include "nq_internal.h"

namespace nq {

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// 8 bf16 (one 16-byte chunk) -> 4 float pairs, element 2i in .x of pair i.
__device__ __forceinline__ void unpack_pairs(const uint4& u, float2 (&v)[4]) {
  v[0] = make_float2(bf16_lo(u.x), bf16_hi(u.x));
  v[1] = make_float2(bf16_lo(u.y), bf16_hi(u.y));
  v[2] = make_float2(bf16_lo(u.z), bf16_hi(u.z));
  v[3] = make_float2(bf16_lo(u.w), bf16_hi(u.w));
}
__device__ __forceinline__ uint4 pack_pairs_bf16(const float2 (&v)[4]) {
  return make_uint4(pack_bf16x2(v[0].x, v[0].y), pack_bf16x2(v[1].x, v[1].y), pack_bf16x2(v[2].x, v[2].y),
                    pack_bf16x2(v[3].x, v[3].y));
}
template <bool E5>
__device__ __forceinline__ uint2 pack_pairs_fp8(const float2 (&t)[4]) {
  return make_uint2(pack_fp8x4<E5>(t[0].x, t[0].y, t[1].x, t[1].y), pack_fp8x4<E5>(t[2].x, t[2].y, t[3].x, t[3].y));
}

// Swizzled block-scale layout of block-scaled tensor-core GEMMs (NVIDIA PTX
// ISA / cuBLAS: 128-row x 4-column tiles of 512 bytes, row tiles outer; inside
// a tile row r, column c at 16 (r % 32) + 4 (r / 32) + c): byte offset of the
// 4-column word (row r, column tile jw) when a row has n_ct column tiles.
__device__ __forceinline__ int64_t sf_swizzled_word(int64_t r, int jw, int n_ct) {
  return ((r >> 7) * n_ct + jw) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4;
}
// The four block scales of chunks c .. c + 7 (held by lanes l .. l + 7, l % 8
// == 0; block b = chunks 2b, 2b + 1) as one little-endian word in lane l.
__device__ __forceinline__ uint32_t sf_word4(uint32_t sfc) {
  return sfc | (__shfl_down_sync(kFull, sfc, 2) << 8) | (__shfl_down_sync(kFull, sfc, 4) << 16) |
         (__shfl_down_sync(kFull, sfc, 6) << 24);
}
// Zero padding of the swizzled layout for rows M .. roundup(M, 128): real row
// `row` clears rows M + row, M + row + M, ... (every padding row once).
template <int T>
__device__ __forceinline__ void sf_zero_padding_rows(const RowArgs& a, int64_t row, int tid) {
  const int64_t m_pad = (a.M + 127) & ~int64_t(127);
  const int n_ct = (a.d / 16 + 3) / 4;
  for (int64_t p = a.M + row; p < m_pad; p += a.M)
    for (int j = tid; j < n_ct; j += T) *reinterpret_cast<uint32_t*>(a.sf + sf_swizzled_word(p, j, n_ct)) = 0u;
}

// NVFP4 block scale of a 16-element block with absmax amax under the global
// scale g: sf = e4m3(RN(RN(amax / 6) / g)), S = RN(dec(sf) * g) and the
// element multiplier RN(1 / S) (0 when S == 0).  Both divisions take the
// bounded division (nq_device.cuh); where a quotient is nonzero and outside
// [2^-24, 2^17], or g is outside the divisor range (ngr = -RN(1 / g), g_fast
// = g in range), the lane takes the library division instead, so the result
// is always the correctly rounded one.  That case is tested once per warp,
// so the library division is a branch that ordinary data never enter.  Every
// lane of the warp must call this together.
struct Nvfp4Scale {
  uint32_t code;
  float mult;
};
// The library-division form of the quotient, out of line: in the raw-row
// kernels (64 registers) ptxas then keeps the common path free of spills.
static __device__ __noinline__ float nvfp4_block_quotient_lib(float amax, float g) {
  return __fdiv_rn(__fdiv_rn(amax, 6.0f), g);
}
template <bool OUT_OF_LINE>
__device__ __forceinline__ Nvfp4Scale nvfp4_block_scale(float amax, float g, float ngr, bool g_fast) {
  constexpr float kSix = 6.0f, kNegRcpSix = -(1.0f / 6.0f);
  constexpr float kLo = 5.9604645e-08f, kHi = 131072.0f;  // 2^-24, 2^17
  float x = div_rn_by(amax, kSix, kNegRcpSix);
  float q = div_rn_by(x, g, ngr);
  // A zero quotient is exact (0 * r, then zero remainders) once ngr is finite.
  const bool fast = (amax == 0.0f || (amax >= kSix * kLo && amax <= kSix * kHi)) &&
                    (g_fast && (x == 0.0f || (x >= g * kLo && x <= g * kHi)));
  if (!__all_sync(kFull, fast)) {
    if (!fast) q = OUT_OF_LINE ? nvfp4_block_quotient_lib(amax, g) : __fdiv_rn(__fdiv_rn(amax, kSix), g);
  }
  const uint32_t code = f32_to_e4m3(q);
  const float S = __fmul_rn(e4m3_to_f32(code), g);
  return {code, (S == 0.0f) ? 0.0f : __frcp_rn(S)};
}
// Block scales of two chunk slots whose blocks each span this lane and its
// xor-1 partner: the even lane computes slot 0's, the odd lane slot 1's, and
// they swap, so each scale is computed once per pair instead of twice.
template <bool OUT_OF_LINE>
__device__ __forceinline__ void nvfp4_pair_scales(float amax0, float amax1, int tid, float g, float ngr, bool g_fast,
                                                  Nvfp4Scale& s0, Nvfp4Scale& s1) {
  const bool odd = (tid & 1) != 0;
  const Nvfp4Scale m = nvfp4_block_scale<OUT_OF_LINE>(odd ? amax1 : amax0, g, ngr, g_fast);
  const Nvfp4Scale o = {__shfl_xor_sync(kFull, m.code, 1), __shfl_xor_sync(kFull, m.mult, 1)};
  s0 = odd ? o : m;
  s1 = odd ? m : o;
}

// MoE dispatch: calls f(r) for each destination row r of `row` (dest[row *
// topk + j] >= 0); a destination at or past dest_rows is skipped and recorded
// in bit 1 of the device error word.
template <typename F>
__device__ __forceinline__ void for_each_dest(const RowArgs& a, int64_t row, F&& f) {
  const int32_t* dp = a.dest + row * a.topk;
  for (int j = 0; j < a.topk; ++j) {
    const int32_t r = __ldg(dp + j);
    if (r < 0) continue;
    if (r >= a.dest_rows) {
      atomicOr(a.err, 2u);
      continue;
    }
    f(int64_t(r));
  }
}

// Chunk partial of the canonical order: even / odd accumulators from +0,
// then RN(even + odd).
template <bool SQUARES>
__device__ __forceinline__ float chunk_partial(const float2 (&v)[4]) {
  float2 acc = f2(0.0f);
#pragma unroll
  for (int i = 0; i < 4; ++i) acc = SQUARES ? fma2(v[i], v[i], acc) : add2(acc, v[i]);
  return __fadd_rn(acc.x, acc.y);
}

// Row sum of the K chunk partials held by each thread of the group (highest
// chunk-index bit first: the thread's own chunks, then across the CTAs of a
// cluster (NC > 1, through xred), then across threads).
template <int T, int K, int NC = 1>
__device__ __forceinline__ float row_total(float (&part)[K], float* red, int tid, float* xred = nullptr) {
#pragma unroll
  for (int h = K / 2; h >= 1; h >>= 1)
#pragma unroll
    for (int i = 0; i < h; ++i) part[i] = __fadd_rn(part[i], part[i + h]);
  return row_sum<T>(cluster_tree_sum<T, NC>(part[0], xred, tid), red, tid);
}

// a1: raw bf16 chunks of one row (zeros past the row or for dead rows).
// FULL: every chunk slot of the schedule is a real chunk of a live row (d ==
// 8 * T * K * NC, one row per CTA or cluster), so no predicate or zero fill is
// needed.  With a cluster of NC CTAs, CTA `rank` owns chunks
// tid + rank * T + k * T * NC.
template <int T, int K, bool VEC, bool FULL, int NC = 1>
__device__ __forceinline__ void load_raw(const RowArgs& a, int64_t row, bool live, bool has_res, int tid,
                                         uint4 (&xr)[K], uint4 (&rr)[K], int rank = 0) {
  const int d = a.d;
  const int C = (d + 7) >> 3;
  const uint16_t* xrow = a.x + row * a.ld_x;
  const uint16_t* rrow = a.res_in + row * a.ld_res;
  const int cb = tid + (NC > 1 ? rank * T : 0);
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = cb + k * T * NC;
    const bool ok = FULL || (live && c < C);
    if constexpr (VEC) {
      xr[k] = ok ? __ldcs(reinterpret_cast<const uint4*>(xrow + 8 * c)) : make_uint4(0u, 0u, 0u, 0u);
      rr[k] = (has_res && ok) ? __ldcs(reinterpret_cast<const uint4*>(rrow + 8 * c)) : make_uint4(0u, 0u, 0u, 0u);
    } else {
      uint32_t w[4], z[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = 8 * c + 2 * j;
        w[j] = ((ok && e < d) ? uint32_t(xrow[e]) : 0u) | ((ok && e + 1 < d) ? uint32_t(xrow[e + 1]) << 16 : 0u);
        z[j] = 0u;
        if (has_res)
          z[j] = ((ok && e < d) ? uint32_t(rrow[e]) : 0u) | ((ok && e + 1 < d) ? uint32_t(rrow[e + 1]) << 16 : 0u);
      }
      xr[k] = make_uint4(w[0], w[1], w[2], w[3]);
      rr[k] = make_uint4(z[0], z[1], z[2], z[3]);
    }
  }
}

// The FP8 codes of a row's K chunk slots, stored to each of its destination
// rows (MoE dispatch).
template <int T, int K, bool VEC, bool FULL, int NC = 1>
__device__ __forceinline__ void scatter_codes(const RowArgs& a, int64_t row, bool live, int tid,
                                              const uint2 (&codes)[K], int rank = 0) {
  if (!live) return;
  const int d = a.d;
  const int C = FULL ? T * K * NC : (d + 7) >> 3;
  const int cb = tid + (NC > 1 ? rank * T : 0);
  for_each_dest(a, row, [&](int64_t r) {
    uint8_t* qrow = a.q + r * a.ld_q;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int c = cb + k * T * NC;
      if (FULL || c < C) {
        if constexpr (VEC) {
          *reinterpret_cast<uint2*>(qrow + 8 * c) = codes[k];
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (8 * c + j < d) qrow[8 * c + j] = uint8_t((j < 4 ? codes[k].x : codes[k].y) >> (8 * (j & 3)));
        }
      }
    }
  });
}

// Per-token-group FP8 of a row's y (chunk c of the row in v[k] for c = tid +
// k*T): a group of G elements is G/8 consecutive chunks, held by G/8
// consecutive threads of the group (T >= 32 and a multiple of G/8), so its
// absmax is an xor-butterfly over those lanes; then s = RN(absmax / max)
// (max 448, or 57344 for e5m2; UE8M0: next power of two), one reciprocal,
// q = fp8(RN(y * RN(1 / s))).  K <= 8, so a warp's K slots hold at most 32
// groups (one per lane).
template <bool E5, bool LAYOUT, int T, int K, bool VEC, bool FULL, bool SCATTER = false, int NC = 1>
__device__ __forceinline__ void quantize_groups(const RowArgs& a, int64_t row, bool live, int tid,
                                                const float2 (&v)[K][4], bool div, int rank = 0) {
  const int d = a.d;
  const int C = FULL ? T * K * NC : (d + 7) >> 3;
  const int cb = tid + (NC > 1 ? rank * T : 0);  // this thread's chunk in slot 0
  const int lcpg = (a.group == 128) ? 4 : 3;  // log2(chunks per group): groups are 64 or 128
  const int cpg = 1 << lcpg;                   // chunks per group: 8 or 16
  const int gpw = 32 >> lcpg;                  // groups per warp per chunk slot
  const int lane = tid & 31;
  const bool ue8m0 = (a.flags & kFlagUe8m0) != 0;
  uint8_t* qrow = a.q + row * a.ld_q;
  float* srow = a.scale_out + row * a.ld_scale;
  // 1. group absmax of every chunk slot (xor-butterfly over the group's lanes)
  float am[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    float m = absmax8(v[k], 0.0f);
    for (int o = cpg >> 1; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    am[k] = m;
  }
  // 2. the warp holds K * gpw <= 32 groups: lane j computes the scale of group
  //    (slot j / gpw, part j % gpw) once, instead of every lane computing the
  //    scale of each of its K groups (a correctly rounded division and
  //    reciprocal per group would otherwise dominate the instruction count).
  float mine = 0.0f;
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const float t = __shfl_sync(kFull, am[k], (lane & (gpw - 1)) << lcpg);
    if ((lane >> (5 - lcpg)) == k) mine = t;
  }
  float s = fp8_scale_of<E5>(mine);
  if (ue8m0) s = ue8m0_ceil(s);
  const float inv = (s == 0.0f) ? 0.0f : __frcp_rn(s);
  {
    const int kj = lane >> (5 - lcpg), part = lane & (gpw - 1);
    const int c0 = (cb & ~31) + (part << lcpg) + kj * T * NC;  // first chunk of lane j's group
    if (kj < K && (FULL || (live && c0 < C))) {
      if constexpr (SCATTER)
        for_each_dest(a, row, [&](int64_t r) { a.scale_out[r * a.ld_scale + (c0 >> lcpg)] = s; });
      else if constexpr (LAYOUT)
        store_group_scale(a.scale_out, a.ld_scale, a.cs_scale, (a.flags & kFlagScalesPacked) != 0, row,
                          c0 >> lcpg, d >> (lcpg + 3), s);
      else
        srow[c0 >> lcpg] = s;
    }
  }
  // 3. each lane takes back the reciprocal (and scale) of its own groups
  uint2 kept[SCATTER ? K : 1];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = cb + k * T * NC;
    const int src = k * gpw + (lane >> lcpg);
    const float ik = __shfl_sync(kFull, inv, src);
    const float sk = div ? __shfl_sync(kFull, s, src) : 0.0f;
    float2 t[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      t[i] = (div && sk != 0.0f) ? make_float2(__fdiv_rn(v[k][i].x, sk), __fdiv_rn(v[k][i].y, sk))
                                 : mul2(v[k][i], f2(ik));
    const uint2 codes = pack_pairs_fp8<E5>(t);
    if constexpr (SCATTER) {
      kept[k] = codes;
    } else if (FULL || (live && c < C)) {
      if constexpr (VEC) {
        *reinterpret_cast<uint2*>(qrow + 8 * c) = codes;
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) qrow[8 * c + j] = uint8_t((j < 4 ? codes.x : codes.y) >> (8 * (j & 3)));
      }
    }
  }
  if constexpr (SCATTER) scatter_codes<T, K, VEC, FULL, NC>(a, row, live, tid, kept, rank);
}

// a2..a6 of one row whose raw chunks are in registers.  Contains the row
// group's barriers (T > 32).  s_sum0 / s_sum1 / s_max are the group's
// reduction buffers.  A row split over a cluster of NC CTAs (this one of rank
// `rank`) also takes the cluster's barriers and its distributed buffers
// x_sum0 / x_sum1 (NC x T floats each) and x_max (one word).
template <int OP, int T, int K, bool VEC, bool FULL, int OUT, bool NARROW = false, int NC = 1>
__device__ __forceinline__ void process_row(const RowArgs& a, int64_t row, bool live_in, bool has_res, int tid,
                                            const uint4 (&xr)[K], const uint4 (&rr)[K], float* s_sum0,
                                            float* s_sum1, uint32_t* s_max, int rank = 0, float* x_sum0 = nullptr,
                                            float* x_sum1 = nullptr, uint32_t* x_max = nullptr) {
  constexpr bool E5 = (OUT & kOutAlt) && OP != kOpRmsNvfp4;   // e5m2 codes
  constexpr bool SWZ = (OUT & kOutAlt) && OP == kOpRmsNvfp4;  // swizzled block scales
  constexpr bool LAYOUT = (OUT & kOutScaleLayout) != 0;       // strided / packed group scales
  constexpr bool SCATTER = (OUT & kOutScatter) != 0;          // MoE destination rows
  const int d = a.d;
  const int C = FULL ? T * K * NC : (d + 7) >> 3;
  constexpr int CS = T * NC;                      // chunk stride between a thread's slots
  const int cb = tid + (NC > 1 ? rank * T : 0);  // this thread's chunk in slot 0
  const bool live = FULL || live_in;
  const bool div_flag = (a.flags & kFlagDiv) != 0;
  const bool bf16_flag = (a.flags & kFlagNormBf16) != 0;
  // NARROW (16-byte rows narrower than the schedule): a chunk slot that lies
  // wholly past the row for this warp is skipped in every per-chunk step
  // except the NVFP4 and group quantization (which run on its zeros); its
  // sums are +0, as zero chunks give.  Only the upper half of the slots can
  // be dead for a planned schedule (see process_raw_row).
  const int wbase = cb & ~31;
  auto slot_live = [&](int k) { return !NARROW || k < K / 2 || wbase + k * CS < C; };
  // ---- a2: r = x + residual, residual_out; a3: chunk partials
  float2 v[K][4];
  float part[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = cb + k * CS;
    if (!slot_live(k)) {
#pragma unroll
      for (int i = 0; i < 4; ++i) v[k][i] = f2(0.0f);
      part[k] = 0.0f;
      continue;
    }
    unpack_pairs(xr[k], v[k]);
    if (has_res) {
      float2 t[4];
      unpack_pairs(rr[k], t);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[k][i] = add2(v[k][i], t[i]);
      if (FULL || (live && c < C)) {
        uint16_t* orow = a.res_out + row * a.ld_res;
        if constexpr (VEC) {
          *reinterpret_cast<uint4*>(orow + 8 * c) = pack_pairs_bf16(v[k]);
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (8 * c + 2 * i < d) orow[8 * c + 2 * i] = f32_to_bf16(v[k][i].x);
            if (8 * c + 2 * i + 1 < d) orow[8 * c + 2 * i + 1] = f32_to_bf16(v[k][i].y);
          }
        }
      }
    }
    part[k] = chunk_partial<OP != kOpLnStaticFp8>(v[k]);
  }
  const float total = row_total<T, K, NC>(part, s_sum0, tid, x_sum0);

  const float fd = float(d);
  float rstd;
  if constexpr (OP == kOpLnStaticFp8) {
    // Centre on the row mean (RN(r - mean) == RN(r + (-mean))), then the
    // biased variance; padding elements of a partial chunk are zeroed.
    const float2 nm = f2(-__fdiv_rn(total, fd));
#pragma unroll
    for (int k = 0; k < K; ++k) {
      if (!slot_live(k)) continue;  // part[k] is +0 already
      const int c = cb + k * CS;
      const bool ok = FULL || (live && c < C);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 t = add2(v[k][i], nm);
        if constexpr (!VEC) {
          if (8 * c + 2 * i >= d) t.x = 0.0f;
          if (8 * c + 2 * i + 1 >= d) t.y = 0.0f;
        }
        v[k][i] = t;
      }
      // a chunk slot past the row adds +0 (its values are never stored)
      part[k] = ok ? chunk_partial<true>(v[k]) : 0.0f;
    }
    const float sq = row_total<T, K, NC>(part, s_sum1, tid, x_sum1);
    rstd = __frcp_rn(__fsqrt_rn(__fadd_rn(__fdiv_rn(sq, fd), a.eps)));
  } else {
    rstd = __frcp_rn(__fsqrt_rn(__fadd_rn(__fdiv_rn(total, fd), a.eps)));
  }

  // ---- a4..a6.  The plain form (the call's default quantization, no bf16
  // rounding, no norm output) is a separate copy with those flags folded
  // away, so its per-chunk code carries no branch on them (K >= 4, below).
  auto finish = [&](auto plain_tag) {
  constexpr bool PLAIN = decltype(plain_tag)::value;
  const bool div = PLAIN ? (OP == kOpRmsDynFp8) : div_flag;
  const bool bf16_round = PLAIN ? false : bf16_flag;
  uint16_t* const norm_out = PLAIN ? nullptr : a.norm_out;
  // ---- a4: normalize (y overwrites v); gamma / beta fetched now, through L1
  const float2 rs2 = f2(rstd);
#pragma unroll
  for (int k = 0; k < K; ++k) {
    if (!slot_live(k)) continue;  // y stays 0
    const int c = cb + k * CS;
    const bool gok = FULL || c < C;
    if constexpr (OP == kOpLnStaticFp8) {
      const float* gp = static_cast<const float*>(a.gamma) + 8 * c;
      const float* bp = a.beta + 8 * c;
      float2 g[4], b[4];
      if constexpr (VEC) {
        float4 g0 = make_float4(0.f, 0.f, 0.f, 0.f), g1 = g0, b0 = g0, b1 = g0;
        if (gok) {
          g0 = __ldg(reinterpret_cast<const float4*>(gp));
          g1 = __ldg(reinterpret_cast<const float4*>(gp + 4));
          b0 = __ldg(reinterpret_cast<const float4*>(bp));
          b1 = __ldg(reinterpret_cast<const float4*>(bp + 4));
        }
        g[0] = make_float2(g0.x, g0.y); g[1] = make_float2(g0.z, g0.w);
        g[2] = make_float2(g1.x, g1.y); g[3] = make_float2(g1.z, g1.w);
        b[0] = make_float2(b0.x, b0.y); b[1] = make_float2(b0.z, b0.w);
        b[2] = make_float2(b1.x, b1.y); b[3] = make_float2(b1.z, b1.w);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int e = 8 * c + 2 * i;
          g[i] = make_float2((gok && e < d) ? __ldg(gp + 2 * i) : 0.f, (gok && e + 1 < d) ? __ldg(gp + 2 * i + 1) : 0.f);
          b[i] = make_float2((gok && e < d) ? __ldg(bp + 2 * i) : 0.f, (gok && e + 1 < d) ? __ldg(bp + 2 * i + 1) : 0.f);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) v[k][i] = fma2(mul2(v[k][i], rs2), g[i], b[i]);
    } else {
      const uint16_t* gp = static_cast<const uint16_t*>(a.gamma) + 8 * c;
      uint4 gu = make_uint4(0u, 0u, 0u, 0u);
      if constexpr (VEC) {
        if (gok) gu = __ldg(reinterpret_cast<const uint4*>(gp));
      } else {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int e = 8 * c + 2 * j;
          w[j] = ((gok && e < d) ? uint32_t(__ldg(gp + 2 * j)) : 0u) |
                 ((gok && e + 1 < d) ? uint32_t(__ldg(gp + 2 * j + 1)) << 16 : 0u);
        }
        gu = make_uint4(w[0], w[1], w[2], w[3]);
      }
      float2 g[4];
      unpack_pairs(gu, g);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[k][i] = mul2(mul2(v[k][i], rs2), g[i]);
    }
    if (bf16_round) {
#pragma unroll
      for (int i = 0; i < 4; ++i) v[k][i] = make_float2(round_bf16(v[k][i].x), round_bf16(v[k][i].y));
    }
  }
  if constexpr (OP != kOpLnStaticFp8) {
    if (norm_out != nullptr) {
      uint16_t* nrow = norm_out + row * a.ld_norm;
#pragma unroll
      for (int k = 0; k < K; ++k) {
        const int c = cb + k * CS;
        if (FULL || (live && c < C)) {
          if constexpr (VEC) {
            *reinterpret_cast<uint4*>(nrow + 8 * c) = pack_pairs_bf16(v[k]);
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if (8 * c + 2 * i < d) nrow[8 * c + 2 * i] = f32_to_bf16(v[k][i].x);
              if (8 * c + 2 * i + 1 < d) nrow[8 * c + 2 * i + 1] = f32_to_bf16(v[k][i].y);
            }
          }
        }
      }
    }
  }

  // ---- a5 + a6: scale, quantize, pack, store
  if constexpr (OP == kOpRmsNvfp4) {
    const float g = __ldg(a.scale);
    const float ngr = -__frcp_rn(g);
    const bool g_fast = fast_div_ok(g);
    uint8_t* qrow = a.q + row * a.ld_q;
    uint8_t* sfrow = a.sf + row * a.ld_sf;
    // A 16-element block is chunks (c, c^1), held by lanes (t, t^1).
    auto block_amax = [&](int k) {
      const float m8 = absmax8(v[k], 0.0f);
      return fmaxf(m8, __shfl_xor_sync(kFull, m8, 1));
    };
    auto quant_store = [&](int k, const Nvfp4Scale& sc, bool sf_here) {
      const int c = cb + k * CS;
      const bool ok = FULL || (live && c < C);
      float t[8];
      const float S = div ? __fmul_rn(e4m3_to_f32(sc.code), g) : 0.0f;
      if (div && S != 0.0f) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          t[2 * i] = __fdiv_rn(v[k][i].x, S);
          t[2 * i + 1] = __fdiv_rn(v[k][i].y, S);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 q = mul2(v[k][i], f2(sc.mult));
          t[2 * i] = q.x;
          t[2 * i + 1] = q.y;
        }
      }
      const uint32_t packed = pack_e2m1x8(t);
      if constexpr (SWZ) {
        const uint32_t word = sf_word4(sc.code);  // padding columns come from zero chunks
        if (ok && (c & 7) == 0)
          *reinterpret_cast<uint32_t*>(a.sf + sf_swizzled_word(row, c >> 3, (C + 7) >> 3)) = word;
      }
      if (ok) {
        if constexpr (VEC) {
          *reinterpret_cast<uint32_t*>(qrow + 4 * c) = packed;
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) qrow[4 * c + j] = uint8_t(packed >> (8 * j));
        }
        if (!SWZ && sf_here && (c & 1) == 0) sfrow[c >> 1] = uint8_t(sc.code);
      }
    };
    if constexpr (K >= 2) {
#pragma unroll
      for (int k = 0; k < K; k += 2) {
        Nvfp4Scale s0, s1;
        nvfp4_pair_scales<false>(block_amax(k), block_amax(k + 1), tid, g, ngr, g_fast, s0, s1);
        quant_store(k, s0, true);
        quant_store(k + 1, s1, true);
      }
    } else {
      quant_store(0, nvfp4_block_scale<false>(block_amax(0), g, ngr, g_fast), true);
    }
    if constexpr (SWZ) {
      if (live && cb < T) sf_zero_padding_rows<T>(a, row, tid);  // rank 0 of a cluster
    }
  } else if constexpr (OP == kOpRmsGroupFp8) {
    quantize_groups<E5, LAYOUT, T, K, VEC, FULL, SCATTER, NC>(a, row, live, tid, v, div, rank);
  } else {
    float s_div, s_inv;
    bool passthrough = false;
    if constexpr (OP == kOpRmsDynFp8) {
      float m = 0.0f;
#pragma unroll
      for (int k = 0; k < K; ++k)
        if (slot_live(k)) m = absmax8(v[k], m);
      const float amax = __uint_as_float(
          cluster_max_u32<NC>(__float_as_uint(row_max_nonneg<T>(m, s_max, tid)), x_max, tid));
      const float s = fp8_scale_of<E5>(amax);
      if constexpr (SCATTER) {
        if (live && cb == 0) for_each_dest(a, row, [&](int64_t r) { a.scale_out[r] = s; });
      } else {
        if (live && cb == 0) a.scale_out[row] = s;
      }
      s_div = s;
      s_inv = __frcp_rn(s);
      passthrough = (s == 0.0f);  // zero row: store the signed zeros of y
    } else {
      s_div = __ldg(a.scale);
      s_inv = __frcp_rn(s_div);
    }
    uint8_t* qrow = a.q + row * a.ld_q;
    uint2 kept[SCATTER ? K : 1];
    auto store_codes = [&](int k, const float2 (&t)[4]) {
      const int c = cb + k * CS;
      const uint2 codes = pack_pairs_fp8<E5>(t);
      if constexpr (SCATTER) {
        kept[k] = codes;
        return;
      }
      if (FULL || (live && c < C)) {
        if constexpr (VEC) {
          *reinterpret_cast<uint2*>(qrow + 8 * c) = codes;
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (8 * c + j < d) qrow[8 * c + j] = uint8_t((j < 4 ? codes.x : codes.y) >> (8 * (j & 3)));
        }
      }
    };
    // Dynamic scale with division: |y / s| <= 448 (57344), so the bounded
    // division from RN(1 / s) is exact (nq_device.cuh); tiny scales keep the
    // library division.  Each form is its own loop.
    const bool fast = (OP == kOpRmsDynFp8) && div && fast_div_ok(s_div);
    if (passthrough) {
#pragma unroll
      for (int k = 0; k < K; ++k)
        if (slot_live(k)) store_codes(k, v[k]);
    } else if (fast) {
      const float2 s2 = f2(s_div), nr2 = f2(-s_inv);
#pragma unroll
      for (int k = 0; k < K; ++k) {
        if (!slot_live(k)) continue;
        float2 t[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) t[i] = div2_rn_by(v[k][i], s2, nr2);
        store_codes(k, t);
      }
    } else if (div) {
#pragma unroll
      for (int k = 0; k < K; ++k) {
        if (!slot_live(k)) continue;
        float2 t[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) t[i] = make_float2(__fdiv_rn(v[k][i].x, s_div), __fdiv_rn(v[k][i].y, s_div));
        store_codes(k, t);
      }
    } else {
      const float2 inv2 = f2(s_inv);
#pragma unroll
      for (int k = 0; k < K; ++k) {
        if (!slot_live(k)) continue;
        float2 t[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) t[i] = mul2(v[k][i], inv2);
        store_codes(k, t);
      }
    }
    if constexpr (SCATTER) scatter_codes<T, K, VEC, FULL, NC>(a, row, live, tid, kept, rank);
  }
  };
  // Measured on B200: the second copy pays with four chunks per thread
  // (4-7 %), but costs an SM slot with two or fewer (38 -> 43 registers).
  if (K >= 4 && !bf16_flag && a.norm_out == nullptr && div_flag == (OP == kOpRmsDynFp8)) finish(BoolTag<true>{});
  else finish(BoolTag<false>{});
}

// The body of a register-row kernel, shared by row_kernel and row_kernel_512,
// which differ only in their launch bounds.  Rows past M (only possible with
// eight rows per CTA) run every step with zeros so that warp-wide shuffles
// stay converged, and store nothing.  griddep_launch_dependents lets the next
// kernel on the stream start its prologue once the row's loads are issued.
#define NQ_ROW_KERNEL_BODY(T)                                                                                    \
  constexpr bool VEC = MODE >= 1;                                                                                \
  constexpr bool FULL = MODE == 2;                                                                               \
  constexpr bool NARROW = MODE == 3;                                                                             \
  constexpr int R = (T == 32) ? 8 : 1; /* rows per CTA */                                                        \
  constexpr int W = T / 32;            /* warps per row */                                                       \
  static_assert(K == 1 || K == 2 || K == 4 || K == 8, "chunks per thread");                                      \
  static_assert(R * T <= 1024, "CTA size");                                                                      \
  __shared__ __align__(16) float s_sum[2][W > 1 ? W * 32 : 1];                                                   \
  __shared__ uint32_t s_max[W > 1 ? W : 1];                                                                      \
  const int tid = (T == 32) ? int(threadIdx.x & 31u) : int(threadIdx.x);                                         \
  const int64_t row = (T == 32) ? int64_t(blockIdx.x) * R + int64_t(threadIdx.x >> 5) : int64_t(blockIdx.x);     \
  const bool live = row < a.M;                                                                                   \
  const bool has_res = (OP != kOpLnStaticFp8) && (a.res_in != nullptr);                                          \
  griddep_wait();                                                                                                \
  uint4 xr[K], rr[K];                                                                                            \
  load_raw<T, K, VEC, FULL>(a, row, live, has_res, tid, xr, rr);                                                 \
  griddep_launch_dependents();                                                                                   \
  process_row<OP, T, K, VEC, FULL, OUT, NARROW>(a, row, live, has_res, tid, xr, rr, s_sum[0], s_sum[1], s_max);

// One row per thread group: loads straight to registers.  Many small CTAs per
// SM keep enough rows in flight; a persistent variant that prefetched the
// next row into a second register set measured slower on B200 (the doubled
// registers halve occupancy), and so did shared-memory cp.async staging.
// MODE 0: any alignment (scalar loads); 1: 16-byte rows; 2: 16-byte rows that
// exactly fill the schedule (d == 8 * T * K, T > 32): no predicates at all;
// 3: 16-byte rows narrower than the schedule (d < 8 * T * K): chunk slots
// wholly past the row are skipped per warp.
// OUT: output-form bits, each a separate instantiation so that the default
// kernels carry no branch on them.  kOutAlt: e5m2 codes for the FP8
// operations, the swizzled block-scale layout for NVFP4; kOutScaleLayout
// (group operation): strided or packed-UE8M0 group scales.
template <int OP, int T, int K, int MODE, int OUT>
__global__ void __launch_bounds__(T == 32 ? 256 : T) row_kernel(const RowArgs a) {
NQ_ROW_KERNEL_BODY(T)
}

// 512 threads with four chunks each (rows of 8193 ... 16384 elements) under a
// launch bound of two CTAs per SM (64 registers) instead of one: measured on
// B200, 16384 x 16384 dynamic 392 -> 303 us, NVFP4 with residual 397 -> 273
// us, fused group with residual 421 -> 299 us, 4096 x 16384 dynamic 104 -> 80
// us (the predicate-free copy spills a few hundred bytes and is still faster).
// The other schedules keep no bound: at 256 threads a 64-register bound moved
// d = 2816 ... 8192 by +-2 %.
template <int OP, int K, int MODE, int OUT>
__global__ void __launch_bounds__(512, 2) row_kernel_512(const RowArgs a) {
NQ_ROW_KERNEL_BODY(512)
}

// Rows wider than one CTA can hold in registers (d > 16384 elements): one row
// per thread-block cluster of NC CTAs of kClusterThreads threads, each holding
// K chunks per thread in registers, so the row is still read once and every
// output written once.  (Measured on B200 at 65536 x d: 256 threads with four
// chunks each, in clusters of 4 or 8, runs 1.5x faster than 1024 threads with
// two chunks in clusters of 2 or 4; 512 x 4 and 128 x 8 land in between.)  The row sums cross the cluster through
// distributed shared memory in the canonical order (cluster_tree_sum); the
// absmax of the dynamic scale likewise (cluster_max_u32).  MODE as for
// row_kernel.
// The launch bound holds a CTA to 64 registers, four CTAs (four rows' quarters
// or eighths) per SM: ptxas then spills a few hundred bytes per thread, but
// the extra rows in flight hide the cluster barriers.  Measured on B200 against
// no bound (80-128 registers, two or three CTAs per SM): dynamic 2048 x 65536
// 289 -> 231 us, 4096 x 32768 254 -> 209 us; static RMSNorm with residual
// 4096 x 32768 179 -> 164 us; NVFP4 without residual 2048 x 65536 187 -> 138
// us; LayerNorm 8192 x 20480 358 -> 316 us; rows of 20480 elements otherwise
// within 3 %.  A bound of three CTAs was no faster.
template <int OP, int K, int MODE, int OUT, int NC>
__global__ void __cluster_dims__(NC, 1, 1) __launch_bounds__(kClusterThreads, 4) row_kernel_cluster(const RowArgs a) {
  constexpr int T = kClusterThreads;
  constexpr bool VEC = MODE >= 1;
  constexpr bool FULL = MODE == 2;
  constexpr bool NARROW = MODE == 3;
  constexpr int W = T / 32;
  static_assert(NC == 2 || NC == 4 || NC == 8, "CTAs per row (8: the portable cluster size limit)");
  __shared__ __align__(16) float s_sum[2][W * 32];
  __shared__ uint32_t s_max[W];
  __shared__ __align__(16) float x_sum[2][NC * T];  // written by every CTA of the cluster
  __shared__ uint32_t x_max[1];                     // read by every CTA of the cluster

  const int tid = int(threadIdx.x);
  const int rank = cluster_rank<NC>();
  const int64_t row = int64_t(blockIdx.x) / NC;  // one row per cluster (clusters are consecutive blocks)
  const bool has_res = (OP != kOpLnStaticFp8) && (a.res_in != nullptr);

  // Every CTA of the cluster has started (its shared memory exists) before
  // any CTA writes to it: the arrive costs nothing here, and the wait, after
  // the row's loads are issued, finds every CTA arrived.
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  griddep_wait();
  uint4 xr[K], rr[K];
  load_raw<T, K, VEC, FULL, NC>(a, row, true, has_res, tid, xr, rr, rank);
  griddep_launch_dependents();
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  process_row<OP, T, K, VEC, FULL, OUT, NARROW, NC>(a, row, true, has_res, tid, xr, rr, s_sum[0], s_sum[1], s_max,
                                                    rank, x_sum[0], x_sum[1], x_max);
  // The absmax (dynamic path only) is read from the other CTAs' buffers: no
  // CTA leaves while another may still read them.
  if constexpr (OP == kOpRmsDynFp8) cooperative_groups::this_cluster().sync();
}

// Per-chunk gamma (RMSNorm: bf16) or gamma and beta (LayerNorm: float32) of
// chunk slot k = tid + k * T, zero past the row, fetched from global memory
// (through L1) at each use.
template <int T>
struct GammaLoads {
  const RowArgs& a;
  int tid, C;
  __device__ __forceinline__ void ln(int k, float4& g0, float4& g1, float4& e0, float4& e1) const {
    const int c = tid + k * T;
    g0 = make_float4(0.f, 0.f, 0.f, 0.f), g1 = g0, e0 = g0, e1 = g0;
    if (c < C) {
      const float* gp = static_cast<const float*>(a.gamma) + 8 * c;
      g0 = __ldg(reinterpret_cast<const float4*>(gp));
      g1 = __ldg(reinterpret_cast<const float4*>(gp + 4));
      e0 = __ldg(reinterpret_cast<const float4*>(a.beta + 8 * c));
      e1 = __ldg(reinterpret_cast<const float4*>(a.beta + 8 * c + 4));
    }
  }
  __device__ __forceinline__ uint4 rms(int k) const {
    const int c = tid + k * T;
    uint4 gu = make_uint4(0u, 0u, 0u, 0u);
    if (c < C) gu = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.gamma) + 8 * c));
    return gu;
  }
  __device__ __forceinline__ void rms2(int k, float2 (&g)[4]) const { unpack_pairs(rms(k), g); }
};

// RMSNorm gamma (bf16) widened to fp32 once per persistent CTA and kept in
// shared memory: per chunk two conflict-free 16-byte loads replace a load and
// eight integer unpack instructions on every row.  Chunk c's first four
// values are lo[c], the last four hi[c]; LayerNorm's fp32 beta follows as
// lo[2 C + c] and lo[3 C + c].
template <int T, int K>
struct GammaSmem {
  const float4* lo;
  const float4* hi;
  int tid, C;
  __device__ __forceinline__ void ln(int k, float4& g0, float4& g1, float4& e0, float4& e1) const {
    const int c = tid + k * T;
    g0 = make_float4(0.f, 0.f, 0.f, 0.f), g1 = g0, e0 = g0, e1 = g0;
    if (c < C) g0 = lo[c], g1 = hi[c], e0 = lo[2 * C + c], e1 = lo[3 * C + c];
  }
  __device__ __forceinline__ void rms2(int k, float2 (&g)[4]) const {
    const int c = tid + k * T;
    float4 l = make_float4(0.f, 0.f, 0.f, 0.f), h = l;
    if (c < C) l = lo[c], h = hi[c];
    g[0] = make_float2(l.x, l.y), g[1] = make_float2(l.z, l.w), g[2] = make_float2(h.x, h.y),
    g[3] = make_float2(h.z, h.w);
  }
};

// a3..a6 of one row without residual whose raw bf16 chunks come from src(k)
// (registers) and whose gamma / beta come from gam.  Rows past M (warp rows only) compute on zeros and store nothing.
template <int OP, int T, int K, int OUT, bool NARROW, typename Src, typename Gam>
__device__ __forceinline__ void process_raw_row(const RowArgs& a, int64_t row, int tid, Src&& src, const Gam& gam,
                                                float* b0, float* b1, float scale_in, float inv_static) {
  constexpr bool E5 = (OUT & kOutAlt) && OP != kOpRmsNvfp4;   // e5m2 codes
  constexpr bool SWZ = (OUT & kOutAlt) && OP == kOpRmsNvfp4;  // swizzled block scales
  constexpr bool LAYOUT = (OUT & kOutScaleLayout) != 0;       // strided / packed group scales
  const int d = a.d;
  const int C = d >> 3;
  const float fd = float(d);
  const bool div_flag = (a.flags & kFlagDiv) != 0;
  const bool bf16_flag = (a.flags & kFlagNormBf16) != 0;
  const bool live = row < a.M;  // rows past M (warp rows only) compute on zeros and store nothing
  // NARROW: the row may be narrower than the schedule (C < T * K, d not a
  // power of two), so chunk slot k of this thread's warp may lie wholly past
  // it; such a slot is skipped (its partial sums are +0, as zero chunks would
  // give).  The test is warp-uniform.  The lower half of the slots is never
  // dead for a schedule the planner picks (T * K is the smallest power of two
  // >= C), so only the upper half is tested; a dead lower slot of a forced,
  // wider schedule is computed on zeros.  Rows that fill the schedule take
  // the NARROW = false copy, free of these tests (they cost 2-4 % there).
  const int wbase = tid & ~31;
  auto slot_live = [&](int k) { return !NARROW || k < K / 2 || wbase + k * T < C; };
  float part[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    part[k] = 0.0f;
    if (slot_live(k)) {
      float2 v[4];
      unpack_pairs(src(k), v);
      part[k] = chunk_partial<OP != kOpLnStaticFp8>(v);
    }
  }
  const float total = row_total<T, K>(part, b0, tid);
  float rstd, mean = 0.0f;
  if constexpr (OP == kOpLnStaticFp8) {
    mean = __fdiv_rn(total, fd);
    const float2 nm = f2(-mean);
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int c = tid + k * T;
      part[k] = 0.0f;
      if (slot_live(k)) {
        float2 v[4];
        unpack_pairs(src(k), v);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = add2(v[i], nm);
        // a chunk past the row adds +0 (as a zero chunk would): one select
        // per chunk instead of one per element
        part[k] = (c < C) ? chunk_partial<true>(v) : 0.0f;
      }
    }
    const float sq = row_total<T, K>(part, b1, tid);
    rstd = __frcp_rn(__fsqrt_rn(__fadd_rn(__fdiv_rn(sq, fd), a.eps)));
  } else {
    rstd = __frcp_rn(__fsqrt_rn(__fadd_rn(__fdiv_rn(total, fd), a.eps)));
  }
  const float2 rs2 = f2(rstd), nm = f2(-mean), inv2 = f2(inv_static);
  uint8_t* qrow = a.q + row * a.ld_q;
  // Pass 3.  The plain form (reciprocal quantization, no bf16 rounding, no
  // norm output: the default of every call) is a separate copy of the loop
  // with those flags folded away, so the per-chunk code carries no branch on
  // them and no library-division call site.
  auto pass3 = [&](auto plain_tag) {
  constexpr bool PLAIN = decltype(plain_tag)::value;
  const bool div = PLAIN ? false : div_flag;
  const bool bf16_round = PLAIN ? false : bf16_flag;
  uint16_t* const norm_out = PLAIN ? nullptr : a.norm_out;
  // y of chunk slot k (and its bf16 norm output)
  auto norm_chunk = [&](int k, float2 (&v)[4]) {
    const int c = tid + k * T;
    const bool ok = live && c < C;
    unpack_pairs(src(k), v);
    if constexpr (OP == kOpLnStaticFp8) {
      float4 g0, g1, e0, e1;
      gam.ln(k, g0, g1, e0, e1);
      const float2 g[4] = {make_float2(g0.x, g0.y), make_float2(g0.z, g0.w), make_float2(g1.x, g1.y),
                           make_float2(g1.z, g1.w)};
      const float2 b[4] = {make_float2(e0.x, e0.y), make_float2(e0.z, e0.w), make_float2(e1.x, e1.y),
                           make_float2(e1.z, e1.w)};
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = fma2(mul2(add2(v[i], nm), rs2), g[i], b[i]);
    } else {
      float2 g[4];
      gam.rms2(k, g);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = mul2(mul2(v[i], rs2), g[i]);
    }
    if (bf16_round) {
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = make_float2(round_bf16(v[i].x), round_bf16(v[i].y));
    }
    if constexpr (OP != kOpLnStaticFp8) {
      if (norm_out != nullptr && ok)
        *reinterpret_cast<uint4*>(norm_out + row * a.ld_norm + 8 * c) = pack_pairs_bf16(v);
    }
  };
  if constexpr (OP == kOpRmsNvfp4) {
    const float ngr = -__frcp_rn(scale_in);
    const bool g_fast = fast_div_ok(scale_in);
    uint8_t* const sfrow = a.sf + row * a.ld_sf;
    auto block_amax = [&](const float2 (&v)[4]) {  // chunks c, c^1 (lanes t, t^1) form a block
      const float m8 = absmax8(v, 0.0f);
      return fmaxf(m8, __shfl_xor_sync(kFull, m8, 1));
    };
    auto quant_store = [&](int k, const float2 (&v)[4], const Nvfp4Scale& sc, bool sf_here) {
      const int c = tid + k * T;
      const bool ok = live && c < C;
      const float S = div ? __fmul_rn(e4m3_to_f32(sc.code), scale_in) : 0.0f;
      float t[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (div && S != 0.0f) {
          t[2 * i] = __fdiv_rn(v[i].x, S);
          t[2 * i + 1] = __fdiv_rn(v[i].y, S);
        } else {
          const float2 q = mul2(v[i], f2(sc.mult));
          t[2 * i] = q.x;
          t[2 * i + 1] = q.y;
        }
      }
      const uint32_t packed = pack_e2m1x8(t);
      if constexpr (SWZ) {
        const uint32_t word = sf_word4(sc.code);
        if (ok && (c & 7) == 0)
          *reinterpret_cast<uint32_t*>(a.sf + sf_swizzled_word(row, c >> 3, (C + 7) >> 3)) = word;
      }
      if (ok) {
        *reinterpret_cast<uint32_t*>(qrow + 4 * c) = packed;
        if (!SWZ && sf_here && (c & 1) == 0) a.sf[row * a.ld_sf + (c >> 1)] = uint8_t(sc.code);
      }
    };
    if constexpr (K >= 2) {
#pragma unroll
      for (int k = 0; k < K; k += 2) {
        if (!slot_live(k + 1)) {  // slot k alone (its own block scales), or nothing
          if (slot_live(k)) {
            float2 v[4];
            norm_chunk(k, v);
            quant_store(k, v, nvfp4_block_scale<true>(block_amax(v), scale_in, ngr, g_fast), true);
          }
          continue;
        }
        float2 v0[4], v1[4];
        norm_chunk(k, v0);
        norm_chunk(k + 1, v1);
        Nvfp4Scale s0, s1;
        nvfp4_pair_scales<true>(block_amax(v0), block_amax(v1), tid, scale_in, ngr, g_fast, s0, s1);
        if constexpr (!SWZ) {
          // Each lane stores the block scale it computed (even lane: slot k,
          // odd lane: slot k + 1): one byte per lane, no divergent store.
          // (Measured: 5-6 % faster here; in register rows it cost registers
          // and was slower, so they keep the even-lane store.)
          const bool odd = (tid & 1) != 0;
          const int cm = tid + (k + (odd ? 1 : 0)) * T;
          if (live && cm < C) sfrow[cm >> 1] = uint8_t(odd ? s1.code : s0.code);
        }
        quant_store(k, v0, s0, false);
        quant_store(k + 1, v1, s1, false);
      }
    } else {
      float2 v[4];
      norm_chunk(0, v);
      quant_store(0, v, nvfp4_block_scale<true>(block_amax(v), scale_in, ngr, g_fast), true);
    }
  } else if constexpr (OP == kOpRmsGroupFp8) {
    // The group's chunks are consecutive lanes (see quantize_groups).  Chunk
    // slots go in pairs: the warp holds 2 * gpw groups of a pair, and lane j
    // < 2 * gpw computes the scale of group (slot j / gpw, part j % gpw) once
    // (a correctly rounded division and reciprocal); every lane then takes
    // its own two groups' scale and reciprocal by shuffles.  Group sizes are
    // 64 or 128, so every index below is a shift or a mask.
    const int lcpg = (a.group == 128) ? 4 : 3;  // log2(chunks per group)
    const int cpg = 1 << lcpg, gpw = 32 >> lcpg;
    const int lane = tid & 31;
    const bool ue8m0 = (a.flags & kFlagUe8m0) != 0;
    const bool packed = (a.flags & kFlagScalesPacked) != 0;
    const int64_t n_groups = d >> (lcpg + 3);
    auto group_max = [&](const float2 (&v)[4]) {
      float m = absmax8(v, 0.0f);
      for (int o = cpg >> 1; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
      return m;
    };
    auto scale_of = [&](float m) {
      const float sg = fp8_scale_of<E5>(m);
      return ue8m0 ? ue8m0_ceil(sg) : sg;
    };
    auto quant_store = [&](int k, const float2 (&v)[4], float sg, float ig) {
      const int c = tid + k * T;
      const bool ok = live && c < C;
      float2 t[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        t[i] = (div && sg != 0.0f) ? make_float2(__fdiv_rn(v[i].x, sg), __fdiv_rn(v[i].y, sg)) : mul2(v[i], f2(ig));
      if (ok) {
        *reinterpret_cast<uint2*>(qrow + 8 * c) = pack_pairs_fp8<E5>(t);
        if ((c & (cpg - 1)) == 0) {
          if constexpr (LAYOUT)
            store_group_scale(a.scale_out, a.ld_scale, a.cs_scale, packed, row, c >> lcpg, n_groups, sg);
          else
            a.scale_out[row * a.ld_scale + (c >> lcpg)] = sg;
        }
      }
    };
    if constexpr (K >= 2) {
#pragma unroll
      for (int k = 0; k < K; k += 2) {
        if (!slot_live(k + 1)) {  // slot k alone (every lane its group's scale), or nothing
          if (slot_live(k)) {
            float2 v[4];
            norm_chunk(k, v);
            const float sg = scale_of(group_max(v));
            quant_store(k, v, sg, (sg == 0.0f) ? 0.0f : __frcp_rn(sg));
          }
          continue;
        }
        float2 v0[4], v1[4];
        norm_chunk(k, v0);
        norm_chunk(k + 1, v1);
        const float m0 = group_max(v0), m1 = group_max(v1);
        const int first = (lane & (gpw - 1)) << lcpg;  // first lane of group part j % gpw
        const float t0 = __shfl_sync(kFull, m0, first), t1 = __shfl_sync(kFull, m1, first);
        const float sg = scale_of(lane < gpw ? t0 : t1);  // lanes >= 2 gpw: unused
        const float ig = (sg == 0.0f) ? 0.0f : __frcp_rn(sg);
        const int own = lane >> lcpg;  // this lane's group part
        quant_store(k, v0, __shfl_sync(kFull, sg, own), __shfl_sync(kFull, ig, own));
        quant_store(k + 1, v1, __shfl_sync(kFull, sg, gpw + own), __shfl_sync(kFull, ig, gpw + own));
      }
    } else {
      float2 v[4];
      norm_chunk(0, v);
      const float sg = scale_of(group_max(v));
      quant_store(0, v, sg, (sg == 0.0f) ? 0.0f : __frcp_rn(sg));
    }
  } else {
#pragma unroll
  for (int k = 0; k < K; ++k) {
    if (!slot_live(k)) continue;
    const int c = tid + k * T;
    const bool ok = live && c < C;
    float2 v[4];
    norm_chunk(k, v);
    float2 t[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      t[i] = div ? make_float2(__fdiv_rn(v[i].x, scale_in), __fdiv_rn(v[i].y, scale_in)) : mul2(v[i], inv2);
    if (ok) *reinterpret_cast<uint2*>(qrow + 8 * c) = pack_pairs_fp8<E5>(t);
  }
  }
  };
  if (!div_flag && !bf16_flag && a.norm_out == nullptr) pass3(BoolTag<true>{});
  else pass3(BoolTag<false>{});
  if constexpr (SWZ) {
    if (live) sf_zero_padding_rows<T>(a, row, tid);
  }
}

// NR rows per thread group on the same columns (static RMSNorm and
// LayerNorm without residual): each thread loads its gamma (and beta) chunk
// once for all NR rows, and the rows' sums share one barrier.  The per-row
// arithmetic and its order are those of process_raw_row.
template <int T, int K, int NR>
__device__ __forceinline__ void row_totals_n(float (&part)[NR][K], float (&out)[NR], float* red, int tid) {
#pragma unroll
  for (int r = 0; r < NR; ++r) {
#pragma unroll
    for (int h = K / 2; h >= 1; h >>= 1)
#pragma unroll
      for (int i = 0; i < h; ++i) part[r][i] = __fadd_rn(part[r][i], part[r][i + h]);
    out[r] = part[r][0];
  }
  if constexpr (T > 32) {
    constexpr int W = T / 32;
    const int lane = tid & 31, w = tid >> 5;
#pragma unroll
    for (int r = 0; r < NR; ++r) red[(r * W + w) * 32 + lane] = out[r];
    __syncthreads();
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      float p[W];
#pragma unroll
      for (int i = 0; i < W; ++i) p[i] = red[(r * W + i) * 32 + lane];
#pragma unroll
      for (int h = W / 2; h >= 1; h >>= 1)
#pragma unroll
        for (int i = 0; i < h; ++i) p[i] = __fadd_rn(p[i], p[i + h]);
      out[r] = p[0];
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1)
#pragma unroll
    for (int r = 0; r < NR; ++r) out[r] = __fadd_rn(out[r], __shfl_xor_sync(kFull, out[r], o));
}

template <int OP, int T, int K, int OUT, int NR, bool NARROW = false>
__device__ __forceinline__ void process_raw_rows_n(const RowArgs& a, const int64_t (&row)[NR], int tid,
                                                   const uint4 (&xr)[NR][K], float* b0, float* b1, float scale_in,
                                                   float inv_static) {
  static_assert(OP == kOpRmsStaticFp8 || OP == kOpLnStaticFp8, "two-row form: static RMSNorm / LayerNorm");
  constexpr bool E5 = (OUT & kOutAlt) != 0;
  constexpr bool LN = OP == kOpLnStaticFp8;
  const int d = a.d;
  const int C = d >> 3;
  const float fd = float(d);
  const bool div_flag = (a.flags & kFlagDiv) != 0;
  const bool bf16_flag = (a.flags & kFlagNormBf16) != 0;
  // NARROW: chunk slots wholly past the row for this warp are skipped (see
  // process_raw_row).
  const int wbase = tid & ~31;
  auto slot_live = [&](int k) { return k < K / 2 || wbase + k * T < C; };
  float part[NR][K], total[NR];
#pragma unroll
  for (int r = 0; r < NR; ++r)
#pragma unroll
    for (int k = 0; k < K; ++k) {
      if constexpr (NARROW) {
        if (!slot_live(k)) {
          part[r][k] = 0.0f;
          continue;
        }
      }
      float2 v[4];
      unpack_pairs(xr[r][k], v);
      part[r][k] = chunk_partial<!LN>(v);
    }
  row_totals_n<T, K, NR>(part, total, b0, tid);
  float rstd[NR], mean[NR] = {};
  if constexpr (LN) {
    float sq[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      mean[r] = __fdiv_rn(total[r], fd);
      const float2 nm = f2(-mean[r]);
#pragma unroll
      for (int k = 0; k < K; ++k) {
        const int c = tid + k * T;
        if constexpr (NARROW) {
          if (!slot_live(k)) {
            part[r][k] = 0.0f;
            continue;
          }
        }
        float2 v[4];
        unpack_pairs(xr[r][k], v);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = (K >= 8 && c >= C) ? f2(0.0f) : add2(v[i], nm);
        // A chunk slot past the row adds +0, as a zero chunk would: one
        // select per chunk.  (With eight chunks per thread the per-element
        // form above is kept: ptxas spills less with it.)
        part[r][k] = (K < 8 && c >= C) ? 0.0f : chunk_partial<true>(v);
      }
    }
    row_totals_n<T, K, NR>(part, sq, b1, tid);
#pragma unroll
    for (int r = 0; r < NR; ++r) rstd[r] = __frcp_rn(__fsqrt_rn(__fadd_rn(__fdiv_rn(sq[r], fd), a.eps)));
  } else {
#pragma unroll
    for (int r = 0; r < NR; ++r) rstd[r] = __frcp_rn(__fsqrt_rn(__fadd_rn(__fdiv_rn(total[r], fd), a.eps)));
  }
  const GammaLoads<T> gam{a, tid, C};
  auto pass3 = [&](auto plain_tag) {
    constexpr bool PLAIN = decltype(plain_tag)::value;
    const bool div = PLAIN ? false : div_flag;
    const bool bf16_round = PLAIN ? false : bf16_flag;
    uint16_t* const norm_out = PLAIN ? nullptr : a.norm_out;
    const float2 inv2 = f2(inv_static);
#pragma unroll
    for (int k = 0; k < K; ++k) {
      if constexpr (NARROW) {
        if (!slot_live(k)) continue;
      }
      const int c = tid + k * T;
      float2 g[4], b[4];
      if constexpr (LN) {
        float4 g0, g1, e0, e1;
        gam.ln(k, g0, g1, e0, e1);
        g[0] = make_float2(g0.x, g0.y); g[1] = make_float2(g0.z, g0.w);
        g[2] = make_float2(g1.x, g1.y); g[3] = make_float2(g1.z, g1.w);
        b[0] = make_float2(e0.x, e0.y); b[1] = make_float2(e0.z, e0.w);
        b[2] = make_float2(e1.x, e1.y); b[3] = make_float2(e1.z, e1.w);
      } else {
        unpack_pairs(gam.rms(k), g);
      }
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        const bool ok = row[r] < a.M && c < C;
        float2 v[4];
        unpack_pairs(xr[r][k], v);
        const float2 rs2 = f2(rstd[r]);
        if constexpr (LN) {
          const float2 nm = f2(-mean[r]);
#pragma unroll
          for (int i = 0; i < 4; ++i) v[i] = fma2(mul2(add2(v[i], nm), rs2), g[i], b[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) v[i] = mul2(mul2(v[i], rs2), g[i]);
        }
        if (bf16_round) {
#pragma unroll
          for (int i = 0; i < 4; ++i) v[i] = make_float2(round_bf16(v[i].x), round_bf16(v[i].y));
        }
        if constexpr (!LN) {
          if (norm_out != nullptr && ok)
            *reinterpret_cast<uint4*>(norm_out + row[r] * a.ld_norm + 8 * c) = pack_pairs_bf16(v);
        }
        float2 t[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          t[i] = div ? make_float2(__fdiv_rn(v[i].x, scale_in), __fdiv_rn(v[i].y, scale_in)) : mul2(v[i], inv2);
        if (ok) *reinterpret_cast<uint2*>(a.q + row[r] * a.ld_q + 8 * c) = pack_pairs_fp8<E5>(t);
      }
    }
  };
  if (!div_flag && !bf16_flag && a.norm_out == nullptr) pass3(BoolTag<true>{});
  else pass3(BoolTag<false>{});
}

template <int T, int K, int NR>
constexpr int rows_n_min_blocks() {
  constexpr int cap = 4 * NR * K + 64;  // NR raw rows (4 registers per chunk each) + working set
  constexpr int blocks = 65536 / (T * (cap < 64 ? 64 : cap));
  return blocks < 1 ? 1 : blocks;
}

// NR rows per CTA (T >= 64), raw bf16 chunks in registers, not persistent.
// Built for NR = 2; four rows per CTA measured slower on B200 (their raw
// rows spill or halve the resident CTAs).
template <int OP, int T, int K, int OUT, int NR, bool NARROW>
__global__ void __launch_bounds__(T, (rows_n_min_blocks<T, K, NR>())) row_kernel_rows_n(const RowArgs a) {
  static_assert(T >= 64, "multi-row form: one CTA per group of NR rows");
  constexpr int W = T / 32;
  __shared__ __align__(16) float s_sum[2][NR * W * 32];
  const int tid = int(threadIdx.x);
  const int C = a.d >> 3;
  int64_t row[NR];
#pragma unroll
  for (int r = 0; r < NR; ++r) row[r] = int64_t(blockIdx.x) * NR + r;
  griddep_wait();
  const float scale_in = __ldg(a.scale);
  const float inv_static = __frcp_rn(scale_in);
  uint4 xr[NR][K];
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    const uint16_t* xrow = a.x + row[r] * a.ld_x;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int c = tid + k * T;
      xr[r][k] = (row[r] < a.M && c < C) ? __ldcs(reinterpret_cast<const uint4*>(xrow + 8 * c))
                                         : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  griddep_launch_dependents();
  process_raw_rows_n<OP, T, K, OUT, NR, NARROW>(a, row, tid, xr, s_sum[0], s_sum[1], scale_in, inv_static);
}

// Rows without a residual (static RMSNorm, LayerNorm, NVFP4 without
// residual), 16-byte rows, T > 32.  Only the raw bf16 chunks are kept (half
// the registers of float32); each pass unpacks them again.  With PERSIST the
// CTA walks rows g, g + G, ... and loads the next row's raw chunks before it
// processes the current one, so a load is always in flight; the static scale's
// reciprocal is then computed once per CTA.
// Register budget of the raw kernel: the raw row (4 registers per chunk, 8
// when the next row is prefetched) plus ~48 working registers, at least 64;
// the launch bound asks ptxas to fit it, which stops it from hoisting every
// chunk's gamma / beta loads at once (more CTAs per SM matter more here).
// NVFP4 and the fused group without prefetch take 32 working registers, at
// least 56, even where ptxas then spills a few words: measured on B200,
// NVFP4 128 x 8 chunks at 64 registers (8 CTAs per SM, was 80 and 6) 8192 x
// 7168 42.7 -> 40.2 us and 65536 x 7168 298.4 -> 277.8 us, 128 x 4 at 56 (9
// CTAs) 65536 x 4096 161.3 -> 156.3 us; the fused group 128 x 4 at 56 32768
// x 4096 99.2 -> 95.3 us.
template <int OP, int T, int K, bool PERSIST>
constexpr int raw_min_blocks() {
  constexpr int threads = (T == 32) ? 256 : T;
  constexpr bool LEAN = (OP == kOpRmsNvfp4 || OP == kOpRmsGroupFp8) && !PERSIST;
  constexpr int cap = (PERSIST ? 8 * K : 4 * K) + (LEAN ? 32 : 48);
  constexpr int lo = LEAN ? 56 : 64;
  constexpr int blocks = 65536 / (threads * (cap < lo ? lo : cap));
  return blocks < 1 ? 1 : blocks;
}

template <int OP, int T, int K, bool PERSIST, int OUT, bool NARROW>
__global__ void __launch_bounds__(T == 32 ? 256 : T, (raw_min_blocks<OP, T, K, PERSIST>()))
    row_kernel_raw(const RowArgs a) {
  static_assert(OP != kOpRmsDynFp8, "raw rows: no residual");
  constexpr int R = (T == 32) ? 8 : 1;  // rows per CTA (one warp per row when T == 32)
  constexpr int W = T / 32;
  __shared__ __align__(16) float s_sum[2][W > 1 ? W * 32 : 1];
  const int tid = (T == 32) ? int(threadIdx.x & 31u) : int(threadIdx.x);
  const int64_t group = int64_t(blockIdx.x) * R + int64_t(threadIdx.x / T);
  const int64_t n_groups = int64_t(gridDim.x) * R;
  const int C = a.d >> 3;

  griddep_wait();
  const float scale_in = (OP == kOpRmsGroupFp8) ? 1.0f : __ldg(a.scale);
  const float inv_static = __frcp_rn(scale_in);

  auto load = [&](int64_t row, uint4 (&xr)[K]) {
    const uint16_t* xrow = a.x + row * a.ld_x;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int c = tid + k * T;
      xr[k] = (row < a.M && c < C) ? __ldcs(reinterpret_cast<const uint4*>(xrow + 8 * c)) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  // Persistent CTAs keep gamma as fp32 in (dynamic) shared memory, widened
  // once by the whole CTA (raw_gamma_smem_bytes) while the first row's load
  // is in flight; LayerNorm keeps its fp32 gamma and beta there.
  constexpr bool GSMEM = PERSIST;
  extern __shared__ __align__(16) float4 s_gamma[];  // [2][C], LayerNorm [4][C]: GSMEM only
  auto stage_gamma = [&] {
    if constexpr (GSMEM) {
      for (int c = int(threadIdx.x); c < C; c += int(blockDim.x)) {
        if constexpr (OP == kOpLnStaticFp8) {
          const float4* gp = reinterpret_cast<const float4*>(static_cast<const float*>(a.gamma) + 8 * c);
          const float4* bp = reinterpret_cast<const float4*>(a.beta + 8 * c);
          s_gamma[c] = __ldg(gp), s_gamma[C + c] = __ldg(gp + 1);
          s_gamma[2 * C + c] = __ldg(bp), s_gamma[3 * C + c] = __ldg(bp + 1);
        } else {
          float2 g[4];
          unpack_pairs(__ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.gamma) + 8 * c)), g);
          s_gamma[c] = make_float4(g[0].x, g[0].y, g[1].x, g[1].y);
          s_gamma[C + c] = make_float4(g[2].x, g[2].y, g[3].x, g[3].y);
        }
      }
      __syncthreads();
    }
  };
  auto process = [&](int64_t row, const uint4 (&xr)[K], float* b0, float* b1) {
    if constexpr (GSMEM)
      process_raw_row<OP, T, K, OUT, NARROW>(a, row, tid, [&](int k) { return xr[k]; },
                                             GammaSmem<T, K>{s_gamma, s_gamma + C, tid, C}, b0, b1, scale_in,
                                             inv_static);
    else
      process_raw_row<OP, T, K, OUT, NARROW>(a, row, tid, [&](int k) { return xr[k]; }, GammaLoads<T>{a, tid, C}, b0,
                                             b1, scale_in, inv_static);
  };

  if constexpr (!PERSIST) {
    uint4 xr[K];
    load(group, xr);
    griddep_launch_dependents();
    process(group, xr, s_sum[0], s_sum[1]);
  } else {
    // Reduction buffers are reused row after row: LayerNorm's two sums use
    // both buffers (each separated from its next use by the other sum's
    // barrier); single-sum operations alternate by row parity.
    uint4 xa[K], xb[K];
    int64_t row = group;
    load(row, xa);
    stage_gamma();
    for (int parity = 0; row < a.M; parity ^= 1) {
      const int64_t next = row + n_groups;
      if (next >= a.M) griddep_launch_dependents();  // nothing left to load
      float* b0 = (OP == kOpLnStaticFp8) ? s_sum[0] : s_sum[parity];
      if (parity == 0) {
        load(next, xb);
        process(row, xa, b0, s_sum[1]);
      } else {
        load(next, xa);
        process(row, xb, b0, s_sum[1]);
      }
      row = next;
    }
  }
}

// Kernel table of one operation and output form (OUT bits): every built
// (threads, chunks, vec) schedule.
template <int OP, int OUT>
struct RowTable {
  RowKernels k;
  RowTable() {
    for (auto& x : k.direct)
      for (auto& y : x)
        for (auto& z : y) z = nullptr;
    for (auto& x : k.raw)
      for (auto& y : x)
        for (auto& z : y)
          for (auto& w : z) w = nullptr;
    for (auto& x : k.rows2)
      for (auto& y : x)
        for (auto& z : y) z = nullptr;
    for (auto& x : k.cluster)
      for (auto& y : x) y = nullptr;
    // Rows of 16385 ... 32768 elements: clusters of four CTAs; up to 65536: eight.
#define NQ_CLUSTER(NCI, NC)                                                                                   \
  k.cluster[NCI][0] = reinterpret_cast<const void*>(&row_kernel_cluster<OP, kClusterChunks, 0, OUT, NC>);     \
  k.cluster[NCI][1] = reinterpret_cast<const void*>(&row_kernel_cluster<OP, kClusterChunks, 1, OUT, NC>);     \
  k.cluster[NCI][2] = reinterpret_cast<const void*>(&row_kernel_cluster<OP, kClusterChunks, 2, OUT, NC>);     \
  k.cluster[NCI][3] = reinterpret_cast<const void*>(&row_kernel_cluster<OP, kClusterChunks, 3, OUT, NC>);
    NQ_CLUSTER(0, 4) NQ_CLUSTER(1, 8)
#undef NQ_CLUSTER
#define NQ_RAW(LT, LK)                                                                                         \
  if constexpr (OP != kOpRmsDynFp8 && !(OUT & kOutScatter)) {                                                  \
    k.raw[LT - kMinLogT][LK][0][0] = reinterpret_cast<const void*>(&row_kernel_raw<OP, (1 << LT), (1 << LK), false, OUT, false>); \
    k.raw[LT - kMinLogT][LK][1][0] = reinterpret_cast<const void*>(&row_kernel_raw<OP, (1 << LT), (1 << LK), true, OUT, false>);  \
    k.raw[LT - kMinLogT][LK][0][1] = reinterpret_cast<const void*>(&row_kernel_raw<OP, (1 << LT), (1 << LK), false, OUT, true>);  \
    k.raw[LT - kMinLogT][LK][1][1] = reinterpret_cast<const void*>(&row_kernel_raw<OP, (1 << LT), (1 << LK), true, OUT, true>);   \
  }                                                                                                            \
  if constexpr (OP == kOpRmsStaticFp8 || OP == kOpLnStaticFp8) {                                               \
    if constexpr (LT > 5 && LK <= 3) {                                                                         \
      k.rows2[LT - kMinLogT][LK][0] = reinterpret_cast<const void*>(&row_kernel_rows_n<OP, (1 << LT), (1 << (LK > 3 ? 3 : LK)), OUT, 2, false>); \
      k.rows2[LT - kMinLogT][LK][1] = reinterpret_cast<const void*>(&row_kernel_rows_n<OP, (1 << LT), (1 << (LK > 3 ? 3 : LK)), OUT, 2, true>); \
    }                                                                                                          \
  }
#define NQ_DIRECT(LT, LK)                                                                                 \
  k.direct[LT - kMinLogT][LK][0] = reinterpret_cast<const void*>(&row_kernel<OP, (1 << LT), (1 << LK), 0, OUT>); \
  k.direct[LT - kMinLogT][LK][1] = reinterpret_cast<const void*>(&row_kernel<OP, (1 << LT), (1 << LK), 1, OUT>); \
  if (LT > 5) k.direct[LT - kMinLogT][LK][2] = reinterpret_cast<const void*>(&row_kernel<OP, (1 << LT), (1 << LK), 2, OUT>); \
  if constexpr (LK > 0) k.direct[LT - kMinLogT][LK][3] = reinterpret_cast<const void*>(&row_kernel<OP, (1 << LT), (1 << LK), 3, OUT>); \
  NQ_RAW(LT, LK)
    NQ_DIRECT(5, 0) NQ_DIRECT(5, 1) NQ_DIRECT(5, 2) NQ_DIRECT(5, 3)
    NQ_DIRECT(6, 0) NQ_DIRECT(6, 1) NQ_DIRECT(6, 2) NQ_DIRECT(6, 3)
    NQ_DIRECT(7, 0) NQ_DIRECT(7, 1) NQ_DIRECT(7, 2) NQ_DIRECT(7, 3)
    NQ_DIRECT(8, 0) NQ_DIRECT(8, 1) NQ_DIRECT(8, 2) NQ_DIRECT(8, 3)
    NQ_DIRECT(9, 0) NQ_DIRECT(9, 1)
    k.direct[9 - kMinLogT][2][0] = reinterpret_cast<const void*>(&row_kernel_512<OP, 4, 0, OUT>);
    k.direct[9 - kMinLogT][2][1] = reinterpret_cast<const void*>(&row_kernel_512<OP, 4, 1, OUT>);
    k.direct[9 - kMinLogT][2][2] = reinterpret_cast<const void*>(&row_kernel_512<OP, 4, 2, OUT>);
    k.direct[9 - kMinLogT][2][3] = reinterpret_cast<const void*>(&row_kernel_512<OP, 4, 3, OUT>);
    NQ_RAW(9, 2)
    NQ_DIRECT(10, 0) NQ_DIRECT(10, 1)
    NQ_RAW(5, 4)  // one warp per row, 16 chunks per lane (rows of up to 4096 elements)
#undef NQ_DIRECT
#undef NQ_RAW
  }
};

}  // namespace nq
