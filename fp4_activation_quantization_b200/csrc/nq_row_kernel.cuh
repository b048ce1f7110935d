// nq_row_kernel.cuh — the fused residual-add + norm + quantize row kernel.
//
// One row (token) is owned by a group of T threads: a single warp (T = 32,
// eight rows per CTA) or the whole CTA (T = 64..1024).  Thread t of the group
// owns the 16-byte chunks c = t + k*T, k = 0..K-1, of the row (8 bf16 values
// each), so every load and store instruction of a warp touches one contiguous
// 512-byte span.  The whole row stays in float32 registers from load to
// quantized store: the row is read once, and each output is written once.
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
//   a6 quantize, pack (cvt.rn.satfinite e4m3x2 / e2m1x2) and store.
#pragma once

#include "nq_device.cuh"
#include "nq_internal.h"

namespace nq {

template <int OP, int T, int K, bool VEC>
__global__ void __launch_bounds__(T == 32 ? 256 : T) row_kernel(const RowArgs a) {
  constexpr int R = (T == 32) ? 8 : 1;  // rows per CTA
  constexpr int W = T / 32;             // warps per row
  static_assert(K == 1 || K == 2 || K == 4, "chunks per thread");
  static_assert(R * T <= 1024, "CTA size");

  __shared__ float s_sum[2][W > 1 ? W * 32 : 1];
  __shared__ uint32_t s_max[W > 1 ? W : 1];

  const int tid = (T == 32) ? int(threadIdx.x & 31u) : int(threadIdx.x);
  const int64_t row = (T == 32) ? int64_t(blockIdx.x) * R + int64_t(threadIdx.x >> 5)
                                : int64_t(blockIdx.x);
  // Rows past M (only possible with eight rows per CTA) run every step with
  // zeros so that warp-wide shuffles stay converged, and store nothing.
  const bool live = row < a.M;
  const int d = a.d;
  const int C = (d + 7) >> 3;
  const bool div = (a.flags & kFlagDiv) != 0;
  const bool has_res = (OP != kOpLnStaticFp8) && (a.res_in != nullptr);

  griddep_wait();

  // ---- a1: loads (all issued before any store, for memory-level parallelism)
  float v[K][8];
  uint4 graw[K];     // bf16 gamma chunks (RMSNorm)
  float gf[K][8];    // float gamma (LayerNorm)
  float bf[K][8];    // float beta (LayerNorm)
  const uint16_t* xrow = a.x + row * a.ld_x;
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = tid + k * T;
    const bool ok = live && c < C;
    if constexpr (VEC) {
      uint4 u = make_uint4(0u, 0u, 0u, 0u);
      if (ok) u = __ldcs(reinterpret_cast<const uint4*>(xrow + 8 * c));
      unpack_bf16x8(u, v[k]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int e = 8 * c + j;
        v[k][j] = (live && c < C && e < d) ? bf16_to_f32(xrow[e]) : 0.0f;
      }
    }
  }
  // gamma / beta: shared by every row, served from L1/L2.
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = tid + k * T;
    const bool ok = c < C;
    if constexpr (OP == kOpLnStaticFp8) {
      const float* g = static_cast<const float*>(a.gamma);
      if constexpr (VEC) {
        float4 g0 = make_float4(0.f, 0.f, 0.f, 0.f), g1 = g0, b0 = g0, b1 = g0;
        if (ok) {
          g0 = __ldg(reinterpret_cast<const float4*>(g + 8 * c));
          g1 = __ldg(reinterpret_cast<const float4*>(g + 8 * c + 4));
          b0 = __ldg(reinterpret_cast<const float4*>(a.beta + 8 * c));
          b1 = __ldg(reinterpret_cast<const float4*>(a.beta + 8 * c + 4));
        }
        gf[k][0] = g0.x; gf[k][1] = g0.y; gf[k][2] = g0.z; gf[k][3] = g0.w;
        gf[k][4] = g1.x; gf[k][5] = g1.y; gf[k][6] = g1.z; gf[k][7] = g1.w;
        bf[k][0] = b0.x; bf[k][1] = b0.y; bf[k][2] = b0.z; bf[k][3] = b0.w;
        bf[k][4] = b1.x; bf[k][5] = b1.y; bf[k][6] = b1.z; bf[k][7] = b1.w;
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int e = 8 * c + j;
          gf[k][j] = (ok && e < d) ? __ldg(g + e) : 0.0f;
          bf[k][j] = (ok && e < d) ? __ldg(a.beta + e) : 0.0f;
        }
      }
    } else {
      const uint16_t* g = static_cast<const uint16_t*>(a.gamma);
      if constexpr (VEC) {
        graw[k] = ok ? __ldg(reinterpret_cast<const uint4*>(g + 8 * c)) : make_uint4(0u, 0u, 0u, 0u);
      } else {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int e = 8 * c + 2 * j;
          const uint32_t lo = (ok && e < d) ? uint32_t(__ldg(g + e)) : 0u;
          const uint32_t hi = (ok && e + 1 < d) ? uint32_t(__ldg(g + e + 1)) : 0u;
          w[j] = lo | (hi << 16);
        }
        graw[k] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }

  // ---- a2: residual add and residual write
  if (has_res) {
    const uint16_t* rrow = a.res_in + row * a.ld_res;
    float rv[K][8];
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int c = tid + k * T;
      const bool ok = live && c < C;
      if constexpr (VEC) {
        uint4 u = make_uint4(0u, 0u, 0u, 0u);
        if (ok) u = __ldcs(reinterpret_cast<const uint4*>(rrow + 8 * c));
        unpack_bf16x8(u, rv[k]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int e = 8 * c + j;
          rv[k][j] = (ok && e < d) ? bf16_to_f32(rrow[e]) : 0.0f;
        }
      }
    }
    uint16_t* orow = a.res_out + row * a.ld_res;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int c = tid + k * T;
      const bool ok = live && c < C;
#pragma unroll
      for (int j = 0; j < 8; ++j) v[k][j] = __fadd_rn(v[k][j], rv[k][j]);
      if (ok) {
        if constexpr (VEC) {
          *reinterpret_cast<uint4*>(orow + 8 * c) = pack_bf16x8(v[k]);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (8 * c + j < d) orow[8 * c + j] = f32_to_bf16(v[k][j]);
        }
      }
    }
  }

  // ---- a3: first row sum (sum of squares, or plain sum for LayerNorm)
  float part[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    float p = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if constexpr (OP == kOpLnStaticFp8) p = __fadd_rn(p, v[k][j]);
      else p = __fmaf_rn(v[k][j], v[k][j], p);
    }
    part[k] = p;
  }
#pragma unroll
  for (int h = K / 2; h >= 1; h >>= 1)
#pragma unroll
    for (int i = 0; i < h; ++i) part[i] = __fadd_rn(part[i], part[i + h]);
  const float total = row_sum<T>(part[0], s_sum[0], tid);

  // The next kernel on the stream may start its prologue now.
  griddep_launch_dependents();

  const float fd = float(d);
  float rstd;
  if constexpr (OP == kOpLnStaticFp8) {
    // Centre on the row mean, then the biased variance (second pass, in registers).
    const float mean = __fdiv_rn(total, fd);
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int c = tid + k * T;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const bool in = live && c < C && (VEC || 8 * c + j < d);
        v[k][j] = in ? __fsub_rn(v[k][j], mean) : 0.0f;
      }
    }
#pragma unroll
    for (int k = 0; k < K; ++k) {
      float p = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j) p = __fmaf_rn(v[k][j], v[k][j], p);
      part[k] = p;
    }
#pragma unroll
    for (int h = K / 2; h >= 1; h >>= 1)
#pragma unroll
      for (int i = 0; i < h; ++i) part[i] = __fadd_rn(part[i], part[i + h]);
    const float sq = row_sum<T>(part[0], s_sum[1], tid);
    rstd = __frcp_rn(__fsqrt_rn(__fadd_rn(__fdiv_rn(sq, fd), a.eps)));
  } else {
    rstd = __frcp_rn(__fsqrt_rn(__fadd_rn(__fdiv_rn(total, fd), a.eps)));
  }

  // ---- a4: normalize (y overwrites v)
  const bool bf16_round = (a.flags & kFlagNormBf16) != 0;
#pragma unroll
  for (int k = 0; k < K; ++k) {
    if constexpr (OP == kOpLnStaticFp8) {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[k][j] = __fmaf_rn(__fmul_rn(v[k][j], rstd), gf[k][j], bf[k][j]);
    } else {
      float g[8];
      unpack_bf16x8(graw[k], g);
#pragma unroll
      for (int j = 0; j < 8; ++j) v[k][j] = __fmul_rn(__fmul_rn(v[k][j], rstd), g[j]);
    }
    if (bf16_round) {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[k][j] = round_bf16(v[k][j]);
    }
  }
  if constexpr (OP != kOpLnStaticFp8) {
    if (a.norm_out != nullptr) {
      uint16_t* nrow = a.norm_out + row * a.ld_norm;
#pragma unroll
      for (int k = 0; k < K; ++k) {
        const int c = tid + k * T;
        if (live && c < C) {
          if constexpr (VEC) {
            *reinterpret_cast<uint4*>(nrow + 8 * c) = pack_bf16x8(v[k]);
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              if (8 * c + j < d) nrow[8 * c + j] = f32_to_bf16(v[k][j]);
          }
        }
      }
    }
  }

  // ---- a5 + a6: scale, quantize, pack, store
  if constexpr (OP == kOpRmsNvfp4) {
    const float g = __ldg(a.scale);
    uint8_t* qrow = a.q + row * a.ld_q;
    uint8_t* sfrow = a.sf + row * a.ld_sf;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int c = tid + k * T;
      const bool ok = live && c < C;
      float m8 = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j) m8 = fmaxf(m8, fabsf(v[k][j]));
      // A 16-element block is chunks (c, c^1), held by lanes (t, t^1).
      const float amax = fmaxf(m8, __shfl_xor_sync(kFull, m8, 1));
      const uint32_t sfc = f32_to_e4m3(__fdiv_rn(__fdiv_rn(amax, kE2M1Max), g));
      const float S = __fmul_rn(e4m3_to_f32(sfc), g);
      const float mult = (S == 0.0f) ? 0.0f : __frcp_rn(S);
      float t[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) t[j] = (div && S != 0.0f) ? __fdiv_rn(v[k][j], S) : __fmul_rn(v[k][j], mult);
      const uint32_t packed = pack_e2m1x8(t);
      if (ok) {
        if constexpr (VEC) {
          *reinterpret_cast<uint32_t*>(qrow + 4 * c) = packed;
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) qrow[4 * c + j] = uint8_t(packed >> (8 * j));
        }
        if ((c & 1) == 0) sfrow[c >> 1] = uint8_t(sfc);
      }
    }
  } else {
    float s_div = 1.0f, s_inv = 1.0f;
    bool passthrough = false;
    if constexpr (OP == kOpRmsDynFp8) {
      float m = 0.0f;
#pragma unroll
      for (int k = 0; k < K; ++k)
#pragma unroll
        for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[k][j]));
      const float amax = row_max_nonneg<T>(m, s_max, tid);
      const float s = __fdiv_rn(amax, kE4M3Max);
      if (live && tid == 0) a.scale_out[row] = s;
      s_div = s;
      s_inv = __frcp_rn(s);
      passthrough = (s == 0.0f);  // zero row: store the signed zeros of y
    } else {
      const float sc = __ldg(a.scale);
      s_div = sc;
      s_inv = __frcp_rn(sc);
    }
    uint8_t* qrow = a.q + row * a.ld_q;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int c = tid + k * T;
      float t[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        t[j] = passthrough ? v[k][j] : (div ? __fdiv_rn(v[k][j], s_div) : __fmul_rn(v[k][j], s_inv));
      const uint32_t lo = pack_e4m3x4(t[0], t[1], t[2], t[3]);
      const uint32_t hi = pack_e4m3x4(t[4], t[5], t[6], t[7]);
      if (live && c < C) {
        if constexpr (VEC) {
          *reinterpret_cast<uint2*>(qrow + 8 * c) = make_uint2(lo, hi);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (8 * c + j < d) qrow[8 * c + j] = uint8_t((j < 4 ? lo : hi) >> (8 * (j & 3)));
        }
      }
    }
  }
}

// Kernel table of one operation: every built (threads, chunks, vec) schedule.
template <int OP>
struct RowTable {
  KernelTable t;
  RowTable() {
    for (auto& a : t)
      for (auto& b : a)
        for (auto& c : b) c = nullptr;
#define NQ_ROW_ENTRY(LT, LK)                                                            \
  t[LT - kMinLogT][LK][0] = reinterpret_cast<const void*>(&row_kernel<OP, (1 << LT), (1 << LK), false>); \
  t[LT - kMinLogT][LK][1] = reinterpret_cast<const void*>(&row_kernel<OP, (1 << LT), (1 << LK), true>);
    NQ_ROW_ENTRY(5, 0) NQ_ROW_ENTRY(5, 1) NQ_ROW_ENTRY(5, 2)
    NQ_ROW_ENTRY(6, 0) NQ_ROW_ENTRY(6, 1) NQ_ROW_ENTRY(6, 2)
    NQ_ROW_ENTRY(7, 0) NQ_ROW_ENTRY(7, 1) NQ_ROW_ENTRY(7, 2)
    NQ_ROW_ENTRY(8, 0) NQ_ROW_ENTRY(8, 1) NQ_ROW_ENTRY(8, 2)
    NQ_ROW_ENTRY(9, 0) NQ_ROW_ENTRY(9, 1) NQ_ROW_ENTRY(9, 2)
    NQ_ROW_ENTRY(10, 0) NQ_ROW_ENTRY(10, 1)
#undef NQ_ROW_ENTRY
  }
};

}  // namespace nq
