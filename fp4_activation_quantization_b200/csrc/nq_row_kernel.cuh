// nq_row_kernel.cuh — the fused residual-add + norm + quantize row kernels.
//
// One row (token) is owned by a group of T threads: a single warp (T = 32,
// eight rows per CTA) or the whole CTA (T = 64..1024).  Thread t of the group
// owns the 16-byte chunks c = t + k*T, k = 0..K-1, of the row (8 bf16 values
// each), so every load and store instruction of a warp touches one contiguous
// 512-byte span.  The row stays in float32 registers from load to quantized
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
//   a6 quantize, pack (cvt.rn.satfinite e4m3x2 / e2m1x2) and store.
//
// Two kernels share that per-row body:
//   row_kernel        one row per thread group, loads straight to registers;
//                     the choice for few rows (latency) and unaligned rows;
//   row_kernel_staged persistent thread groups that walk rows with a stride
//                     and keep the next STAGES-1 rows in flight through a
//                     per-thread cp.async ring in shared memory, so HBM
//                     traffic never stalls on the row's reductions.  Each
//                     thread copies and later reads only its own chunks, so
//                     the ring needs no barrier and no flag: cp.async.wait_group
//                     is the only wait.
#pragma once

#include "nq_device.cuh"
#include "nq_internal.h"

namespace nq {

// Per-thread copies of gamma (and beta) for the chunks the thread owns.
template <int K>
struct GammaRegs {
  uint4 g16[K];     // bf16 gamma (RMSNorm)
  float gf[K][8];   // float gamma (LayerNorm)
  float bf[K][8];   // float beta (LayerNorm)
};

template <int OP, int T, int K, bool VEC>
__device__ __forceinline__ void load_gamma(const RowArgs& a, int tid, int C, GammaRegs<K>& G) {
  const int d = a.d;
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
        G.gf[k][0] = g0.x; G.gf[k][1] = g0.y; G.gf[k][2] = g0.z; G.gf[k][3] = g0.w;
        G.gf[k][4] = g1.x; G.gf[k][5] = g1.y; G.gf[k][6] = g1.z; G.gf[k][7] = g1.w;
        G.bf[k][0] = b0.x; G.bf[k][1] = b0.y; G.bf[k][2] = b0.z; G.bf[k][3] = b0.w;
        G.bf[k][4] = b1.x; G.bf[k][5] = b1.y; G.bf[k][6] = b1.z; G.bf[k][7] = b1.w;
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int e = 8 * c + j;
          G.gf[k][j] = (ok && e < d) ? __ldg(g + e) : 0.0f;
          G.bf[k][j] = (ok && e < d) ? __ldg(a.beta + e) : 0.0f;
        }
      }
    } else {
      const uint16_t* g = static_cast<const uint16_t*>(a.gamma);
      if constexpr (VEC) {
        G.g16[k] = ok ? __ldg(reinterpret_cast<const uint4*>(g + 8 * c)) : make_uint4(0u, 0u, 0u, 0u);
      } else {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int e = 8 * c + 2 * j;
          const uint32_t lo = (ok && e < d) ? uint32_t(__ldg(g + e)) : 0u;
          const uint32_t hi = (ok && e + 1 < d) ? uint32_t(__ldg(g + e + 1)) : 0u;
          w[j] = lo | (hi << 16);
        }
        G.g16[k] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
}

// Row chunks of a bf16 row straight from global memory (zeros past the row).
template <int T, int K, bool VEC>
__device__ __forceinline__ void load_row(const uint16_t* rowp, int d, int C, int tid, bool live,
                                         float (&v)[K][8]) {
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = tid + k * T;
    const bool ok = live && c < C;
    if constexpr (VEC) {
      uint4 u = make_uint4(0u, 0u, 0u, 0u);
      if (ok) u = __ldcs(reinterpret_cast<const uint4*>(rowp + 8 * c));
      unpack_bf16x8(u, v[k]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int e = 8 * c + j;
        v[k][j] = (ok && e < d) ? bf16_to_f32(rowp[e]) : 0.0f;
      }
    }
  }
}

// Steps a2..a6 of one row whose x (v) and residual (rv, when has_res) chunks
// are in registers.  Contains the row group's barriers (T > 32).
template <int OP, int T, int K, bool VEC>
__device__ __forceinline__ void row_finish(const RowArgs& a, int64_t row, bool live, int tid,
                                           float (&v)[K][8], const float (&rv)[K][8], bool has_res,
                                           const GammaRegs<K>& G, float* s_sum0, float* s_sum1,
                                           uint32_t* s_max) {
  const int d = a.d;
  const int C = (d + 7) >> 3;
  const bool div = (a.flags & kFlagDiv) != 0;

  // ---- a2: residual add and residual write
  if (has_res) {
    uint16_t* orow = a.res_out + row * a.ld_res;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int c = tid + k * T;
#pragma unroll
      for (int j = 0; j < 8; ++j) v[k][j] = __fadd_rn(v[k][j], rv[k][j]);
      if (live && c < C) {
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
  const float total = row_sum<T>(part[0], s_sum0, tid);

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
    const float sq = row_sum<T>(part[0], s_sum1, tid);
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
      for (int j = 0; j < 8; ++j) v[k][j] = __fmaf_rn(__fmul_rn(v[k][j], rstd), G.gf[k][j], G.bf[k][j]);
    } else {
      float g[8];
      unpack_bf16x8(G.g16[k], g);
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

// ------------------------------------------------------------- direct ----
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
  const int C = (a.d + 7) >> 3;
  const bool has_res = (OP != kOpLnStaticFp8) && (a.res_in != nullptr);

  griddep_wait();

  // All loads are issued before any store, for memory-level parallelism.
  float v[K][8], rv[K][8];
  load_row<T, K, VEC>(a.x + row * a.ld_x, a.d, C, tid, live, v);
  GammaRegs<K> G;
  load_gamma<OP, T, K, VEC>(a, tid, C, G);
  if (has_res) load_row<T, K, VEC>(a.res_in + row * a.ld_res, a.d, C, tid, live, rv);
  // The next kernel on the stream may start its prologue now.
  griddep_launch_dependents();
  row_finish<OP, T, K, VEC>(a, row, live, tid, v, rv, has_res, G, s_sum[0], s_sum[1], s_max);
}

// ------------------------------------------------------------- staged ----
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
               "l"(gmem), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
// Wait until at most n of this thread's committed groups are pending (n in 0..7).
__device__ __forceinline__ void cp_async_wait_pending(int n) {
  switch (n) {
    case 0: asm volatile("cp.async.wait_group 0;\n" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;\n" ::: "memory"); break;
    case 2: asm volatile("cp.async.wait_group 2;\n" ::: "memory"); break;
    case 3: asm volatile("cp.async.wait_group 3;\n" ::: "memory"); break;
    case 4: asm volatile("cp.async.wait_group 4;\n" ::: "memory"); break;
    case 5: asm volatile("cp.async.wait_group 5;\n" ::: "memory"); break;
    case 6: asm volatile("cp.async.wait_group 6;\n" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 7;\n" ::: "memory"); break;
  }
}

// Persistent, 16-byte-aligned rows only.  Thread group g (of G = gridDim.x * R
// groups) handles rows g, g + G, g + 2G, ...  Dynamic shared memory holds
// `stages` ring slots of NT (1 or 2: x, residual) x K chunks per thread.  The
// row being processed stays in its slot and is streamed through registers one
// chunk at a time, once per pass (sum; LayerNorm variance; absmax; quantize):
// r = x + residual is recomputed from the slot in each pass (same bits), so
// the register count does not grow with the row width and many rows can be
// in flight per SM.  gamma / beta are re-read per chunk through L1.
template <int OP, int T, int K>
__global__ void __launch_bounds__(T == 32 ? 256 : T, 1024 / (T == 32 ? 256 : T))
    row_kernel_staged(const RowArgs a, int stages) {  // <= 64 registers: >= 1024 threads per SM
  constexpr int R = (T == 32) ? 8 : 1;
  constexpr int W = T / 32;
  constexpr int NTHR = R * T;
  __shared__ float s_sum[2][W > 1 ? W * 32 : 1];
  __shared__ uint32_t s_max[W > 1 ? W : 1];
  extern __shared__ uint4 ring[];

  const int tid = (T == 32) ? int(threadIdx.x & 31u) : int(threadIdx.x);
  const int64_t group = int64_t(blockIdx.x) * R + int64_t(threadIdx.x / T);
  const int64_t n_groups = int64_t(gridDim.x) * R;
  const int64_t nrows = group < a.M ? (a.M - group + n_groups - 1) / n_groups : 0;
  const int d = a.d;
  const int C = d >> 3;  // 16-byte rows: d % 8 == 0
  const bool has_res = (OP != kOpLnStaticFp8) && (a.res_in != nullptr);
  const int NT = has_res ? 2 : 1;
  const bool div = (a.flags & kFlagDiv) != 0;
  const bool bf16_round = (a.flags & kFlagNormBf16) != 0;
  const float fd = float(d);

  griddep_wait();

  auto issue = [&](int64_t j) {  // prefetch row j of this group into slot j % stages
    if (j < nrows) {
      const int64_t row = group + j * n_groups;
      uint4* base = ring + size_t(j % stages) * NT * K * NTHR + threadIdx.x;
      const uint16_t* xr = a.x + row * a.ld_x;
      const uint16_t* rr = a.res_in + row * a.ld_res;
#pragma unroll
      for (int k = 0; k < K; ++k) {
        const int c = tid + k * T;
        const bool ok = c < C;
        cp_async16(base + k * NTHR, ok ? xr + 8 * c : a.x, ok ? 16u : 0u);
        if (has_res) cp_async16(base + (K + k) * NTHR, ok ? rr + 8 * c : a.res_in, ok ? 16u : 0u);
      }
    }
    cp_async_commit();  // one group per row index, empty past the end, so the counting stays uniform
  };
  for (int j = 0; j < stages - 1; ++j) issue(j);

  const int64_t trigger = nrows > stages - 1 ? nrows - (stages - 1) : 0;
  if (nrows == 0) griddep_launch_dependents();
  const float scale_static = (OP == kOpRmsStaticFp8 || OP == kOpLnStaticFp8 || OP == kOpRmsNvfp4)
                                 ? __ldg(a.scale) : 1.0f;

  for (int64_t j = 0; j < nrows; ++j) {
    issue(j + stages - 1);  // refills the slot consumed in iteration j - 1
    cp_async_wait_pending(stages - 1);
    if (j == trigger) griddep_launch_dependents();  // every remaining row is in flight
    const int64_t row = group + j * n_groups;
    const uint4* xs = ring + size_t(j % stages) * NT * K * NTHR + threadIdx.x;
    const uint4* rs = xs + K * NTHR;
    // r (8 values of chunk k): x, plus the residual when there is one.
    auto load_r = [&](int k, float (&r)[8]) {
      unpack_bf16x8(xs[k * NTHR], r);
      if (has_res) {
        float t[8];
        unpack_bf16x8(rs[k * NTHR], t);
#pragma unroll
        for (int e = 0; e < 8; ++e) r[e] = __fadd_rn(r[e], t[e]);
      }
    };
    // Reduction buffers are reused row after row.  LayerNorm's two sums use
    // both buffers, each separated from its next use by the other sum's
    // barrier; single-sum operations alternate by row parity.
    float* b0 = (OP == kOpLnStaticFp8) ? s_sum[0] : s_sum[j & 1];

    // ---- pass A: residual write and first row sum
    float part[K];
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int c = tid + k * T;
      float r[8];
      load_r(k, r);
      if (has_res && c < C) *reinterpret_cast<uint4*>(a.res_out + row * a.ld_res + 8 * c) = pack_bf16x8(r);
      float p = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if constexpr (OP == kOpLnStaticFp8) p = __fadd_rn(p, r[e]);
        else p = __fmaf_rn(r[e], r[e], p);
      }
      part[k] = p;
    }
#pragma unroll
    for (int h = K / 2; h >= 1; h >>= 1)
#pragma unroll
      for (int i = 0; i < h; ++i) part[i] = __fadd_rn(part[i], part[i + h]);
    const float total = row_sum<T>(part[0], b0, tid);

    float rstd, mean = 0.0f;
    if constexpr (OP == kOpLnStaticFp8) {
      mean = __fdiv_rn(total, fd);
#pragma unroll
      for (int k = 0; k < K; ++k) {
        const int c = tid + k * T;
        float r[8];
        load_r(k, r);
        float p = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float ce = (c < C) ? __fsub_rn(r[e], mean) : 0.0f;
          p = __fmaf_rn(ce, ce, p);
        }
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

    // y (8 values of chunk k) from the slot.
    auto make_y = [&](int k, float (&y)[8]) {
      const int c = tid + k * T;
      float r[8];
      load_r(k, r);
      if constexpr (OP == kOpLnStaticFp8) {
        float4 g0 = make_float4(0.f, 0.f, 0.f, 0.f), g1 = g0, e0 = g0, e1 = g0;
        if (c < C) {
          const float* gp = static_cast<const float*>(a.gamma) + 8 * c;
          g0 = __ldg(reinterpret_cast<const float4*>(gp));
          g1 = __ldg(reinterpret_cast<const float4*>(gp + 4));
          e0 = __ldg(reinterpret_cast<const float4*>(a.beta + 8 * c));
          e1 = __ldg(reinterpret_cast<const float4*>(a.beta + 8 * c + 4));
        }
        const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        const float bb[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float ce = (c < C) ? __fsub_rn(r[e], mean) : 0.0f;
          y[e] = __fmaf_rn(__fmul_rn(ce, rstd), gg[e], bb[e]);
        }
      } else {
        uint4 gu = make_uint4(0u, 0u, 0u, 0u);
        if (c < C) gu = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.gamma) + 8 * c));
        float g[8];
        unpack_bf16x8(gu, g);
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = __fmul_rn(__fmul_rn(r[e], rstd), g[e]);
      }
      if (bf16_round) {
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = round_bf16(y[e]);
      }
    };
    auto store_e4m3 = [&](int k, const float (&t)[8]) {
      const int c = tid + k * T;
      const uint32_t lo = pack_e4m3x4(t[0], t[1], t[2], t[3]);
      const uint32_t hi = pack_e4m3x4(t[4], t[5], t[6], t[7]);
      if (c < C) *reinterpret_cast<uint2*>(a.q + row * a.ld_q + 8 * c) = make_uint2(lo, hi);
    };

    // ---- pass B: normalize; static scales and NVFP4 quantize here
    float m = 0.0f;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int c = tid + k * T;
      float y[8];
      make_y(k, y);
      if constexpr (OP != kOpLnStaticFp8) {
        if (a.norm_out != nullptr && c < C)
          *reinterpret_cast<uint4*>(a.norm_out + row * a.ld_norm + 8 * c) = pack_bf16x8(y);
      }
      if constexpr (OP == kOpRmsDynFp8) {
#pragma unroll
        for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(y[e]));
      } else if constexpr (OP == kOpRmsNvfp4) {
        float m8 = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) m8 = fmaxf(m8, fabsf(y[e]));
        const float amax = fmaxf(m8, __shfl_xor_sync(kFull, m8, 1));  // chunks c, c^1 form a block
        const uint32_t sfc = f32_to_e4m3(__fdiv_rn(__fdiv_rn(amax, kE2M1Max), scale_static));
        const float S = __fmul_rn(e4m3_to_f32(sfc), scale_static);
        const float mult = (S == 0.0f) ? 0.0f : __frcp_rn(S);
        float t[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) t[e] = (div && S != 0.0f) ? __fdiv_rn(y[e], S) : __fmul_rn(y[e], mult);
        const uint32_t packed = pack_e2m1x8(t);
        if (c < C) {
          *reinterpret_cast<uint32_t*>(a.q + row * a.ld_q + 4 * c) = packed;
          if ((c & 1) == 0) a.sf[row * a.ld_sf + (c >> 1)] = uint8_t(sfc);
        }
      } else {
        const float inv = __frcp_rn(scale_static);
        float t[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) t[e] = div ? __fdiv_rn(y[e], scale_static) : __fmul_rn(y[e], inv);
        store_e4m3(k, t);
      }
    }

    // ---- pass C (dynamic per-token scale): quantize with the row's scale
    if constexpr (OP == kOpRmsDynFp8) {
      const float amax = row_max_nonneg<T>(m, s_max, tid);
      const float sc = __fdiv_rn(amax, kE4M3Max);
      if (tid == 0) a.scale_out[row] = sc;
      const float inv = __frcp_rn(sc);
      const bool passthrough = (sc == 0.0f);  // zero row: store the signed zeros of y
#pragma unroll
      for (int k = 0; k < K; ++k) {
        float y[8], t[8];
        make_y(k, y);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          t[e] = passthrough ? y[e] : (div ? __fdiv_rn(y[e], sc) : __fmul_rn(y[e], inv));
        store_e4m3(k, t);
      }
    }
  }
  cp_async_wait_pending(0);
}

// Kernel tables of one operation: every built (threads, chunks, vec) schedule
// of the direct kernel, and every (threads, chunks) of the staged kernel.
template <int OP>
struct RowTable {
  RowKernels k;
  RowTable() {
    for (auto& x : k.direct)
      for (auto& y : x)
        for (auto& z : y) z = nullptr;
    for (auto& x : k.staged)
      for (auto& y : x) y = nullptr;
#define NQ_DIRECT(LT, LK)                                                                                     \
  k.direct[LT - kMinLogT][LK][0] = reinterpret_cast<const void*>(&row_kernel<OP, (1 << LT), (1 << LK), false>); \
  k.direct[LT - kMinLogT][LK][1] = reinterpret_cast<const void*>(&row_kernel<OP, (1 << LT), (1 << LK), true>);
#define NQ_STAGED(LT, LK) \
  k.staged[LT - kMinLogT][LK] = reinterpret_cast<const void*>(&row_kernel_staged<OP, (1 << LT), (1 << LK)>);
    NQ_DIRECT(5, 0) NQ_DIRECT(5, 1) NQ_DIRECT(5, 2)
    NQ_DIRECT(6, 0) NQ_DIRECT(6, 1) NQ_DIRECT(6, 2)
    NQ_DIRECT(7, 0) NQ_DIRECT(7, 1) NQ_DIRECT(7, 2)
    NQ_DIRECT(8, 0) NQ_DIRECT(8, 1) NQ_DIRECT(8, 2)
    NQ_DIRECT(9, 0) NQ_DIRECT(9, 1) NQ_DIRECT(9, 2)
    NQ_DIRECT(10, 0) NQ_DIRECT(10, 1)
    NQ_STAGED(5, 0) NQ_STAGED(5, 1) NQ_STAGED(5, 2) NQ_STAGED(5, 3) NQ_STAGED(5, 4)
    NQ_STAGED(6, 0) NQ_STAGED(6, 1) NQ_STAGED(6, 2) NQ_STAGED(6, 3) NQ_STAGED(6, 4)
    NQ_STAGED(7, 0) NQ_STAGED(7, 1) NQ_STAGED(7, 2) NQ_STAGED(7, 3) NQ_STAGED(7, 4)
    NQ_STAGED(8, 0) NQ_STAGED(8, 1) NQ_STAGED(8, 2) NQ_STAGED(8, 3)
    NQ_STAGED(9, 0) NQ_STAGED(9, 1) NQ_STAGED(9, 2)
#undef NQ_DIRECT
#undef NQ_STAGED
  }
};

}  // namespace nq
