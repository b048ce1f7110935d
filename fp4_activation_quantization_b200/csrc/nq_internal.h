// nq_internal.h — argument blocks and kernel tables shared by the host
// launcher (nq_host.cu) and the kernel translation units.  Not installed.
#pragma once

#include <cstdint>

namespace nq {

// Operations served by the row kernel (one token = one row of d elements).
enum RowOp : int {
  kOpRmsDynFp8 = 0,     // residual-add + RMSNorm + dynamic per-token e4m3
  kOpRmsStaticFp8 = 1,  // RMSNorm (+residual) + static-scale e4m3
  kOpLnStaticFp8 = 2,   // LayerNorm + static-scale e4m3
  kOpRmsNvfp4 = 3,      // RMSNorm (+residual) + NVFP4
  kOpRmsGroupFp8 = 4,   // RMSNorm (+residual) + per-token-group e4m3
  kNumRowOps = 5
};

// Kernel-side flag bits (the public NQ_FLAG_* values, repeated for the
// device code, which does not include the public header).
constexpr uint32_t kFlagDiv = 1u << 1;
constexpr uint32_t kFlagUe8m0 = 1u << 3;
constexpr uint32_t kFlagNormBf16 = 1u << 4;
constexpr uint32_t kFlagE5m2 = 1u << 5;           // FP8 outputs in e5m2
constexpr uint32_t kFlagScalesPacked = 1u << 8;   // group scales as packed UE8M0 exponent bytes

// Output-form bits of the kernel instantiations (template parameter OUT).
constexpr int kOutAlt = 1;          // e5m2 codes (FP8 ops) / swizzled block scales (NVFP4)
constexpr int kOutScaleLayout = 2;  // group ops: column-major or packed-UE8M0 group scales
constexpr int kOutScatter = 4;      // dynamic / group FP8 rows stored to MoE destination rows

struct RowArgs {
  const uint16_t* x;  // bf16 [M, ld_x]
  int64_t ld_x;
  const uint16_t* res_in;  // bf16 [M, ld_res] or null
  uint16_t* res_out;       // bf16 [M, ld_res] or null (may equal res_in)
  int64_t ld_res;
  const void* gamma;   // bf16 [d] (RMSNorm) or float [d] (LayerNorm)
  const float* beta;   // float [d] (LayerNorm)
  const float* scale;  // device scalar: static scale or NVFP4 global scale
  uint8_t* q;          // e4m3 [M, ld_q] or packed e2m1 [M, ld_q]
  int64_t ld_q;
  float* scale_out;  // float [M] (dynamic per-token) or the group scales
  int64_t ld_scale;  // group scale (row, g) at row * ld_scale + g * cs_scale (elements; bytes
  int64_t cs_scale;  // and g / 4 in place of g when packed, see store_group_scale)
  int32_t group;     // 64 or 128 (group op)
  uint8_t* sf;       // e4m3 block scales [M, ld_sf] (NVFP4)
  int64_t ld_sf;
  uint16_t* norm_out;  // bf16 [M, ld_norm] or null
  int64_t ld_norm;
  int64_t M;
  int32_t d;
  float eps;
  uint32_t flags;  // kFlag* bits; kFlagDiv set means divide, clear means reciprocal
  uint32_t* err;   // device error word: bit 1 a destination row out of range
  const int32_t* dest;  // [M, topk] destination rows (kOutScatter); < 0 skips
  int32_t topk;
  int64_t dest_rows;    // rows of q / scales when scattering
};

struct GroupArgs {
  const uint16_t* x;  // bf16 [M, ld_x]
  int64_t ld_x;
  uint8_t* q;  // e4m3 [M, ld_q]
  int64_t ld_q;
  float* s;      // group scales: (row, g) at row * ld_s + g * cs_s (see store_group_scale)
  int64_t ld_s;
  int64_t cs_s;
  int64_t groups_per_row;
  int64_t G;  // M * groups_per_row
  // Row of flat group g (g / groups_per_row) without a 64-bit division: for G
  // < 2^31, (g * row_magic) >> row_shift with row_shift = 32 + ceil(log2
  // groups_per_row) and row_magic = ceil(2^row_shift / groups_per_row) < 2^33
  // is exact (the error g * (row_magic - 2^row_shift / gpr) / 2^row_shift stays
  // below 1 / (2 gpr), Granlund and Montgomery, PLDI 1994).  row_magic = 0:
  // divide.
  uint64_t row_magic;
  int32_t row_shift;
  uint32_t flags;
};

// Schedules: 2^t threads per row (t = 5..10), 2^k chunks of 8 elements per
// thread (k = 0..3, with t + k <= 11, i.e. up to 2048 chunks = 16384
// elements).  Rows per CTA: 8 when t == 5 (one warp per row), else 1.  Wider
// rows take a cluster of CTAs (ClusterTable).
constexpr int kMinLogT = 5, kMaxLogT = 10, kMaxLogK = 3;
inline int rows_per_cta(int threads) { return threads == 32 ? 8 : 1; }
inline bool schedule_built(int log_t, int log_k) {
  return log_t >= kMinLogT && log_t <= kMaxLogT && log_k >= 0 && log_k <= kMaxLogK && log_t + log_k <= 11;
}

// Host-side kernel tables (pointer to the __global__ stub), one per
// translation unit: [log_t - 5][log_k][mode], mode 0 = any alignment,
// 1 = 16-byte rows, 2 = 16-byte rows with d == 8 * threads * chunks (t > 5),
// 3 = 16-byte rows with d < 8 * threads * chunks (k > 0).
using KernelTable = const void* [kMaxLogT - kMinLogT + 1][kMaxLogK + 1][4];
// Raw-row schedules: those of the direct kernel, plus one warp per row with 16
// chunks per lane (t = 5, k = 4).
inline bool raw_schedule_built(int log_t, int log_k) {
  return schedule_built(log_t, log_k) || (log_t == 5 && log_k == 4);
}
using RawTable = const void* [kMaxLogT - kMinLogT + 1][kMaxLogK + 2][2][2];
using Rows2Table = const void* [kMaxLogT - kMinLogT + 1][kMaxLogK + 2][2];
// Rows wider than 16384 elements: one row per cluster of 4 (rows of up to
// 32768 elements) or 8 (up to 65536) CTAs of 256 threads, 4 chunks per
// thread: [clusters of 4, 8][mode as KernelTable].
constexpr int kClusterThreads = 256, kClusterChunks = 4;
using ClusterTable = const void* [2][4];
struct RowKernels {
  KernelTable direct;    // one row per thread group
  RawTable raw;          // rows without residual, raw bf16 in registers: [.][.][persistent][row narrower than T * K * 8]
  Rows2Table rows2;      // two rows per CTA on the same columns (static RMSNorm / LayerNorm): [.][.][narrow row]
  ClusterTable cluster;  // one row per thread-block cluster
};
// Dynamic shared memory of a persistent raw-row kernel: gamma as fp32 (the
// RMSNorm-type operations), or LayerNorm's fp32 gamma and beta.
inline size_t raw_gamma_smem_bytes(int op, int64_t d) { return size_t(d) * (op == kOpLnStaticFp8 ? 8u : 4u); }
const RowKernels& row_kernels_rms_dyn();
const RowKernels& row_kernels_rms_static();
const RowKernels& row_kernels_ln_static();
const RowKernels& row_kernels_rms_nvfp4();
const RowKernels& row_kernels_rms_group();
const RowKernels& row_kernels_rms_dyn_e5m2();
const RowKernels& row_kernels_rms_static_e5m2();
const RowKernels& row_kernels_ln_static_e5m2();
const RowKernels& row_kernels_rms_group_e5m2();
const RowKernels& row_kernels_rms_nvfp4_swizzled();
const RowKernels& row_kernels_rms_group_layout();
const RowKernels& row_kernels_rms_group_e5m2_layout();
const RowKernels& row_kernels_rms_dyn_scatter();
const RowKernels& row_kernels_rms_group_scatter();

// Group kernel: [e5m2][strided / packed scales][group == 128][log2(lanes per group) - 1]
// [log2(groups per thread)][vec]
using GroupTable = const void* [2][2][2][4][3][2];
const GroupTable& group_kernels();
constexpr int kGroupThreads = 256;

}  // namespace nq
