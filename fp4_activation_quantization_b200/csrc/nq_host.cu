// nq_host.cu — the C ABI of libnq: argument validation, schedule planning and
// kernel launch.  Declarations and the contract of every entry point are in
// include/nq.h.  Nothing here allocates, synchronizes or reads device memory.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <string>
#include <vector>

#include "nq.h"
#include "nq_device.cuh"
#include "nq_internal.h"

// Device error word of this library: bit 1 is set by a MoE dispatch whose
// destination row was out of range (read and cleared by
// nq_check_device_errors).  A symbol, not an allocation; one per device.
__device__ uint32_t g_nq_device_error;
// Where take_error_word leaves the word it cleared, for the host to read.
__device__ uint32_t g_nq_device_error_taken;

// Read and clear the error word in one atomic step, so that a bit a kernel
// sets between the read and the clear cannot be lost.
__global__ void take_error_word_kernel() { g_nq_device_error_taken = atomicExch(&g_nq_device_error, 0u); }

// Exhaustive check of the bounded division (nq_selftest_division): for
// a = the float with bits a_begin + i and each divisor b in its domain, count
// quotients q of div_rn_by / div2_rn_by that break its contract against the
// correctly rounded ref = __fdiv_rn(a, b): q == ref bit for bit when
// |ref| >= 2^-24; below, q has the sign of ref and |q| < 2^-20, so both give
// the same (signed zero) FP8 code.
__device__ __forceinline__ unsigned selftest_bad(float q, float ref) {
  if (fabsf(ref) >= 5.9604645e-08f) return __float_as_uint(q) != __float_as_uint(ref);  // 2^-24
  return ((__float_as_uint(q) ^ __float_as_uint(ref)) >> 31) | (fabsf(q) >= 9.5367432e-07f);  // 2^-20
}
__global__ void __launch_bounds__(256) selftest_division_kernel(uint32_t a_begin, uint64_t count, const float* divs,
                                                                int n_div, unsigned long long* mismatches) {
  unsigned long long local = 0;
  const uint64_t stride = uint64_t(gridDim.x) * blockDim.x;
  for (uint64_t i = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < count; i += stride) {
    const float a = __uint_as_float(uint32_t(a_begin + i));
    const float a2 = __uint_as_float(uint32_t(a_begin + i) ^ 0x80000000u);  // the other sign, second lane
    for (int j = 0; j < n_div; ++j) {
      const float b = divs[j];
      if (!nq::fast_div_ok(b) || !(fabsf(a) <= 131072.0f * b)) continue;  // outside the domain (NaN too)
      const float nr = -__frcp_rn(b);
      const float ref = __fdiv_rn(a, b), ref2 = __fdiv_rn(a2, b);
      const float2 q2 = nq::div2_rn_by(make_float2(a, a2), make_float2(b, b), make_float2(nr, nr));
      local += selftest_bad(nq::div_rn_by(a, b, nr), ref);
      local += selftest_bad(q2.x, ref) + selftest_bad(q2.y, ref2);
    }
  }
  for (int o = 16; o >= 1; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
  if ((threadIdx.x & 31) == 0 && local) atomicAdd(mismatches, local);
}

namespace {

using nq::RowArgs;
using nq::GroupArgs;

thread_local std::string g_last_error;

nq_status fail(nq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr uint32_t kKnownFlags = NQ_FLAG_PDL | NQ_FLAG_SCALE_DIV | NQ_FLAG_SCALE_RECIP |
                                 NQ_FLAG_UE8M0 | NQ_FLAG_NORM_BF16_ROUND | NQ_FLAG_E5M2 |
                                 NQ_FLAG_SF_SWIZZLED | NQ_FLAG_SCALES_COL_MAJOR | NQ_FLAG_SCALES_PACKED_UE8M0 |
                                 NQ_FLAG_SCHEDULE_MASK | NQ_FLAG_VARIANT_MASK;

nq_status check_flags(const char* fn, uint32_t flags, bool allow_ue8m0, bool allow_schedule,
                      bool allow_bf16_round, bool nvfp4 = false) {
  if (flags & ~kKnownFlags) return fail(NQ_ERR_INVALID_ARGUMENT, "%s: unknown flag bits 0x%x", fn, flags & ~kKnownFlags);
  if ((flags & NQ_FLAG_E5M2) && nvfp4)
    return fail(NQ_ERR_INVALID_ARGUMENT, "%s: NQ_FLAG_E5M2 applies to the FP8 calls only", fn);
  if ((flags & NQ_FLAG_SF_SWIZZLED) && !nvfp4)
    return fail(NQ_ERR_INVALID_ARGUMENT, "%s: NQ_FLAG_SF_SWIZZLED applies to the NVFP4 call only", fn);
  if ((flags & NQ_FLAG_SCALE_DIV) && (flags & NQ_FLAG_SCALE_RECIP))
    return fail(NQ_ERR_INVALID_ARGUMENT, "%s: NQ_FLAG_SCALE_DIV and NQ_FLAG_SCALE_RECIP are exclusive", fn);
  if ((flags & (NQ_FLAG_UE8M0 | NQ_FLAG_SCALES_COL_MAJOR | NQ_FLAG_SCALES_PACKED_UE8M0)) && !allow_ue8m0)
    return fail(NQ_ERR_INVALID_ARGUMENT,
                "%s: NQ_FLAG_UE8M0 / NQ_FLAG_SCALES_* apply to group quantization only", fn);
  if ((flags & (NQ_FLAG_SCHEDULE_MASK | NQ_FLAG_VARIANT_MASK)) && !allow_schedule)
    return fail(NQ_ERR_INVALID_ARGUMENT, "%s: NQ_FLAG_SCHEDULE / NQ_FLAG_VARIANT apply to the norm calls only", fn);
  if ((flags & NQ_FLAG_NORM_BF16_ROUND) && !allow_bf16_round)
    return fail(NQ_ERR_INVALID_ARGUMENT, "%s: NQ_FLAG_NORM_BF16_ROUND needs a norm", fn);
  return NQ_OK;
}

uint32_t kernel_flags(uint32_t flags, bool default_div) {
  const bool div = (flags & NQ_FLAG_SCALE_DIV) ? true : (flags & NQ_FLAG_SCALE_RECIP) ? false : default_div;
  uint32_t k = 0;
  if (div) k |= nq::kFlagDiv;
  if (flags & NQ_FLAG_UE8M0) k |= nq::kFlagUe8m0;
  if (flags & NQ_FLAG_NORM_BF16_ROUND) k |= nq::kFlagNormBf16;
  if (flags & NQ_FLAG_E5M2) k |= nq::kFlagE5m2;
  if (flags & NQ_FLAG_SCALES_PACKED_UE8M0) k |= nq::kFlagUe8m0 | nq::kFlagScalesPacked;
  return k;
}

struct Schedule {
  int log_t, log_k;
};

// Group-scale layout of the two group calls: checks ld_s and returns the
// kernel's row / group strides (elements of float, or bytes when packed).
nq_status group_scale_strides(const char* fn, uint32_t flags, int64_t M, int64_t groups, int64_t ld_s,
                              int64_t* rs, int64_t* cs) {
  const bool col = (flags & NQ_FLAG_SCALES_COL_MAJOR) != 0;
  const bool packed = (flags & NQ_FLAG_SCALES_PACKED_UE8M0) != 0;
  const int64_t need = col ? M : (packed ? (groups + 3) / 4 : groups);
  if (ld_s < need)
    return fail(NQ_ERR_INVALID_ARGUMENT, "%s: ld_s = %lld < %lld for this scale layout", fn, (long long)ld_s,
                (long long)need);
  const int64_t unit = packed ? 4 : 1;
  *rs = col ? unit : unit * ld_s;
  *cs = col ? unit * ld_s : unit;
  return NQ_OK;
}

// Row -> thread mapping.  C = ceil(d / 8) chunks of 16 bytes, P = the next
// power of two.  Rows of <= 1024 elements: one warp per row (eight rows per
// CTA), 2^max(0, log P - 5) chunks per thread.  Wider rows: one CTA per row;
// the chunks per thread follow rows per SM (measured on B200 for every
// operation at d = 2816 ... 8192, M = 148 ... 65536):
//   M < 148 (fewer rows than SMs): up to 1024 threads, one or two chunks each;
//   M < 192 and P <= 512: one chunk per thread; M < 384: two;
//   P <= 512 (d <= 4096): two for the residual-add dynamic path at any M
//     (more rows in flight per SM beat the longer per-thread chain), and for
//     static RMSNorm, LayerNorm and NVFP4 while M < 768;
//   LayerNorm with P = 1024 and M >= 768: eight;
//   otherwise four (64 bytes of the row per thread, 128 with a residual, in
//   flight at once).
// Every mapping gives identical bits.
nq_status plan_rows(const char* fn, int op, int64_t M, int64_t d, uint32_t flags, Schedule* s, bool raw = false,
                    bool has_res = false) {
  const int64_t C = (d + 7) / 8;
  int lp = 0;
  while ((int64_t(1) << lp) < C) ++lp;
  const uint32_t ft = (flags >> 16) & 0xFu, fk = (flags >> 20) & 0x7u;
  if (ft || fk) {
    if (!ft || !fk) return fail(NQ_ERR_INVALID_ARGUMENT, "%s: NQ_FLAG_SCHEDULE needs both fields", fn);
    const int lt = int(ft) + 4, lk = int(fk) - 1;
    if (!(raw ? nq::raw_schedule_built(lt, lk) : nq::schedule_built(lt, lk)))
      return fail(NQ_ERR_UNSUPPORTED, "%s: schedule of 2^%d threads x 2^%d chunks is not built", fn, lt, lk);
    if ((int64_t(1) << (lt + lk)) < C)
      return fail(NQ_ERR_INVALID_ARGUMENT, "%s: schedule covers %lld chunks, a row has %lld", fn,
                  (long long)(int64_t(1) << (lt + lk)), (long long)C);
    *s = {lt, lk};
    return NQ_OK;
  }
  if (lp <= 7) {
    s->log_t = 5;
    s->log_k = lp > 5 ? lp - 5 : 0;
  } else if (M < 148) {
    // Fewer rows than SMs: latency first.  Up to 512 threads with one chunk
    // each; rows of 4097 ... 8192 elements take 512 threads with two chunks,
    // not 1024 with one (1 x 8192 dynamic: 3.20 -> 2.56 us, 64 x 7168:
    // 3.50 -> 2.64 us; 8-13 % for the NVFP4 and group forms).
    s->log_t = lp < 10 ? lp : (lp == 10 ? 9 : 10);
    s->log_k = lp - s->log_t;
  } else {
    int lk = 2;
    if (M < 192 && lp <= 9) lk = 0;
    else if (M < 384) lk = 1;
    else if (lp <= 9 && ((op == nq::kOpRmsDynFp8 && !(lp == 9 && C < (int64_t(1) << lp))) ||
                         (M < 768 && (op == nq::kOpRmsStaticFp8 || op == nq::kOpLnStaticFp8 || op == nq::kOpRmsNvfp4))))
      lk = 1;
    // (The dynamic path keeps four chunks for rows of 257 ... 511 chunks, d =
    // 2056 ... 4088: their upper slots are skipped whole per warp, 65536 x
    // 2816: 225 -> 197 us.)
    // LayerNorm takes two rows per CTA (run_rows); with P = 1024 it runs
    // best at eight chunks per thread (8192 x 7168: 54.1 -> 49.9 us).
    if (op == nq::kOpLnStaticFp8 && lp == 10 && M >= 768) lk = 3;
    // NVFP4 without residual (raw rows): eight chunks per thread for P = 1024
    // (16384 x 8192: 87.8 -> 85.4 us; 8192 x 7168: 45.3 -> 42.4 us, its dead
    // upper slots then whole slots of every warp) and for rows narrower than
    // P = 512 (65536 x 2816: 142.5 -> 130.2 us); at d = 4096 four stay faster.
    if (op == nq::kOpRmsNvfp4 && !has_res && M >= 768 && (lp == 10 || (lp == 9 && C < (int64_t(1) << lp)))) lk = 3;
    // Rows of 8193 ... 16384 elements without residual: eight chunks per
    // thread (256 threads) on rows narrower than P = 2048 (16384 x 10240:
    // static RMSNorm 120.7 -> 94.3 us, NVFP4 164.1 -> 130.3, group 177.3 ->
    // 152.8, LayerNorm 180.3 -> 143.6), and on full rows for static RMSNorm
    // (16384 x 16384: 150.2 -> 133.4 us) and, from 4096 rows, NVFP4 (185.5 ->
    // 172.7 us) and the fused group (217.5 -> 208.6 us); LayerNorm keeps four
    // on full rows.
    if (!has_res && lp == 11 && M >= 768 &&
        (C < 2048 ? op != nq::kOpRmsDynFp8
                  : (op == nq::kOpRmsStaticFp8 ||
                     ((op == nq::kOpRmsNvfp4 || op == nq::kOpRmsGroupFp8) && M >= 4096))))
      lk = 3;
    int lt = lp - lk;
    if (lt > 10) lt = 10;
    s->log_t = lt;
    s->log_k = lp - lt;
  }
  if (!nq::schedule_built(s->log_t, s->log_k))
    return fail(NQ_ERR_UNSUPPORTED, "%s: no built schedule for d = %lld", fn, (long long)d);
  return NQ_OK;
}

nq_status launch(const char* fn, const void* kernel, unsigned grid, unsigned block, size_t smem,
                 void** args, bool pdl, cudaStream_t stream) {
  if (kernel == nullptr) return fail(NQ_ERR_UNSUPPORTED, "%s: kernel variant not built", fn);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(block, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (pdl) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  const cudaError_t e = cudaLaunchKernelExC(&cfg, kernel, args);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();  // launch errors are not sticky: clear so later callers do not see them
    return fail(NQ_ERR_CUDA, "%s: launch failed: %s", fn, cudaGetErrorString(e));
  }
  return NQ_OK;
}

nq_status check_common(const char* fn, int64_t M, int64_t d, float eps) {
  if (M < 0) return fail(NQ_ERR_INVALID_ARGUMENT, "%s: M = %lld < 0", fn, (long long)M);
  if (d < 1) return fail(NQ_ERR_INVALID_ARGUMENT, "%s: d = %lld < 1", fn, (long long)d);
  if (d > NQ_MAX_D) return fail(NQ_ERR_UNSUPPORTED, "%s: d = %lld > NQ_MAX_D (%d)", fn, (long long)d, NQ_MAX_D);
  if (!(eps >= 0.0f) || !std::isfinite(eps))
    return fail(NQ_ERR_INVALID_ARGUMENT, "%s: eps must be finite and >= 0", fn);
  if (M > int64_t(0x7fffffff)) return fail(NQ_ERR_UNSUPPORTED, "%s: M = %lld too large", fn, (long long)M);
  return NQ_OK;
}

#define NQ_REQUIRE(cond, ...)                                   \
  do {                                                          \
    if (!(cond)) return fail(NQ_ERR_INVALID_ARGUMENT, __VA_ARGS__); \
  } while (0)

// Kernel table of an operation and output form (alt: e5m2 codes for the FP8
// operations, swizzled block scales for NVFP4; layout: column-major or packed
// group scales).
const nq::RowKernels& table_of(int op, bool alt, bool layout, bool scatter) {
  if (scatter) return op == nq::kOpRmsDynFp8 ? nq::row_kernels_rms_dyn_scatter() : nq::row_kernels_rms_group_scatter();
  switch (op) {
    case nq::kOpRmsDynFp8: return alt ? nq::row_kernels_rms_dyn_e5m2() : nq::row_kernels_rms_dyn();
    case nq::kOpRmsStaticFp8: return alt ? nq::row_kernels_rms_static_e5m2() : nq::row_kernels_rms_static();
    case nq::kOpLnStaticFp8: return alt ? nq::row_kernels_ln_static_e5m2() : nq::row_kernels_ln_static();
    case nq::kOpRmsGroupFp8:
      if (layout) return alt ? nq::row_kernels_rms_group_e5m2_layout() : nq::row_kernels_rms_group_layout();
      return alt ? nq::row_kernels_rms_group_e5m2() : nq::row_kernels_rms_group();
    default: return alt ? nq::row_kernels_rms_nvfp4_swizzled() : nq::row_kernels_rms_nvfp4();
  }
}

// The current CUDA device (-1 when there is none or it is out of the caches'
// range).  Kernel attributes, the shared-memory opt-in and occupancy are per
// device, so the caches below are keyed by (device, kernel).
constexpr int kMaxDevices = 64;
int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return -1;
  }
  return dev;
}

// Registers per thread of a kernel (host query, cached per device and kernel).
struct RegsKey {
  int dev;
  const void* k;
  int regs;
};
std::mutex g_regs_mu;
std::vector<RegsKey> g_regs;
int kernel_regs(const void* k) {
  const int dev = current_device();
  if (dev < 0) return -1;
  std::lock_guard<std::mutex> lk(g_regs_mu);
  for (const auto& p : g_regs)
    if (p.dev == dev && p.k == k) return p.regs;
  cudaFuncAttributes attr;
  int regs = -1;
  if (cudaFuncGetAttributes(&attr, k) == cudaSuccess) regs = attr.numRegs;
  else (void)cudaGetLastError();
  g_regs.push_back({dev, k, regs});
  return regs;
}

// Device address of a __device__ symbol on the current device (cached per
// device: each device holds its own copy of the symbol).
std::mutex g_err_mu;
uint32_t* g_err_ptr[kMaxDevices] = {};
uint32_t* g_taken_ptr[kMaxDevices] = {};
uint32_t* symbol_on_device(uint32_t** cache, const void* symbol) {
  const int dev = current_device();
  if (dev < 0) return nullptr;
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (cache[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, symbol) == cudaSuccess) cache[dev] = static_cast<uint32_t*>(p);
    else (void)cudaGetLastError();
  }
  return cache[dev];
}
uint32_t* device_error_word() { return symbol_on_device(g_err_ptr, &g_nq_device_error); }

// Dynamic shared memory above the default 48 KB needs an opt-in per device
// and kernel.
struct SmemKey {
  int dev;
  const void* k;
  size_t bytes;
};
std::mutex g_smem_mu;
std::vector<SmemKey> g_smem;
// Opt kernel k in to `bytes` of dynamic shared memory on the current device.
// Set whenever a kernel takes any: the 48 KB default covers static and
// dynamic memory together, so 48 KB of dynamic memory on top of a kernel's
// static buffers needs it too.
bool allow_smem(const void* k, size_t bytes) {
  if (bytes == 0) return true;
  const int dev = current_device();
  if (dev < 0) return false;
  std::lock_guard<std::mutex> lk(g_smem_mu);
  for (const auto& p : g_smem)
    if (p.dev == dev && p.k == k && p.bytes >= bytes) return true;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes)) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  g_smem.push_back({dev, k, bytes});
  return true;
}

// SM count of each device and resident CTAs per SM of a kernel (host queries,
// cached per device).
struct OccKey {
  int dev;
  const void* k;
  int block;
  size_t smem;
  int occ;
};
std::mutex g_occ_mu;
std::vector<OccKey> g_occ;
int g_sms[kMaxDevices] = {};
int64_t resident_ctas(const void* k, int block, size_t smem = 0) {
  const int dev = current_device();
  if (dev < 0) return 0;
  std::lock_guard<std::mutex> lk(g_occ_mu);
  if (g_sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      (void)cudaGetLastError();
      return 0;
    }
    g_sms[dev] = n;
  }
  for (const auto& p : g_occ)
    if (p.dev == dev && p.k == k && p.block == block && p.smem == smem) return int64_t(g_sms[dev]) * p.occ;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, block, smem) != cudaSuccess) {
    (void)cudaGetLastError();
    occ = 0;
  }
  g_occ.push_back({dev, k, block, smem, occ});
  return int64_t(g_sms[dev]) * occ;
}

// Shared tail of the norm calls.
//
// Kernel variants (same bits): register rows (row_kernel: the row as float32
// in registers; any op, any alignment), raw rows (row_kernel_raw: ops without
// a residual, 16-byte rows, raw bf16 kept and unpacked per pass), raw rows
// persistent (one CTA per resident slot, next row prefetched), and two rows
// per CTA (row_kernel_rows_n: static RMSNorm / LayerNorm).  NQ_FLAG_VARIANT
// forces one where it applies.
// CTAs per row of a row wider than 16384 elements (2048 chunks): 4 up to
// 32768 elements, 8 up to 65536; 0 for rows one CTA holds.
int cluster_ctas(int64_t d) {
  const int64_t C = (d + 7) / 8;
  return C <= 2048 ? 0 : (C <= 4096 ? 4 : 8);
}

// Rows wider than 16384 elements: one row per thread-block cluster of 4 or 8
// CTAs of 256 threads (register rows; the variants do not apply).
nq_status run_cluster_rows(const char* fn, int op, RowArgs& a, bool vec, uint32_t flags, cudaStream_t stream) {
  if (flags & NQ_FLAG_SCHEDULE_MASK)
    return fail(NQ_ERR_INVALID_ARGUMENT, "%s: NQ_FLAG_SCHEDULE covers at most 2048 chunks; d = %lld takes a cluster "
                "per row", fn, (long long)a.d);
  const int nc = cluster_ctas(a.d);
  const int64_t grid = a.M * nc;
  if (grid > int64_t(0x7fffffff)) return fail(NQ_ERR_UNSUPPORTED, "%s: M = %lld too large for rows of d = %lld", fn,
                                              (long long)a.M, (long long)a.d);
  const nq::RowKernels& table = table_of(op, (flags & (NQ_FLAG_E5M2 | NQ_FLAG_SF_SWIZZLED)) != 0,
                                        (flags & (NQ_FLAG_SCALES_COL_MAJOR | NQ_FLAG_SCALES_PACKED_UE8M0)) != 0,
                                        a.dest != nullptr);
  const auto& tab = table.cluster[nc == 8 ? 1 : 0];
  const int64_t span = int64_t(8) * nq::kClusterThreads * nq::kClusterChunks * nc;  // elements a cluster covers
  const void* k = tab[vec ? 1 : 0];
  // As for one CTA per row: the predicate-free copy for rows that fill the
  // cluster, the copy that skips dead chunk slots for narrower rows, each when
  // it needs no more registers.
  const int mode = !vec ? 0 : (a.d == span ? 2 : 3);
  if (mode >= 2 && tab[mode] != nullptr) {
    const int r_m = kernel_regs(tab[mode]), r_vec = kernel_regs(tab[1]);
    if (r_m > 0 && r_vec > 0 && r_m <= r_vec) k = tab[mode];
  }
  a.err = device_error_word();
  if (a.err == nullptr) return fail(NQ_ERR_CUDA, "%s: no CUDA device", fn);
  void* args[] = {&a};
  return launch(fn, k, unsigned(grid), unsigned(nq::kClusterThreads), 0, args, (flags & NQ_FLAG_PDL) != 0, stream);
}

nq_status run_rows(const char* fn, int op, RowArgs& a, bool vec, uint32_t flags, cudaStream_t stream) {
  const bool has_res = a.res_in != nullptr;
  uint32_t variant = (flags & NQ_FLAG_VARIANT_MASK) >> 24;
  if (variant == 4 || variant == 5 || variant == 7)
    return fail(NQ_ERR_UNSUPPORTED, "%s: NQ_FLAG_VARIANT(%u) is not built (variants 1, 2, 3 and 6 are)", fn, variant);
  if (cluster_ctas(a.d) > 0) return run_cluster_rows(fn, op, a, vec, flags, stream);
  if (a.dest != nullptr) variant = 1;  // MoE scatter: register rows only
  const bool raw_forced = variant >= 2 && vec && !has_res && op != nq::kOpRmsDynFp8;
  Schedule s;
  nq_status st = plan_rows(fn, op, a.M, a.d, flags, &s, raw_forced, has_res);
  if (st != NQ_OK) return st;
  const int threads = 1 << s.log_t;
  const int rows = nq::rows_per_cta(threads);
  int64_t grid = (a.M + rows - 1) / rows;
  if (variant == 0 && !has_res) {
    // Automatic choice, from measurements on B200: static RMSNorm gains from
    // raw rows (fewer registers, more CTAs per SM) and, once every resident
    // CTA gets two or more rows, from the persistent prefetching form; NVFP4
    // from raw rows once a row is wider than a warp (10-15 % at d = 1536 ...
    // 3584); LayerNorm from raw rows once a row
    // has 1024 elements or more (up to 1.37x at d = 7168: its float32 row
    // would hold twice the registers); the fused group quantization from raw
    // rows at every width (1.13x - 1.26x).  LayerNorm rows wider than a warp
    // take two rows per CTA (gamma / beta loaded once for both: 1.27x at
    // 65536 x 4096); rows wider than 8192 elements (one CTA per SM, bound by
    // the 8 d bytes of shared memory) from persistent CTAs that prefetch the
    // next row and keep gamma / beta in shared memory (1.2x - 1.3x at d =
    // 10240 ... 16384, M >= 1024), and from raw rows where persistence does
    // not pay (100 x 16384: 7.0 -> 5.4 us); with eight chunks per thread
    // (rows narrower than 16384 elements, M >= 768) two rows per CTA again
    // (16384 x 12288: 178.3 -> 160.8 us).
    if (op == nq::kOpRmsStaticFp8) variant = 3;
    else if (op == nq::kOpRmsNvfp4 && threads > 32) variant = 2;
    else if (op == nq::kOpLnStaticFp8 && a.d > 8192) variant = s.log_k == 3 ? 6 : 3;
    else if (op == nq::kOpLnStaticFp8 && threads > 32) variant = 6;
    else if (op == nq::kOpLnStaticFp8 && a.d >= 1024) variant = 2;
    else if (op == nq::kOpRmsGroupFp8) variant = 2;
  }
  const void* k = nullptr;
  size_t smem = 0;
  const bool scatter = a.dest != nullptr;
  const nq::RowKernels& table = table_of(op, (flags & (NQ_FLAG_E5M2 | NQ_FLAG_SF_SWIZZLED)) != 0,
                                        (flags & (NQ_FLAG_SCALES_COL_MAJOR | NQ_FLAG_SCALES_PACKED_UE8M0)) != 0,
                                        scatter);
  if (vec && !has_res && variant == 6 && threads > 32 && (op == nq::kOpRmsStaticFp8 || op == nq::kOpLnStaticFp8)) {
    // The narrow copy skips chunk slots wholly past rows narrower than the schedule.
    k = table.rows2[s.log_t - nq::kMinLogT][s.log_k][a.d < (8 * int64_t(threads)) << s.log_k ? 1 : 0];
    if (k != nullptr) grid = (a.M + 1) / 2;
  }
  if (vec && !has_res && op != nq::kOpRmsDynFp8 && (variant == 2 || variant == 3)) {
    // The narrow copy tests for chunk slots past the row; a row that fills
    // the schedule (d == 8 * threads * chunks) takes the copy without tests.
    const int narrow = a.d == (8 * int64_t(threads)) << s.log_k ? 0 : 1;
    const auto& raw = table.raw[s.log_t - nq::kMinLogT][s.log_k];
    if (variant == 3 && raw[1][narrow] != nullptr) {
      // Persistent CTAs hold gamma (LayerNorm: gamma and beta) as fp32 in
      // shared memory.
      const size_t gsmem = nq::raw_gamma_smem_bytes(op, a.d);
      if (!allow_smem(raw[1][narrow], gsmem))
        return fail(NQ_ERR_UNSUPPORTED, "%s: %zu bytes of shared memory per CTA not available", fn, gsmem);
      const int64_t slots = resident_ctas(raw[1][narrow], threads * rows, gsmem);
      // Persistent pays once each resident CTA walks two or more rows.
      const bool forced = ((flags & NQ_FLAG_VARIANT_MASK) >> 24) == 3;
      if (slots > 0 && (forced || grid >= 2 * slots)) {
        k = raw[1][narrow];
        smem = gsmem;
        grid = grid < slots ? grid : slots;
      }
    }
    if (k == nullptr) k = raw[0][narrow];
  }
  if (k == nullptr) {
    const auto& tab = table.direct[s.log_t - nq::kMinLogT][s.log_k];
    k = tab[vec ? 1 : 0];
    // 16-byte rows narrower than the schedule skip the chunk slots wholly
    // past the row (mode 3), when that needs no more registers (measured on
    // B200: with fewer registers 3-15 % faster at d = 1536 ... 7168; with
    // more, at two chunks per thread, 4 % slower).
    if (vec && a.d < (8 * int64_t(threads)) << s.log_k && tab[3] != nullptr) {
      const int r_narrow = kernel_regs(tab[3]), r_vec = kernel_regs(tab[1]);
      if (r_narrow > 0 && r_vec > 0 && r_narrow <= r_vec) k = tab[3];
    }
    // The predicate-free variant for rows that exactly fill the schedule, when
    // it does not need more registers (occupancy decides this kernel's speed).
    if (vec && threads > 32 && a.d == (8 * int64_t(threads)) << s.log_k && tab[2] != nullptr) {
      const int r_full = kernel_regs(tab[2]), r_vec = kernel_regs(tab[1]);
      if (r_full > 0 && r_vec > 0 && r_full <= r_vec) k = tab[2];
    }
  }
  a.err = device_error_word();
  if (a.err == nullptr) return fail(NQ_ERR_CUDA, "%s: no CUDA device", fn);
  void* args[] = {&a};
  return launch(fn, k, unsigned(grid), unsigned(threads * rows), smem, args, (flags & NQ_FLAG_PDL) != 0, stream);
}

bool vec_bf16(const void* p, int64_t ld) { return p == nullptr || (aligned(p, 16) && ld % 8 == 0); }

}  // namespace

extern "C" {

int nq_version(void) { return 100; }

const char* nq_status_string(nq_status status) {
  switch (status) {
    case NQ_OK: return "NQ_OK";
    case NQ_ERR_INVALID_ARGUMENT: return "NQ_ERR_INVALID_ARGUMENT";
    case NQ_ERR_UNSUPPORTED: return "NQ_ERR_UNSUPPORTED";
    case NQ_ERR_CUDA: return "NQ_ERR_CUDA";
  }
  return "unknown nq_status";
}

const char* nq_last_error(void) { return g_last_error.c_str(); }

nq_status nq_selftest_division(uint32_t a_bits_begin, uint64_t count, const float* divisors, int32_t n_divisors,
                               unsigned long long* mismatches, nq_stream_t stream) {
  const char* fn = "nq_selftest_division";
  NQ_REQUIRE(count <= (uint64_t(1) << 32) && uint64_t(a_bits_begin) + count <= (uint64_t(1) << 32),
             "%s: the bit range must stay within 32 bits", fn);
  NQ_REQUIRE(n_divisors >= 0 && (n_divisors == 0 || divisors != nullptr) && mismatches != nullptr,
             "%s: divisors and mismatches are required", fn);
  if (count == 0 || n_divisors == 0) return NQ_OK;
  int sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      (void)cudaGetLastError();
      sms = 148;
    }
  }
  const uint64_t blocks = (count + 255) / 256;
  const unsigned grid = unsigned(blocks < uint64_t(sms) * 16 ? blocks : uint64_t(sms) * 16);
  void* args[] = {&a_bits_begin, &count, &divisors, &n_divisors, &mismatches};
  return launch(fn, reinterpret_cast<const void*>(&selftest_division_kernel), grid, 256, 0, args, false,
                static_cast<cudaStream_t>(stream));
}

nq_status nq_check_device_errors(void) {
  const char* fn = "nq_check_device_errors";
  uint32_t* taken = symbol_on_device(g_taken_ptr, &g_nq_device_error_taken);
  if (device_error_word() == nullptr || taken == nullptr) return fail(NQ_ERR_CUDA, "%s: no CUDA device", fn);
  // Every kernel on every stream of this device first (torch's side streams
  // do not synchronize with the legacy stream), then one thread swaps the word
  // for zero, then the legacy-stream copy reads what it took.
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) {
    take_error_word_kernel<<<1, 1, 0, 0>>>();
    e = cudaGetLastError();
  }
  uint32_t word = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&word, taken, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return fail(NQ_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
  }
  if (word == 0) return NQ_OK;
  return fail(NQ_ERR_CUDA, "%s: device error word 0x%x (bit 1: a MoE destination row was out of range; its "
              "store was skipped)", fn, word);
}

nq_status nq_query_schedule(int op, int64_t M, int64_t d, uint32_t flags, int* threads_per_row,
                            int* chunks_per_thread, int* rows_per_cta) {
  const char* fn = "nq_query_schedule";
  NQ_REQUIRE(op >= 0 && op < nq::kNumRowOps, "%s: op %d out of range", fn, op);
  NQ_REQUIRE(threads_per_row && chunks_per_thread && rows_per_cta, "%s: null output pointer", fn);
  nq_status st = check_common(fn, M, d, 1.0f);
  if (st != NQ_OK) return st;
  if (const int nc = cluster_ctas(d)) {
    // One row per cluster of nc CTAs: threads_per_row counts the cluster's threads.
    NQ_REQUIRE(!(flags & NQ_FLAG_SCHEDULE_MASK), "%s: NQ_FLAG_SCHEDULE does not cover d = %lld", fn, (long long)d);
    *threads_per_row = nq::kClusterThreads * nc;
    *chunks_per_thread = nq::kClusterChunks;
    *rows_per_cta = 1;
    return NQ_OK;
  }
  Schedule s;
  st = plan_rows(fn, op, M, d, flags, &s);
  if (st != NQ_OK) return st;
  *threads_per_row = 1 << s.log_t;
  *chunks_per_thread = 1 << s.log_k;
  *rows_per_cta = nq::rows_per_cta(1 << s.log_t);
  return NQ_OK;
}

nq_status nq_fused_add_rmsnorm_quant_fp8(const void* x, int64_t ld_x, const void* residual_in,
                                         void* residual_out, int64_t ld_res, const void* gamma,
                                         void* q_out, int64_t ld_q, float* scale_out,
                                         void* norm_out, int64_t ld_norm, int64_t M, int64_t d,
                                         float eps, uint32_t flags, nq_stream_t stream) {
  const char* fn = "nq_fused_add_rmsnorm_quant_fp8";
  nq_status st = check_common(fn, M, d, eps);
  if (st != NQ_OK) return st;
  if ((st = check_flags(fn, flags, false, true, true)) != NQ_OK) return st;
  NQ_REQUIRE(ld_x >= d && ld_res >= d && ld_q >= d && (!norm_out || ld_norm >= d),
             "%s: every row stride must be >= d", fn);
  if (M == 0) return NQ_OK;
  NQ_REQUIRE(x && residual_in && residual_out && gamma && q_out && scale_out,
             "%s: x, residual_in, residual_out, gamma, q_out and scale_out are required", fn);
  RowArgs a{};
  a.x = static_cast<const uint16_t*>(x);
  a.ld_x = ld_x;
  a.res_in = static_cast<const uint16_t*>(residual_in);
  a.res_out = static_cast<uint16_t*>(residual_out);
  a.ld_res = ld_res;
  a.gamma = gamma;
  a.q = static_cast<uint8_t*>(q_out);
  a.ld_q = ld_q;
  a.scale_out = scale_out;
  a.norm_out = static_cast<uint16_t*>(norm_out);
  a.ld_norm = ld_norm;
  a.M = M;
  a.d = int32_t(d);
  a.eps = eps;
  a.flags = kernel_flags(flags, /*default_div=*/true);
  const bool vec = d % 8 == 0 && vec_bf16(x, ld_x) && vec_bf16(residual_in, ld_res) &&
                   vec_bf16(residual_out, ld_res) && aligned(gamma, 16) && vec_bf16(norm_out, ld_norm) &&
                   aligned(q_out, 8) && ld_q % 8 == 0;
  return run_rows(fn, nq::kOpRmsDynFp8, a, vec, flags, stream);
}

nq_status nq_rmsnorm_quant_fp8_static(const void* x, int64_t ld_x, const void* residual_in,
                                      void* residual_out, int64_t ld_res, const void* gamma,
                                      const float* scale, void* q_out, int64_t ld_q,
                                      void* norm_out, int64_t ld_norm, int64_t M, int64_t d,
                                      float eps, uint32_t flags, nq_stream_t stream) {
  const char* fn = "nq_rmsnorm_quant_fp8_static";
  nq_status st = check_common(fn, M, d, eps);
  if (st != NQ_OK) return st;
  if ((st = check_flags(fn, flags, false, true, true)) != NQ_OK) return st;
  NQ_REQUIRE((residual_in == nullptr) == (residual_out == nullptr),
             "%s: residual_in and residual_out must both be given or both be NULL", fn);
  NQ_REQUIRE(ld_x >= d && ld_q >= d && (!residual_in || ld_res >= d) && (!norm_out || ld_norm >= d),
             "%s: every row stride must be >= d", fn);
  if (M == 0) return NQ_OK;
  NQ_REQUIRE(x && gamma && scale && q_out, "%s: x, gamma, scale and q_out are required", fn);
  RowArgs a{};
  a.x = static_cast<const uint16_t*>(x);
  a.ld_x = ld_x;
  a.res_in = static_cast<const uint16_t*>(residual_in);
  a.res_out = static_cast<uint16_t*>(residual_out);
  a.ld_res = ld_res;
  a.gamma = gamma;
  a.scale = scale;
  a.q = static_cast<uint8_t*>(q_out);
  a.ld_q = ld_q;
  a.norm_out = static_cast<uint16_t*>(norm_out);
  a.ld_norm = ld_norm;
  a.M = M;
  a.d = int32_t(d);
  a.eps = eps;
  a.flags = kernel_flags(flags, /*default_div=*/false);
  const bool vec = d % 8 == 0 && vec_bf16(x, ld_x) && vec_bf16(residual_in, ld_res) &&
                   vec_bf16(residual_out, ld_res) && aligned(gamma, 16) && vec_bf16(norm_out, ld_norm) &&
                   aligned(q_out, 8) && ld_q % 8 == 0;
  return run_rows(fn, nq::kOpRmsStaticFp8, a, vec, flags, stream);
}

nq_status nq_layernorm_quant_fp8(const void* x, int64_t ld_x, const float* gamma,
                                 const float* beta, const float* scale, void* q_out, int64_t ld_q,
                                 int64_t M, int64_t d, float eps, uint32_t flags,
                                 nq_stream_t stream) {
  const char* fn = "nq_layernorm_quant_fp8";
  nq_status st = check_common(fn, M, d, eps);
  if (st != NQ_OK) return st;
  if ((st = check_flags(fn, flags, false, true, true)) != NQ_OK) return st;
  NQ_REQUIRE(ld_x >= d && ld_q >= d, "%s: every row stride must be >= d", fn);
  if (M == 0) return NQ_OK;
  NQ_REQUIRE(x && gamma && beta && scale && q_out, "%s: x, gamma, beta, scale and q_out are required", fn);
  RowArgs a{};
  a.x = static_cast<const uint16_t*>(x);
  a.ld_x = ld_x;
  a.gamma = gamma;
  a.beta = beta;
  a.scale = scale;
  a.q = static_cast<uint8_t*>(q_out);
  a.ld_q = ld_q;
  a.M = M;
  a.d = int32_t(d);
  a.eps = eps;
  a.flags = kernel_flags(flags, /*default_div=*/false);
  const bool vec = d % 8 == 0 && vec_bf16(x, ld_x) && aligned(gamma, 16) && aligned(beta, 16) &&
                   aligned(q_out, 8) && ld_q % 8 == 0;
  return run_rows(fn, nq::kOpLnStaticFp8, a, vec, flags, stream);
}

nq_status nq_rmsnorm_quant_nvfp4(const void* x, int64_t ld_x, const void* residual_in,
                                 void* residual_out, int64_t ld_res, const void* gamma,
                                 const float* global_scale, void* q_out, int64_t ld_q,
                                 void* sf_out, int64_t ld_sf, void* norm_out, int64_t ld_norm,
                                 int64_t M, int64_t d, float eps, uint32_t flags,
                                 nq_stream_t stream) {
  const char* fn = "nq_rmsnorm_quant_nvfp4";
  nq_status st = check_common(fn, M, d, eps);
  if (st != NQ_OK) return st;
  if ((st = check_flags(fn, flags, false, true, true, /*nvfp4=*/true)) != NQ_OK) return st;
  NQ_REQUIRE(d % 16 == 0, "%s: d = %lld is not a multiple of 16", fn, (long long)d);
  NQ_REQUIRE((residual_in == nullptr) == (residual_out == nullptr),
             "%s: residual_in and residual_out must both be given or both be NULL", fn);
  const bool swizzled = (flags & NQ_FLAG_SF_SWIZZLED) != 0;  // ld_sf unused
  NQ_REQUIRE(ld_x >= d && ld_q >= d / 2 && (swizzled || ld_sf >= d / 16) && (!residual_in || ld_res >= d) &&
                 (!norm_out || ld_norm >= d),
             "%s: row strides too small (ld_x >= d, ld_q >= d/2, ld_sf >= d/16)", fn);
  if (M == 0) return NQ_OK;
  NQ_REQUIRE(x && gamma && global_scale && q_out && sf_out,
             "%s: x, gamma, global_scale, q_out and sf_out are required", fn);
  NQ_REQUIRE(!swizzled || aligned(sf_out, 4), "%s: swizzled sf_out must be 4-byte aligned", fn);
  RowArgs a{};
  a.x = static_cast<const uint16_t*>(x);
  a.ld_x = ld_x;
  a.res_in = static_cast<const uint16_t*>(residual_in);
  a.res_out = static_cast<uint16_t*>(residual_out);
  a.ld_res = ld_res;
  a.gamma = gamma;
  a.scale = global_scale;
  a.q = static_cast<uint8_t*>(q_out);
  a.ld_q = ld_q;
  a.sf = static_cast<uint8_t*>(sf_out);
  a.ld_sf = ld_sf;
  a.norm_out = static_cast<uint16_t*>(norm_out);
  a.ld_norm = ld_norm;
  a.M = M;
  a.d = int32_t(d);
  a.eps = eps;
  a.flags = kernel_flags(flags, /*default_div=*/false);
  const bool vec = vec_bf16(x, ld_x) && vec_bf16(residual_in, ld_res) && vec_bf16(residual_out, ld_res) &&
                   aligned(gamma, 16) && vec_bf16(norm_out, ld_norm) && aligned(q_out, 4) && ld_q % 4 == 0;
  return run_rows(fn, nq::kOpRmsNvfp4, a, vec, flags, stream);
}

nq_status nq_rmsnorm_quant_fp8_group(const void* x, int64_t ld_x, const void* residual_in,
                                     void* residual_out, int64_t ld_res, const void* gamma, void* q_out,
                                     int64_t ld_q, float* scales_out, int64_t ld_s, void* norm_out,
                                     int64_t ld_norm, int64_t M, int64_t d, int32_t group, float eps,
                                     uint32_t flags, nq_stream_t stream) {
  const char* fn = "nq_rmsnorm_quant_fp8_group";
  nq_status st = check_common(fn, M, d, eps);
  if (st != NQ_OK) return st;
  if ((st = check_flags(fn, flags, true, true, true)) != NQ_OK) return st;
  if (group != 64 && group != 128) return fail(NQ_ERR_UNSUPPORTED, "%s: group %d not in {64, 128}", fn, group);
  NQ_REQUIRE(d % group == 0, "%s: d = %lld is not a multiple of group %d", fn, (long long)d, group);
  NQ_REQUIRE((residual_in == nullptr) == (residual_out == nullptr),
             "%s: residual_in and residual_out must both be given or both be NULL", fn);
  NQ_REQUIRE(ld_x >= d && ld_q >= d && (!residual_in || ld_res >= d) && (!norm_out || ld_norm >= d),
             "%s: row strides too small", fn);
  int64_t s_rs = 0, s_cs = 0;
  if ((st = group_scale_strides(fn, flags, M, d / group, ld_s, &s_rs, &s_cs)) != NQ_OK) return st;
  if (M == 0) return NQ_OK;
  NQ_REQUIRE(x && gamma && q_out && scales_out, "%s: x, gamma, q_out and scales_out are required", fn);
  RowArgs a{};
  a.x = static_cast<const uint16_t*>(x);
  a.ld_x = ld_x;
  a.res_in = static_cast<const uint16_t*>(residual_in);
  a.res_out = static_cast<uint16_t*>(residual_out);
  a.ld_res = ld_res;
  a.gamma = gamma;
  a.q = static_cast<uint8_t*>(q_out);
  a.ld_q = ld_q;
  a.scale_out = scales_out;
  a.ld_scale = s_rs;
  a.cs_scale = s_cs;
  a.group = group;
  a.norm_out = static_cast<uint16_t*>(norm_out);
  a.ld_norm = ld_norm;
  a.M = M;
  a.d = int32_t(d);
  a.eps = eps;
  a.flags = kernel_flags(flags, /*default_div=*/false);
  const bool vec = d % 8 == 0 && vec_bf16(x, ld_x) && vec_bf16(residual_in, ld_res) &&
                   vec_bf16(residual_out, ld_res) && aligned(gamma, 16) && vec_bf16(norm_out, ld_norm) &&
                   aligned(q_out, 8) && ld_q % 8 == 0;
  return run_rows(fn, nq::kOpRmsGroupFp8, a, vec, flags, stream);
}

nq_status nq_fused_add_rmsnorm_quant_fp8_moe(const void* x, int64_t ld_x, const void* residual_in,
                                             void* residual_out, int64_t ld_res, const void* gamma,
                                             const int32_t* dest, int32_t topk, int64_t rows, void* q_out,
                                             int64_t ld_q, float* scales_out, int64_t ld_s, void* norm_out,
                                             int64_t ld_norm, int64_t M, int64_t d, int32_t group, float eps,
                                             uint32_t flags, nq_stream_t stream) {
  const char* fn = "nq_fused_add_rmsnorm_quant_fp8_moe";
  nq_status st = check_common(fn, M, d, eps);
  if (st != NQ_OK) return st;
  if ((st = check_flags(fn, flags, group != 0, true, true)) != NQ_OK) return st;
  if (flags & (NQ_FLAG_E5M2 | NQ_FLAG_SCALES_COL_MAJOR | NQ_FLAG_SCALES_PACKED_UE8M0 | NQ_FLAG_VARIANT_MASK))
    return fail(NQ_ERR_UNSUPPORTED, "%s: e4m3 codes, row-major scales and the automatic variant only", fn);
  if (group != 0 && group != 64 && group != 128)
    return fail(NQ_ERR_UNSUPPORTED, "%s: group %d not in {0 (per token), 64, 128}", fn, group);
  NQ_REQUIRE(group == 0 || d % group == 0, "%s: d = %lld is not a multiple of group %d", fn, (long long)d, group);
  NQ_REQUIRE(topk >= 1 && topk <= 64, "%s: topk = %d not in 1..64", fn, topk);
  NQ_REQUIRE(rows >= 0 && rows <= int64_t(0x7fffffff), "%s: rows = %lld out of range", fn, (long long)rows);
  NQ_REQUIRE((residual_in == nullptr) == (residual_out == nullptr),
             "%s: residual_in and residual_out must both be given or both be NULL", fn);
  NQ_REQUIRE(ld_x >= d && ld_q >= d && (group == 0 || ld_s >= d / group) && (!residual_in || ld_res >= d) &&
                 (!norm_out || ld_norm >= d),
             "%s: row strides too small", fn);
  if (M == 0) return NQ_OK;
  NQ_REQUIRE(x && gamma && dest && (rows == 0 || (q_out && scales_out)),
             "%s: x, gamma, dest, q_out and scales_out are required", fn);
  RowArgs a{};
  a.x = static_cast<const uint16_t*>(x);
  a.ld_x = ld_x;
  a.res_in = static_cast<const uint16_t*>(residual_in);
  a.res_out = static_cast<uint16_t*>(residual_out);
  a.ld_res = ld_res;
  a.gamma = gamma;
  a.q = static_cast<uint8_t*>(q_out);
  a.ld_q = ld_q;
  a.scale_out = scales_out;
  a.ld_scale = group == 0 ? 1 : ld_s;
  a.cs_scale = 1;
  a.group = group;
  a.norm_out = static_cast<uint16_t*>(norm_out);
  a.ld_norm = ld_norm;
  a.M = M;
  a.d = int32_t(d);
  a.eps = eps;
  a.flags = kernel_flags(flags, /*default_div=*/group == 0);
  a.dest = dest;
  a.topk = topk;
  a.dest_rows = rows;
  const bool vec = d % 8 == 0 && vec_bf16(x, ld_x) && vec_bf16(residual_in, ld_res) &&
                   vec_bf16(residual_out, ld_res) && aligned(gamma, 16) && vec_bf16(norm_out, ld_norm) &&
                   aligned(q_out, 8) && ld_q % 8 == 0;
  return run_rows(fn, group == 0 ? nq::kOpRmsDynFp8 : nq::kOpRmsGroupFp8, a, vec, flags, stream);
}

nq_status nq_per_token_group_quant_fp8(const void* x, int64_t ld_x, void* q_out, int64_t ld_q,
                                       float* scales_out, int64_t ld_s, int64_t M, int64_t K,
                                       int32_t group, uint32_t flags, nq_stream_t stream) {
  const char* fn = "nq_per_token_group_quant_fp8";
  nq_status st = check_flags(fn, flags, true, true, false);
  if (st != NQ_OK) return st;
  if (flags & NQ_FLAG_VARIANT_MASK)
    return fail(NQ_ERR_INVALID_ARGUMENT, "%s: NQ_FLAG_VARIANT applies to the norm calls only", fn);
  NQ_REQUIRE(M >= 0 && K >= 1, "%s: need M >= 0 and K >= 1", fn);
  if (group != 64 && group != 128) return fail(NQ_ERR_UNSUPPORTED, "%s: group %d not in {64, 128}", fn, group);
  NQ_REQUIRE(K % group == 0, "%s: K = %lld is not a multiple of group %d", fn, (long long)K, group);
  NQ_REQUIRE(ld_x >= K && ld_q >= K, "%s: row strides too small", fn);
  int64_t s_rs = 0, s_cs = 0;
  if ((st = group_scale_strides(fn, flags, M, K / group, ld_s, &s_rs, &s_cs)) != NQ_OK) return st;
  if (M == 0) return NQ_OK;
  NQ_REQUIRE(x && q_out && scales_out, "%s: x, q_out and scales_out are required", fn);
  GroupArgs a{};
  a.x = static_cast<const uint16_t*>(x);
  a.ld_x = ld_x;
  a.q = static_cast<uint8_t*>(q_out);
  a.ld_q = ld_q;
  a.s = scales_out;
  a.ld_s = s_rs;
  a.cs_s = s_cs;
  a.groups_per_row = K / group;
  a.G = M * (K / group);
  if (a.G < (int64_t(1) << 31)) {
    int l = 0;
    while ((int64_t(1) << l) < a.groups_per_row) ++l;
    a.row_shift = 32 + l;
    a.row_magic = ((uint64_t(1) << a.row_shift) + uint64_t(a.groups_per_row) - 1) / uint64_t(a.groups_per_row);
  }
  a.flags = kernel_flags(flags, /*default_div=*/false);
  const bool vec = vec_bf16(x, ld_x) && aligned(q_out, 8) && ld_q % 8 == 0;
  // Team of 2^t lanes per group, 2^u groups per thread.  Many groups: teams
  // of four lanes, one group per thread (measured best on B200: each lane pays
  // the group's scale once per 32 elements, a team reads 64 contiguous bytes,
  // 48 registers, 5 CTAs per SM).  Few groups: a lane per chunk for the
  // shortest latency.
  // NQ_FLAG_GROUP_SCHEDULE(t, u) forces it.
  int lt = a.G >= int64_t(148) * 64 ? 2 : (group == 128 ? 4 : 3), lu = 0;
  const uint32_t ft = (flags >> 16) & 0xFu, fk = (flags >> 20) & 0x7u;
  if (ft || fk) {
    if (!ft || !fk) return fail(NQ_ERR_INVALID_ARGUMENT, "%s: NQ_FLAG_SCHEDULE needs both fields", fn);
    lt = int(ft);  // NQ_FLAG_GROUP_SCHEDULE stores t itself
    lu = int(fk) - 1;
    if (lt < 1 || lt > (group == 128 ? 4 : 3) || lu < 0 || lu > 2)
      return fail(NQ_ERR_UNSUPPORTED, "%s: 2^%d lanes per group x 2^%d groups per thread is not built", fn, lt, lu);
  }
  const int tpg = 1 << lt, units = 1 << lu;
  const int slot = nq::kGroupThreads / tpg;
  const int64_t grid = (a.G + int64_t(slot) * units - 1) / (int64_t(slot) * units);
  if (grid > int64_t(0x7fffffff)) return fail(NQ_ERR_UNSUPPORTED, "%s: too many groups", fn);
  const bool layout = (flags & (NQ_FLAG_SCALES_COL_MAJOR | NQ_FLAG_SCALES_PACKED_UE8M0)) != 0;
  const void* k =
      nq::group_kernels()[(flags & NQ_FLAG_E5M2) ? 1 : 0][layout ? 1 : 0][group == 128 ? 1 : 0][lt - 1][lu][vec ? 1 : 0];
  void* args[] = {&a};
  return launch(fn, k, unsigned(grid), nq::kGroupThreads, 0, args, (flags & NQ_FLAG_PDL) != 0, stream);
}

}  // extern "C"
