/*
 * nq.h — C ABI of the fused norm + activation-quantization library (libnq.so)
 * for NVIDIA B200 (sm_100a).
 *
 * One call = one kernel launch that, per token (row of d elements), adds the
 * residual, normalizes (RMSNorm or LayerNorm) in float32 registers and
 * quantizes the float32 result once, to e4m3 (FP8) or to NVFP4 (packed e2m1 +
 * e4m3 block scales).  A fifth call quantizes raw bf16 activations per group
 * of 128 (or 64) elements, and a sixth fuses RMSNorm with that group
 * quantization.
 *
 * Conventions shared by every call
 * --------------------------------
 * Status. Every call returns an nq_status. NQ_OK = 0. On any other value
 *   nothing was launched and nq_last_error() (thread-local) says why. No call
 *   throws across the ABI, traps on the device or allocates memory, and no
 *   call but nq_check_device_errors synchronizes a stream or the device.
 * Memory. Every pointer is caller-owned DEVICE memory on the current CUDA
 *   device (the "scale" arguments too: they are read by the kernel at execution
 *   time, so a captured CUDA graph sees scale updates made between replays).
 *   bf16 tensors are row-major with a row stride ("ld_*") in ELEMENTS of that
 *   tensor; e4m3 / packed-e2m1 / block-scale outputs have row strides in BYTES
 *   (= elements); float32 scale arrays in elements.  The last dimension is
 *   contiguous.  A column slice of a wider tensor is passed as a pointer to its
 *   first column plus the wide tensor's row stride.
 * Aliasing. residual_out may equal residual_in (in-place update, same stride);
 *   no other output may overlap any input or another output.
 * Asynchrony. Work is enqueued on `stream` (NULL = legacy default stream).
 * Alignment. Any alignment is accepted. When every pointer is 16-byte aligned
 *   (8-byte for e4m3 outputs, 4-byte for packed e2m1), every row stride keeps
 *   rows so aligned and d % 8 == 0, the 16-byte vector path runs; otherwise a
 *   scalar path with identical results runs.
 * Sizes. M == 0 returns NQ_OK without a launch. 1 <= d <= NQ_MAX_D for the
 *   norm calls; row strides must be >= d.
 * Numerics (identical on every schedule, reproduced exactly by the oracle):
 *   r = RN(x + residual) in float32; the bf16 residual_out is RN_bf16(r);
 *   row sums use a fixed chunked pairwise order (8 consecutive elements per
 *   chunk; its even- and odd-position elements summed in order from +0 in two
 *   accumulators, then RN(even + odd); then a pairwise tree over chunk index,
 *   highest index bit first);
 *   rstd = RN(1 / RN(sqrt(RN(mean + eps)))) with mean = RN(sum / d);
 *   RMSNorm y = RN(RN(r * rstd) * gamma); LayerNorm y = fma(RN((r - mu) * rstd),
 *   gamma, beta); e4m3 / e5m2 / e2m1 conversion rounds to nearest even and
 *   saturates to +-448 / +-57344 / +-6.
 *
 * Sources (web pages, by title and section):
 *  - "Fusing RMSNorm and FP8 Quantization Under torch.compile" (netraruntime
 *    blog): TL;DR and "Where norm+quant sits" (residual add + RMSNorm +
 *    per-token e4m3, quantized once from float32 registers); FAQ (residual
 *    update exact, bf16 normed output written identically).
 *  - FlashInfer PR #3962 "feat: fused FP8 quantization output for LayerNorm":
 *    Description (layernorm_quant(out, input, gamma, beta, scale, eps); scale
 *    applied as a division; float32 gamma/beta).
 *  - TensorRT-LLM PR #14848 "RMSNorm nvfp4 quant fusion for DS V3.2 /
 *    Kimi-K2.5": Description and commit notes (RMSNorm with or without
 *    residual -> packed E2M1 + per-16 E4M3 block scales; row-strided column
 *    slice input; hidden % 16 == 0; mandatory outputs non-null; residual sum
 *    returned as a separate tensor).
 *  - vLLM PR #61343 "per_token_group_quant_8bit: multiply by reciprocal
 *    instead of dividing per element": Overview and Details (groups of 128,
 *    one reciprocal per group, UE8M0 power-of-two scales).
 *  - FlashInfer PR #2459 "RMSNorm/FusedRMSNorm + Quant kernels cuda graph
 *    fixes": Description and Changes (scale passed as a one-element float32
 *    device tensor, read as scale[0], inverse computed in the kernel).
 */
#ifndef NQ_H_
#define NQ_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* nq_stream_t;

typedef enum nq_status {
  NQ_OK = 0,
  NQ_ERR_INVALID_ARGUMENT = 1, /* null mandatory pointer, bad size/stride/flag */
  NQ_ERR_UNSUPPORTED = 2,      /* valid request outside what is built (d > NQ_MAX_D, group) */
  NQ_ERR_CUDA = 3              /* the CUDA runtime refused the launch */
} nq_status;

/* Widest row the norm calls accept (elements).  Rows of up to 16384 elements
 * take one CTA (or one warp) per row; wider rows one thread-block cluster of 4
 * (up to 32768) or 8 (up to 65536) CTAs of 256 threads per row, with identical
 * numerics. */
#define NQ_MAX_D 65536

/* ---- flags (bitwise OR) ---- */
/* Launch with programmatic dependent launch: the kernel's prologue may
 * overlap the tail of the previous kernel on the stream. */
#define NQ_FLAG_PDL (1u << 0)
/* Quantize by exact per-element division RN(y / s). */
#define NQ_FLAG_SCALE_DIV (1u << 1)
/* Quantize by multiplying with the rounded reciprocal RN(y * RN(1 / s)).
 * At most one of DIV / RECIP; with neither, each call's documented default. */
#define NQ_FLAG_SCALE_RECIP (1u << 2)
/* Group quantization: round every group scale up to a power of two (UE8M0). */
#define NQ_FLAG_UE8M0 (1u << 3)
/* Round y to bf16 before quantizing: reproduces the two-kernel (norm -> bf16
 * -> quant) numerics for A/B comparisons.  Not for production use. */
#define NQ_FLAG_NORM_BF16_ROUND (1u << 4)
/* FP8 outputs in e5m2 (5 exponent bits, 2 mantissa bits, largest finite
 * 57344) instead of e4m3: the dynamic and group scales become
 * RN(absmax / 57344) and the codes saturate to +-57344.  FP8 calls only
 * (FlashInfer PR #3962 Description: the output tensor's FP8 type picks the
 * format). */
#define NQ_FLAG_E5M2 (1u << 5)
/* NVFP4 only: write the block scales in the swizzled layout that block-scaled
 * tensor-core GEMMs read (TensorRT-LLM PR #14848 commit notes: the production
 * quantizer's default).  The [M, d/16] scale matrix is cut into tiles of 128
 * rows x 4 columns, 512 bytes each, stored row tile by row tile and, within a
 * row tile, column tile by column tile; inside a tile, row r and column c are
 * byte 16 * (r % 32) + 4 * (r / 32) + c (NVIDIA PTX ISA / cuBLAS block-scaling
 * layout).  sf_out must hold roundup(M, 128) * roundup(d / 16, 4) bytes and be
 * 4-byte aligned; ld_sf is ignored.  Padding rows and columns are written as
 * zero. */
#define NQ_FLAG_SF_SWIZZLED (1u << 6)
/* Group calls only: GEMM-ready group-scale layouts (for per-token-group FP8
 * GEMMs that read one k-block's scales for many tokens at once).
 * NQ_FLAG_SCALES_COL_MAJOR: float scale (m, g) at scales_out[g * ld_s + m],
 *   ld_s >= M (M-major).
 * NQ_FLAG_SCALES_PACKED_UE8M0 (implies NQ_FLAG_UE8M0): scales_out holds
 *   32-bit words, each the biased exponent bytes (e + 127 of the scale 2^e) of
 *   four consecutive groups of a row, group 4j + b in byte b (little-endian);
 *   bytes past the row's last group are zero.  Word (m, j) at
 *   ((uint32_t*)scales_out)[m * ld_s + j] with ld_s >= ceil(G / 4), or with
 *   NQ_FLAG_SCALES_COL_MAJOR at [j * ld_s + m] with ld_s >= M.
 * ld_s counts floats, or 32-bit words when packed. */
#define NQ_FLAG_SCALES_COL_MAJOR (1u << 7)
#define NQ_FLAG_SCALES_PACKED_UE8M0 (1u << 8)
/* Force a schedule: 2^t threads per row (t = 5..10) and 2^k 16-byte chunks per
 * thread (k = 0..3, t + k <= 11), with 2^(t+k) * 8 >= d.  Every schedule gives
 * bitwise identical results; this exists for tests and tuning.  0 = automatic.
 * Rows wider than 16384 elements always take a cluster of CTAs; a forced
 * schedule is rejected there (NQ_ERR_INVALID_ARGUMENT). */
#define NQ_FLAG_SCHEDULE(t, k) ((((uint32_t)(t) - 4u) & 0xFu) << 16 | (((uint32_t)(k) + 1u) & 0x7u) << 20)
#define NQ_FLAG_SCHEDULE_MASK (0x7Fu << 16)
/* Group quantization's schedule (same bit field): 2^t lanes per group, 2^k
 * groups per thread; see nq_per_token_group_quant_fp8. */
#define NQ_FLAG_GROUP_SCHEDULE(t, k) ((((uint32_t)(t)) & 0xFu) << 16 | (((uint32_t)(k) + 1u) & 0x7u) << 20)
/* Force a kernel variant (tests and tuning; same bits either way): n = 1 keeps
 * the row in float32 registers; n = 2 keeps only the raw bf16 row and unpacks
 * it per pass; n = 3 is n = 2 with persistent CTAs that prefetch the next row
 * and keep gamma (LayerNorm: gamma and beta) as fp32 in shared memory;
 * n = 6 (static RMSNorm and LayerNorm, t >= 6) gives each CTA two rows on the
 * same columns, so each thread loads its gamma / beta once for both.  n = 2, 3
 * and 6 apply to 16-byte-aligned rows without a residual and are ignored
 * otherwise; with n = 2 or 3, NQ_FLAG_SCHEDULE also accepts t = 5, k = 4 (one
 * warp per row, 16 chunks per lane, rows of up to 4096 elements).  n = 4, 5
 * and 7 are not built (NQ_ERR_UNSUPPORTED).  0 = automatic. */
#define NQ_FLAG_VARIANT(n) ((((uint32_t)(n)) & 0x7u) << 24)
#define NQ_FLAG_VARIANT_MASK (0x7u << 24)
/* Library version (major * 10000 + minor * 100 + patch). */
int nq_version(void);
/* Static text of a status code. */
const char* nq_status_string(nq_status status);
/* Synchronous: waits for all work on the current device (every stream), then
 * reads and clears this library's device error word in one atomic step.
 * NQ_OK if no kernel recorded an error since the last check; NQ_ERR_CUDA
 * (message in nq_last_error) if a MoE destination row was out of range (bit 1:
 * that store was skipped, the other rows are written), or if the device
 * reported an error while synchronizing.  Kernels never trap or hang, and no
 * kernel of this library waits on anything. */
nq_status nq_check_device_errors(void);
/* Diagnostic (tests): checks, on the device, the bounded division the dynamic
 * FP8 path uses for RN(y / s) (a correctly rounded reciprocal r = RN(1 / s),
 * then two FMA remainder corrections; Markstein 1990).  For every a whose
 * bits are a_bits_begin .. a_bits_begin + count - 1 (and -a), and every
 * divisor b of divisors[n_divisors] (device memory) in the domain the kernels
 * use it on (b in [2^-60, 2^100], |a / b| <= 2^17), compares the scalar and the
 * packed forms with the correctly rounded quotient and adds to *mismatches (a
 * device unsigned long long) the quotients that break the contract: equal bit
 * for bit when |a / b| >= 2^-24, else the same sign and magnitude < 2^-20 (so
 * the same signed-zero FP8 code).
 * Asynchronous on stream. */
nq_status nq_selftest_division(uint32_t a_bits_begin, uint64_t count, const float* divisors, int32_t n_divisors,
                               unsigned long long* mismatches, nq_stream_t stream);
/* Message of the last failing call on this thread ("" if none). */
const char* nq_last_error(void);

/*
 * Schedule the planner picks for a norm call (op: 0 = fused add+RMSNorm+
 * dynamic FP8, 1 = RMSNorm static FP8, 2 = LayerNorm static FP8, 3 = RMSNorm
 * NVFP4, 4 = RMSNorm group FP8) at (M, d, flags): threads per row, 16-byte
 * chunks per thread and rows per CTA; for ops 1, 3 and 4, the call without a
 * residual.
 * A row of more than 16384 elements is split over a cluster of CTAs:
 * threads_per_row then counts the cluster's threads (1024 or 2048) and
 * chunks_per_thread is 4.
 * Pure host function; launches nothing.
 */
nq_status nq_query_schedule(int op, int64_t M, int64_t d, uint32_t flags, int* threads_per_row,
                            int* chunks_per_thread, int* rows_per_cta);

/*
 * Fused residual-add + RMSNorm + dynamic per-token e4m3.
 * ("Fusing RMSNorm and FP8 Quantization Under torch.compile": TL;DR, "Where
 * norm+quant sits"; per-token scale s = absmax(y) / 448.)
 *   x            bf16 [M, ld_x]   input (first d columns used)          required
 *   residual_in  bf16 [M, ld_res] residual stream                        required
 *   residual_out bf16 [M, ld_res] RN_bf16(x + residual); may == residual_in  required
 *   gamma        bf16 [d]         RMSNorm weight                         required
 *   q_out        e4m3 [M, ld_q]   codes of y / s                         required
 *   scale_out    f32  [M]         s = RN(max|y| / 448) (dequant: y ~ q * s)  required
 *   norm_out     bf16 [M, ld_norm] RN_bf16(y), or NULL to skip
 * Default quantization: exact division (NQ_FLAG_SCALE_DIV); NQ_FLAG_SCALE_RECIP
 * multiplies by RN(1 / s).  A row with s == 0 stores the signed zeros of y.
 */
nq_status nq_fused_add_rmsnorm_quant_fp8(const void* x, int64_t ld_x, const void* residual_in,
                                         void* residual_out, int64_t ld_res, const void* gamma,
                                         void* q_out, int64_t ld_q, float* scale_out,
                                         void* norm_out, int64_t ld_norm, int64_t M, int64_t d,
                                         float eps, uint32_t flags, nq_stream_t stream);

/*
 * RMSNorm (residual-add optional) + e4m3 with a static scale held in device
 * memory ("RMSNorm/FusedRMSNorm + Quant kernels cuda graph fixes": Changes;
 * scale is a dequantization multiplier, q = e4m3(y / scale[0])).
 *   residual_in / residual_out: both NULL (no residual) or both non-NULL.
 *   scale: float32 device pointer, 1 element, read at kernel execution.
 * Default quantization: NQ_FLAG_SCALE_RECIP (y * RN(1 / scale[0])).
 * scale[0] must be positive and finite; 0 follows IEEE (1/0 = inf: nonzero y
 * saturate to +-448, y = 0 gives a NaN code); it is never trapped.
 */
nq_status nq_rmsnorm_quant_fp8_static(const void* x, int64_t ld_x, const void* residual_in,
                                      void* residual_out, int64_t ld_res, const void* gamma,
                                      const float* scale, void* q_out, int64_t ld_q,
                                      void* norm_out, int64_t ld_norm, int64_t M, int64_t d,
                                      float eps, uint32_t flags, nq_stream_t stream);

/*
 * LayerNorm + e4m3 with a static device scale ("feat: fused FP8 quantization
 * output for LayerNorm": Description; out = normed / scale).
 *   x bf16 [M, ld_x]; gamma, beta float32 [d]; scale float32 device [1];
 *   q_out e4m3 [M, ld_q].  mean and biased variance (two-pass) of each row.
 * Default quantization: NQ_FLAG_SCALE_RECIP, as the RMSNorm static call.
 */
nq_status nq_layernorm_quant_fp8(const void* x, int64_t ld_x, const float* gamma,
                                 const float* beta, const float* scale, void* q_out, int64_t ld_q,
                                 int64_t M, int64_t d, float eps, uint32_t flags,
                                 nq_stream_t stream);

/*
 * Residual-add (optional) + RMSNorm + e4m3, stored straight into the permuted
 * input of a mixture-of-experts layer ("Fusing RMSNorm and FP8 Quantization
 * Under torch.compile", "What we'd tell anyone shipping this": the MoE expert
 * path quantizes inside the fused-MoE kernel and needs its own analogous
 * fusion).  Each token is normalized and quantized once, exactly as by
 * nq_fused_add_rmsnorm_quant_fp8 (group == 0: dynamic per-token scale,
 * division by default) or nq_rmsnorm_quant_fp8_group (group 64 or 128:
 * per-token-group scales, reciprocal by default), and its codes and scales
 * are written to each of its destination rows.
 *   dest int32 [M, topk] device memory: the row of (token t, slot j) in the
 *     experts' permuted input (e.g. expert-major, as the MoE alignment step
 *     lays it out); < 0 skips the slot (a dropped token).  A destination
 *     >= rows is skipped and sets bit 1 of the device error word
 *     (nq_check_device_errors).  topk in 1..64.
 *   q_out e4m3 [rows, ld_q]; scales_out float32 [rows] (group == 0) or
 *     [rows, ld_s] row-major (group scales).  Rows no slot targets are not
 *     written.  x, residual_in / residual_out, gamma, norm_out as in
 *     nq_rmsnorm_quant_fp8_group (residual_out and norm_out in token order).
 * e4m3 only, row-major scales, automatic schedule; NQ_FLAG_UE8M0 applies with
 * group scales.
 */
nq_status nq_fused_add_rmsnorm_quant_fp8_moe(const void* x, int64_t ld_x, const void* residual_in,
                                             void* residual_out, int64_t ld_res, const void* gamma,
                                             const int32_t* dest, int32_t topk, int64_t rows, void* q_out,
                                             int64_t ld_q, float* scales_out, int64_t ld_s, void* norm_out,
                                             int64_t ld_norm, int64_t M, int64_t d, int32_t group, float eps,
                                             uint32_t flags, nq_stream_t stream);

/*
 * Per-token-group e4m3 of raw bf16 activations ("per_token_group_quant_8bit:
 * multiply by reciprocal instead of dividing per element": Overview, Details).
 *   x bf16 [M, ld_x] (first K columns); q_out e4m3 [M, ld_q];
 *   scales_out float32 [M, ld_s] row-major, K / group scales per row
 *   (NQ_FLAG_SCALES_COL_MAJOR / NQ_FLAG_SCALES_PACKED_UE8M0: the GEMM-ready
 *   layouts above): s = RN(absmax / 448) (57344 with NQ_FLAG_E5M2), or with
 *   NQ_FLAG_UE8M0 the smallest power of two >= s (a zero group gives 2^-127).
 *   group in {64, 128}; K % group == 0.
 * Default quantization: NQ_FLAG_SCALE_RECIP; a zero fp32 scale stores the
 * signed zeros of x.  NQ_FLAG_GROUP_SCHEDULE(t, k) forces the mapping (tests
 * and tuning; same bits): 2^t lanes per group (t = 1..4 for group 128, 1..3
 * for group 64) and 2^k groups per thread (k = 0..2).
 */
nq_status nq_per_token_group_quant_fp8(const void* x, int64_t ld_x, void* q_out, int64_t ld_q,
                                       float* scales_out, int64_t ld_s, int64_t M, int64_t K,
                                       int32_t group, uint32_t flags, nq_stream_t stream);

/*
 * RMSNorm (residual-add optional) + per-token-group e4m3 of y, for block-FP8
 * GEMMs ("per_token_group_quant_8bit: multiply by reciprocal instead of
 * dividing per element": Details, the fused RMSNorm + group-quant path).
 *   x bf16 [M, ld_x]; residual_in / residual_out both NULL or both given;
 *   gamma bf16 [d]; q_out e4m3 [M, ld_q]; scales_out float32 [M, ld_s],
 *   d / group per row, or a layout of NQ_FLAG_SCALES_*: s = RN(absmax(y over
 *   the group) / 448), or with NQ_FLAG_UE8M0 the smallest power of two >= s;
 *   norm_out bf16 or NULL.
 *   group in {64, 128}; d % group == 0.
 * Default quantization: NQ_FLAG_SCALE_RECIP (y * RN(1 / s)), as the standalone
 * group call; a zero fp32 scale stores the signed zeros of y.
 */
nq_status nq_rmsnorm_quant_fp8_group(const void* x, int64_t ld_x, const void* residual_in,
                                     void* residual_out, int64_t ld_res, const void* gamma, void* q_out,
                                     int64_t ld_q, float* scales_out, int64_t ld_s, void* norm_out,
                                     int64_t ld_norm, int64_t M, int64_t d, int32_t group, float eps,
                                     uint32_t flags, nq_stream_t stream);

/*
 * RMSNorm (residual-add optional) + NVFP4 ("RMSNorm nvfp4 quant fusion for
 * DS V3.2 / Kimi-K2.5": Description, commit notes).
 *   x bf16 [M, ld_x] (may be a column slice of a wider tensor);
 *   residual_in / residual_out: both NULL or both non-NULL;
 *   global_scale float32 device [1]: dequantization multiplier g (x ~ e2m1 *
 *     block_scale * g), read at kernel execution, positive and finite;
 *   q_out uint8 [M, ld_q] packed e2m1, element 2i in the low nibble of byte i
 *     (d / 2 bytes per row);
 *   sf_out uint8 [M, ld_sf] e4m3 block scales, one per 16 elements, row-major
 *     (NQ_FLAG_SF_SWIZZLED: the swizzled 128 x 4-tile layout instead):
 *     sf = e4m3(RN(RN(absmax / 6) / g)); element multiplier RN(1 / RN(sf * g));
 *   norm_out bf16 [M, ld_norm] or NULL.
 *   d % 16 == 0.
 * Default quantization: NQ_FLAG_SCALE_RECIP; NQ_FLAG_SCALE_DIV divides by
 * RN(sf * g).  A block whose scale decodes to 0 stores zero codes.
 */
nq_status nq_rmsnorm_quant_nvfp4(const void* x, int64_t ld_x, const void* residual_in,
                                 void* residual_out, int64_t ld_res, const void* gamma,
                                 const float* global_scale, void* q_out, int64_t ld_q,
                                 void* sf_out, int64_t ld_sf, void* norm_out, int64_t ld_norm,
                                 int64_t M, int64_t d, float eps, uint32_t flags,
                                 nq_stream_t stream);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* NQ_H_ */
