"""Fused residual-add + RMSNorm / LayerNorm + activation quantization for B200.

A thin ctypes binding over ``libnq.so`` (see ``include/nq.h`` for the
contract of every call).  This module only marshals arguments: it checks
tensor dtypes / devices / layouts, allocates outputs with torch when the
caller does not pass them, and forwards raw device pointers, strides and the
current CUDA stream.  Every arithmetic step runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback.  The library is loaded on first
use, and that use raises ImportError when it has not been built
(``python -m fp4_activation_quantization_b200.build``).

Functions carry the C names:
``nq_fused_add_rmsnorm_quant_fp8``, ``nq_rmsnorm_quant_fp8_static``,
``nq_layernorm_quant_fp8``, ``nq_per_token_group_quant_fp8``,
``nq_rmsnorm_quant_nvfp4``, ``nq_rmsnorm_quant_fp8_group``; plus
``nq_query_schedule``.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "NQ_OK", "NQ_ERR_INVALID_ARGUMENT", "NQ_ERR_UNSUPPORTED", "NQ_ERR_CUDA", "NQ_MAX_D",
    "FLAG_PDL", "FLAG_SCALE_DIV", "FLAG_SCALE_RECIP", "FLAG_UE8M0", "FLAG_NORM_BF16_ROUND", "FLAG_E5M2",
    "FLAG_SF_SWIZZLED", "sf_swizzled_size", "FLAG_SCALES_COL_MAJOR", "FLAG_SCALES_PACKED_UE8M0",
    "flag_schedule", "flag_group_schedule", "flag_variant", "NQError", "lib", "library_path", "version",
    "nq_fused_add_rmsnorm_quant_fp8", "nq_rmsnorm_quant_fp8_static", "nq_layernorm_quant_fp8",
    "nq_per_token_group_quant_fp8", "nq_rmsnorm_quant_nvfp4", "nq_query_schedule",
    "OP_RMS_DYN_FP8", "OP_RMS_STATIC_FP8", "OP_LN_STATIC_FP8", "OP_RMS_NVFP4", "OP_RMS_GROUP_FP8",
    "nq_rmsnorm_quant_fp8_group", "nq_check_device_errors", "nq_selftest_division",
    "nq_fused_add_rmsnorm_quant_fp8_moe",
]

NQ_OK, NQ_ERR_INVALID_ARGUMENT, NQ_ERR_UNSUPPORTED, NQ_ERR_CUDA = 0, 1, 2, 3
NQ_MAX_D = 65536
FLAG_PDL = 1 << 0
FLAG_SCALE_DIV = 1 << 1
FLAG_SCALE_RECIP = 1 << 2
FLAG_UE8M0 = 1 << 3
FLAG_NORM_BF16_ROUND = 1 << 4
FLAG_E5M2 = 1 << 5
FLAG_SF_SWIZZLED = 1 << 6
FLAG_SCALES_COL_MAJOR = 1 << 7
FLAG_SCALES_PACKED_UE8M0 = 1 << 8
OP_RMS_DYN_FP8, OP_RMS_STATIC_FP8, OP_LN_STATIC_FP8, OP_RMS_NVFP4, OP_RMS_GROUP_FP8 = 0, 1, 2, 3, 4


def flag_schedule(log2_threads: int, log2_chunks: int) -> int:
    """NQ_FLAG_SCHEDULE(t, k): force 2^t threads per row and 2^k chunks per thread."""
    return (((log2_threads - 4) & 0xF) << 16) | (((log2_chunks + 1) & 0x7) << 20)


def flag_group_schedule(log2_lanes: int, log2_groups: int) -> int:
    """NQ_FLAG_GROUP_SCHEDULE(t, k): 2^t lanes per group, 2^k groups per thread (group quantization)."""
    return ((log2_lanes & 0xF) << 16) | (((log2_groups + 1) & 0x7) << 20)


def flag_variant(n: int) -> int:
    """NQ_FLAG_VARIANT(n): 1 register rows, 2 raw rows, 3 raw rows persistent, 6 two rows per CTA
    (0 = automatic; 4, 5 and 7 are not built)."""
    return (n & 0x7) << 24


_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libnq.so")


def library_path() -> str:
    return _LIB_PATH


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is missing: build it with `python -m fp4_activation_quantization_b200.build` "
            "(nvcc, sm_100a). There is no fallback implementation.")
    L = ctypes.CDLL(_LIB_PATH)
    P, I64, I32, U32, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32, ctypes.c_float
    st = ctypes.c_int
    L.nq_version.argtypes, L.nq_version.restype = [], ctypes.c_int
    L.nq_status_string.argtypes, L.nq_status_string.restype = [st], ctypes.c_char_p
    L.nq_last_error.argtypes, L.nq_last_error.restype = [], ctypes.c_char_p
    L.nq_check_device_errors.argtypes, L.nq_check_device_errors.restype = [], st
    L.nq_selftest_division.argtypes = [U32, ctypes.c_uint64, P, I32, P, P]
    L.nq_selftest_division.restype = st
    L.nq_query_schedule.argtypes = [ctypes.c_int, I64, I64, U32, ctypes.POINTER(ctypes.c_int),
                                    ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
    L.nq_query_schedule.restype = st
    L.nq_fused_add_rmsnorm_quant_fp8.argtypes = [P, I64, P, P, I64, P, P, I64, P, P, I64, I64, I64, F, U32, P]
    L.nq_rmsnorm_quant_fp8_static.argtypes = [P, I64, P, P, I64, P, P, P, I64, P, I64, I64, I64, F, U32, P]
    L.nq_layernorm_quant_fp8.argtypes = [P, I64, P, P, P, P, I64, I64, I64, F, U32, P]
    L.nq_per_token_group_quant_fp8.argtypes = [P, I64, P, I64, P, I64, I64, I64, I32, U32, P]
    L.nq_rmsnorm_quant_fp8_group.argtypes = [P, I64, P, P, I64, P, P, I64, P, I64, P, I64, I64, I64, I32, F, U32, P]
    L.nq_rmsnorm_quant_nvfp4.argtypes = [P, I64, P, P, I64, P, P, P, I64, P, I64, P, I64, I64, I64, F, U32, P]
    L.nq_fused_add_rmsnorm_quant_fp8_moe.argtypes = [P, I64, P, P, I64, P, P, I32, I64, P, I64, P, I64, P, I64,
                                                     I64, I64, I32, F, U32, P]
    for name in ("nq_fused_add_rmsnorm_quant_fp8", "nq_rmsnorm_quant_fp8_static", "nq_layernorm_quant_fp8",
                 "nq_per_token_group_quant_fp8", "nq_rmsnorm_quant_nvfp4", "nq_rmsnorm_quant_fp8_group",
                 "nq_fused_add_rmsnorm_quant_fp8_moe"):
        getattr(L, name).restype = st
    return L


_lib = None


def _get_lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


def __getattr__(name):  # module attribute `lib`, loaded on first access
    if name == "lib":
        return _get_lib()
    raise AttributeError(name)


def version() -> int:
    return _get_lib().nq_version()


def nq_selftest_division(divisors, a_bits_begin: int = 0, count: int = 1 << 32, stream=None) -> int:
    """Mismatches of the dynamic path's bounded division against the correctly
    rounded quotient, over a bit range of dividends and float32 CUDA `divisors`."""
    _need(isinstance(divisors, torch.Tensor) and divisors.is_cuda and divisors.dtype == torch.float32
          and divisors.dim() == 1 and divisors.is_contiguous(), "divisors must be a contiguous float32 CUDA vector")
    out = torch.zeros(1, dtype=torch.int64, device=divisors.device)
    with torch.cuda.device(divisors.device):
        _check(_get_lib().nq_selftest_division(a_bits_begin, count, _ptr(divisors), divisors.numel(), _ptr(out),
                                               _stream(stream)), "nq_selftest_division")
    return int(out.item())


def nq_check_device_errors() -> None:
    """Raise NQError if a kernel recorded an error since the last check (a MoE
    destination row out of range).  Synchronous: waits for every stream of the
    current device, then reads and clears the device error word atomically."""
    _check(_get_lib().nq_check_device_errors(), "nq_check_device_errors")


class NQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        L = _get_lib()
        msg = L.nq_last_error().decode()
        super().__init__(f"{where}: {L.nq_status_string(status).decode()}: {msg}")


def _check(status: int, where: str) -> None:
    if status != NQ_OK:
        raise NQError(status, where)


# ----------------------------------------------------------- marshalling ----
def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(cond: bool, msg: str) -> None:
    if not cond:
        raise ValueError(msg)


def _rows(t: torch.Tensor, name: str, dtype, cols: int | None = None):
    """2-D tensor on CUDA with a contiguous last dimension; returns (M, ncols, row stride)."""
    _need(isinstance(t, torch.Tensor), f"{name} must be a torch.Tensor")
    _need(t.is_cuda, f"{name} must be a CUDA tensor")
    _need(t.dtype == dtype, f"{name} must be {dtype}, got {t.dtype}")
    _need(t.dim() == 2, f"{name} must be 2-D [M, d], got shape {tuple(t.shape)}")
    _need(t.stride(1) == 1 or t.shape[1] <= 1, f"{name} must have a contiguous last dimension")
    if cols is not None:
        _need(t.shape[1] == cols, f"{name} must have {cols} columns, got {t.shape[1]}")
    ld = t.stride(0) if t.shape[0] > 1 else max(t.stride(0), t.shape[1])
    return t.shape[0], t.shape[1], ld


def _vec(t: torch.Tensor, name: str, dtype, n: int):
    _need(isinstance(t, torch.Tensor) and t.is_cuda, f"{name} must be a CUDA tensor")
    _need(t.dtype == dtype, f"{name} must be {dtype}, got {t.dtype}")
    _need(t.dim() == 1 and t.shape[0] == n and t.stride(0) == 1, f"{name} must be contiguous [{n}]")


def _scalar(t: torch.Tensor, name: str):
    _need(isinstance(t, torch.Tensor) and t.is_cuda, f"{name} must be a one-element float32 CUDA tensor")
    _need(t.dtype == torch.float32 and t.numel() == 1, f"{name} must be a one-element float32 CUDA tensor")


def _same_device(*ts):
    devs = {t.device for t in ts if t is not None}
    _need(len(devs) == 1, f"all tensors must be on one device, got {devs}")


def _out(t, shape, dtype, like: torch.Tensor, name: str):
    if t is None:
        return torch.empty(shape, dtype=dtype, device=like.device)
    _need(t.dtype == dtype and tuple(t.shape) == tuple(shape), f"{name} must be {dtype} {tuple(shape)}")
    return t


def _fp8_format(flags: int, q_out):
    """(flags, dtype) of an FP8 call's codes: a float8_e5m2 ``q_out`` selects
    e5m2 (FLAG_E5M2); otherwise the flag picks the dtype of a new ``q_out``."""
    if q_out is not None and isinstance(q_out, torch.Tensor) and q_out.dtype == torch.float8_e5m2:
        flags |= FLAG_E5M2
    return flags, (torch.float8_e5m2 if flags & FLAG_E5M2 else torch.float8_e4m3fn)


def _group_scales(scales_out, M: int, G: int, flags: int, like: torch.Tensor):
    """Group-scale output for the layout the flags select; returns (tensor, ld).

    Row-major: float32 [M, G].  FLAG_SCALES_COL_MAJOR: a [M, G] view with
    strides (1, ld) of a [G, ld] buffer.  FLAG_SCALES_PACKED_UE8M0: int32
    words, [M, ceil(G/4)] (row-major) or its column-major view likewise.
    """
    packed = bool(flags & FLAG_SCALES_PACKED_UE8M0)
    col = bool(flags & FLAG_SCALES_COL_MAJOR)
    n = (G + 3) // 4 if packed else G
    dtype = torch.int32 if packed else torch.float32
    if scales_out is None:
        buf = torch.empty((n, M) if col else (M, n), dtype=dtype, device=like.device)
        return (buf.t() if col else buf), (M if col else n)
    _need(isinstance(scales_out, torch.Tensor) and scales_out.is_cuda, "scales_out must be a CUDA tensor")
    _need(scales_out.dtype == dtype and tuple(scales_out.shape) == (M, n),
          f"scales_out must be {dtype} {(M, n)} for this layout")
    if col:
        _need(scales_out.stride(0) == 1 or M <= 1, "column-major scales_out needs stride(0) == 1")
        return scales_out, (scales_out.stride(1) if n > 1 else max(scales_out.stride(1), M))
    _need(scales_out.stride(1) == 1 or n <= 1, "scales_out must have a contiguous last dimension")
    return scales_out, (scales_out.stride(0) if M > 1 else max(scales_out.stride(0), n))


# ------------------------------------------------------------ the calls ----
def nq_query_schedule(op: int, M: int, d: int, flags: int = 0):
    """(threads per row, 16-byte chunks per thread, rows per CTA) the planner picks."""
    t, k, r = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(_get_lib().nq_query_schedule(op, M, d, flags, ctypes.byref(t), ctypes.byref(k), ctypes.byref(r)),
           "nq_query_schedule")
    return t.value, k.value, r.value


def nq_fused_add_rmsnorm_quant_fp8(x, residual, gamma, eps: float = 1e-6, *, residual_out=None,
                                   q_out=None, scale_out=None, norm_out=None, want_norm: bool = False,
                                   flags: int = 0, stream=None):
    """Residual-add + RMSNorm + dynamic per-token e4m3.

    ``x`` bf16 [M, d] (may be a column slice), ``residual`` bf16 [M, d],
    ``gamma`` bf16 [d].  ``residual_out`` defaults to a new tensor; pass
    ``residual_out=residual`` for the in-place update.  Returns
    ``(q float8_e4m3fn [M, d], scale float32 [M], residual_out, norm_out or None)``;
    with ``flags |= FLAG_E5M2`` or a float8_e5m2 ``q_out`` the codes are e5m2
    and s = absmax / 57344 (this holds for every FP8 call).
    """
    M, d, ld_x = _rows(x, "x", torch.bfloat16)
    _, _, ld_r = _rows(residual, "residual", torch.bfloat16, d)
    _need(residual.shape[0] == M, "residual must have M rows")
    _vec(gamma, "gamma", torch.bfloat16, d)
    residual_out = _out(residual_out, (M, d), torch.bfloat16, x, "residual_out")
    _, _, ld_ro = _rows(residual_out, "residual_out", torch.bfloat16, d)
    _need(ld_ro == ld_r, "residual_out must have the row stride of residual")
    flags, f8 = _fp8_format(flags, q_out)
    q_out = _out(q_out, (M, d), f8, x, "q_out")
    _, _, ld_q = _rows(q_out, "q_out", f8, d)
    scale_out = _out(scale_out, (M,), torch.float32, x, "scale_out")
    _vec(scale_out, "scale_out", torch.float32, M)
    if want_norm and norm_out is None:
        norm_out = torch.empty((M, d), dtype=torch.bfloat16, device=x.device)
    ld_n = _rows(norm_out, "norm_out", torch.bfloat16, d)[2] if norm_out is not None else d
    _same_device(x, residual, gamma, residual_out, q_out, scale_out, norm_out)
    with torch.cuda.device(x.device):
        _check(_get_lib().nq_fused_add_rmsnorm_quant_fp8(
            _ptr(x), ld_x, _ptr(residual), _ptr(residual_out), ld_r, _ptr(gamma), _ptr(q_out), ld_q,
            _ptr(scale_out), _ptr(norm_out), ld_n, M, d, eps, flags, _stream(stream)),
            "nq_fused_add_rmsnorm_quant_fp8")
    return q_out, scale_out, residual_out, norm_out


def nq_rmsnorm_quant_fp8_static(x, gamma, scale, eps: float = 1e-6, *, residual=None, residual_out=None,
                                q_out=None, norm_out=None, want_norm: bool = False, flags: int = 0,
                                stream=None):
    """RMSNorm (optional residual-add) + e4m3 with a one-element device scale.

    Returns ``(q float8_e4m3fn [M, d], residual_out or None, norm_out or None)``.
    """
    M, d, ld_x = _rows(x, "x", torch.bfloat16)
    _vec(gamma, "gamma", torch.bfloat16, d)
    _scalar(scale, "scale")
    ld_r = d
    if residual is not None:
        _, _, ld_r = _rows(residual, "residual", torch.bfloat16, d)
        _need(residual.shape[0] == M, "residual must have M rows")
        residual_out = _out(residual_out, (M, d), torch.bfloat16, x, "residual_out")
        _need(_rows(residual_out, "residual_out", torch.bfloat16, d)[2] == ld_r,
              "residual_out must have the row stride of residual")
    else:
        _need(residual_out is None, "residual_out needs residual")
    flags, f8 = _fp8_format(flags, q_out)
    q_out = _out(q_out, (M, d), f8, x, "q_out")
    _, _, ld_q = _rows(q_out, "q_out", f8, d)
    if want_norm and norm_out is None:
        norm_out = torch.empty((M, d), dtype=torch.bfloat16, device=x.device)
    ld_n = _rows(norm_out, "norm_out", torch.bfloat16, d)[2] if norm_out is not None else d
    _same_device(x, gamma, scale, residual, residual_out, q_out, norm_out)
    with torch.cuda.device(x.device):
        _check(_get_lib().nq_rmsnorm_quant_fp8_static(
            _ptr(x), ld_x, _ptr(residual), _ptr(residual_out), ld_r, _ptr(gamma), _ptr(scale), _ptr(q_out),
            ld_q, _ptr(norm_out), ld_n, M, d, eps, flags, _stream(stream)), "nq_rmsnorm_quant_fp8_static")
    return q_out, residual_out, norm_out


def nq_layernorm_quant_fp8(x, gamma, beta, scale, eps: float = 1e-5, *, q_out=None, flags: int = 0,
                           stream=None):
    """LayerNorm (float32 gamma, beta) + e4m3 with a one-element device scale. Returns q."""
    M, d, ld_x = _rows(x, "x", torch.bfloat16)
    _vec(gamma, "gamma", torch.float32, d)
    _vec(beta, "beta", torch.float32, d)
    _scalar(scale, "scale")
    flags, f8 = _fp8_format(flags, q_out)
    q_out = _out(q_out, (M, d), f8, x, "q_out")
    _, _, ld_q = _rows(q_out, "q_out", f8, d)
    _same_device(x, gamma, beta, scale, q_out)
    with torch.cuda.device(x.device):
        _check(_get_lib().nq_layernorm_quant_fp8(_ptr(x), ld_x, _ptr(gamma), _ptr(beta), _ptr(scale), _ptr(q_out),
                                          ld_q, M, d, eps, flags, _stream(stream)), "nq_layernorm_quant_fp8")
    return q_out


def nq_per_token_group_quant_fp8(x, group: int = 128, *, q_out=None, scales_out=None, flags: int = 0,
                                 stream=None):
    """Per-token-group e4m3. Returns ``(q float8_e4m3fn [M, K], scales float32 [M, K/group])``;
    the scales follow the layout FLAG_SCALES_COL_MAJOR / FLAG_SCALES_PACKED_UE8M0 select."""
    M, K, ld_x = _rows(x, "x", torch.bfloat16)
    _need(group > 0 and K % group == 0, f"K = {K} must be a multiple of group = {group}")
    flags, f8 = _fp8_format(flags, q_out)
    q_out = _out(q_out, (M, K), f8, x, "q_out")
    _, _, ld_q = _rows(q_out, "q_out", f8, K)
    scales_out, ld_s = _group_scales(scales_out, M, K // group, flags, x)
    _same_device(x, q_out, scales_out)
    with torch.cuda.device(x.device):
        _check(_get_lib().nq_per_token_group_quant_fp8(_ptr(x), ld_x, _ptr(q_out), ld_q, _ptr(scales_out), ld_s, M, K,
                                                group, flags, _stream(stream)), "nq_per_token_group_quant_fp8")
    return q_out, scales_out


def nq_rmsnorm_quant_fp8_group(x, gamma, eps: float = 1e-6, *, group: int = 128, residual=None,
                               residual_out=None, q_out=None, scales_out=None, norm_out=None,
                               want_norm: bool = False, flags: int = 0, stream=None):
    """RMSNorm (optional residual-add) + per-token-group e4m3 of y.

    Returns ``(q float8_e4m3fn [M, d], scales float32 [M, d/group], residual_out
    or None, norm_out or None)``.
    """
    M, d, ld_x = _rows(x, "x", torch.bfloat16)
    _need(group > 0 and d % group == 0, f"d = {d} must be a multiple of group = {group}")
    _vec(gamma, "gamma", torch.bfloat16, d)
    ld_r = d
    if residual is not None:
        _, _, ld_r = _rows(residual, "residual", torch.bfloat16, d)
        _need(residual.shape[0] == M, "residual must have M rows")
        residual_out = _out(residual_out, (M, d), torch.bfloat16, x, "residual_out")
        _need(_rows(residual_out, "residual_out", torch.bfloat16, d)[2] == ld_r,
              "residual_out must have the row stride of residual")
    else:
        _need(residual_out is None, "residual_out needs residual")
    flags, f8 = _fp8_format(flags, q_out)
    q_out = _out(q_out, (M, d), f8, x, "q_out")
    _, _, ld_q = _rows(q_out, "q_out", f8, d)
    scales_out, ld_s = _group_scales(scales_out, M, d // group, flags, x)
    if want_norm and norm_out is None:
        norm_out = torch.empty((M, d), dtype=torch.bfloat16, device=x.device)
    ld_n = _rows(norm_out, "norm_out", torch.bfloat16, d)[2] if norm_out is not None else d
    _same_device(x, gamma, residual, residual_out, q_out, scales_out, norm_out)
    with torch.cuda.device(x.device):
        _check(_get_lib().nq_rmsnorm_quant_fp8_group(
            _ptr(x), ld_x, _ptr(residual), _ptr(residual_out), ld_r, _ptr(gamma), _ptr(q_out), ld_q,
            _ptr(scales_out), ld_s, _ptr(norm_out), ld_n, M, d, group, eps, flags, _stream(stream)),
            "nq_rmsnorm_quant_fp8_group")
    return q_out, scales_out, residual_out, norm_out


def sf_swizzled_size(M: int, d: int) -> int:
    """Bytes of the swizzled block-scale buffer of an [M, d] NVFP4 output."""
    return ((M + 127) // 128 * 128) * ((d // 16 + 3) // 4 * 4)


def nq_rmsnorm_quant_nvfp4(x, gamma, global_scale, eps: float = 1e-6, *, residual=None, residual_out=None,
                           q_out=None, sf_out=None, norm_out=None, want_norm: bool = False, flags: int = 0,
                           stream=None):
    """RMSNorm (optional residual-add) + NVFP4.

    Returns ``(q uint8 [M, d/2] packed e2m1, sf float8_e4m3fn [M, d/16],
    residual_out or None, norm_out or None)``.  With ``flags |=
    FLAG_SF_SWIZZLED`` sf is the flat float8_e4m3fn buffer of
    ``sf_swizzled_size(M, d)`` bytes in the swizzled 128 x 4-tile layout.
    """
    M, d, ld_x = _rows(x, "x", torch.bfloat16)
    _need(d % 16 == 0, f"d = {d} must be a multiple of 16")
    _vec(gamma, "gamma", torch.bfloat16, d)
    _scalar(global_scale, "global_scale")
    ld_r = d
    if residual is not None:
        _, _, ld_r = _rows(residual, "residual", torch.bfloat16, d)
        _need(residual.shape[0] == M, "residual must have M rows")
        residual_out = _out(residual_out, (M, d), torch.bfloat16, x, "residual_out")
        _need(_rows(residual_out, "residual_out", torch.bfloat16, d)[2] == ld_r,
              "residual_out must have the row stride of residual")
    else:
        _need(residual_out is None, "residual_out needs residual")
    q_out = _out(q_out, (M, d // 2), torch.uint8, x, "q_out")
    _, _, ld_q = _rows(q_out, "q_out", torch.uint8, d // 2)
    if flags & FLAG_SF_SWIZZLED:
        sf_out = _out(sf_out, (sf_swizzled_size(M, d),), torch.float8_e4m3fn, x, "sf_out")
        _need(sf_out.is_cuda and sf_out.is_contiguous(), "sf_out must be a contiguous CUDA tensor")
        ld_sf = 0
    else:
        sf_out = _out(sf_out, (M, d // 16), torch.float8_e4m3fn, x, "sf_out")
        _, _, ld_sf = _rows(sf_out, "sf_out", torch.float8_e4m3fn, d // 16)
    if want_norm and norm_out is None:
        norm_out = torch.empty((M, d), dtype=torch.bfloat16, device=x.device)
    ld_n = _rows(norm_out, "norm_out", torch.bfloat16, d)[2] if norm_out is not None else d
    _same_device(x, gamma, global_scale, residual, residual_out, q_out, sf_out, norm_out)
    with torch.cuda.device(x.device):
        _check(_get_lib().nq_rmsnorm_quant_nvfp4(
            _ptr(x), ld_x, _ptr(residual), _ptr(residual_out), ld_r, _ptr(gamma), _ptr(global_scale), _ptr(q_out),
            ld_q, _ptr(sf_out), ld_sf, _ptr(norm_out), ld_n, M, d, eps, flags, _stream(stream)),
            "nq_rmsnorm_quant_nvfp4")
    return q_out, sf_out, residual_out, norm_out


def nq_fused_add_rmsnorm_quant_fp8_moe(x, gamma, dest, rows: int, eps: float = 1e-6, *, group: int = 0,
                                       residual=None, residual_out=None, q_out=None, scales_out=None,
                                       norm_out=None, want_norm: bool = False, flags: int = 0, stream=None):
    """Residual-add (optional) + RMSNorm + e4m3 stored into a MoE layer's permuted input.

    ``dest`` int32 [M, topk] (CUDA): the permuted row of each (token, slot), < 0
    skips.  ``group`` 0 gives one dynamic scale per token, 64 / 128 per-token-
    group scales.  Returns ``(q float8_e4m3fn [rows, d], scales float32 [rows]
    or [rows, d/group], residual_out or None, norm_out or None)``.
    """
    M, d, ld_x = _rows(x, "x", torch.bfloat16)
    _vec(gamma, "gamma", torch.bfloat16, d)
    _need(isinstance(dest, torch.Tensor) and dest.is_cuda and dest.dtype == torch.int32 and dest.dim() == 2
          and dest.shape[0] == M and dest.is_contiguous(), "dest must be a contiguous int32 CUDA tensor [M, topk]")
    topk = dest.shape[1]
    _need(group in (0, 64, 128) and (group == 0 or d % group == 0), f"group must be 0, 64 or 128 dividing d = {d}")
    ld_r = d
    if residual is not None:
        _, _, ld_r = _rows(residual, "residual", torch.bfloat16, d)
        _need(residual.shape[0] == M, "residual must have M rows")
        residual_out = _out(residual_out, (M, d), torch.bfloat16, x, "residual_out")
        _need(_rows(residual_out, "residual_out", torch.bfloat16, d)[2] == ld_r,
              "residual_out must have the row stride of residual")
    else:
        _need(residual_out is None, "residual_out needs residual")
    q_out = _out(q_out, (rows, d), torch.float8_e4m3fn, x, "q_out")
    ld_q = q_out.stride(0) if rows > 1 else d
    _need(q_out.stride(-1) == 1 or d <= 1, "q_out must have a contiguous last dimension")
    if group == 0:
        scales_out = _out(scales_out, (rows,), torch.float32, x, "scales_out")
        ld_s = 1
    else:
        scales_out = _out(scales_out, (rows, d // group), torch.float32, x, "scales_out")
        ld_s = scales_out.stride(0) if rows > 1 else d // group
    if want_norm and norm_out is None:
        norm_out = torch.empty((M, d), dtype=torch.bfloat16, device=x.device)
    ld_n = _rows(norm_out, "norm_out", torch.bfloat16, d)[2] if norm_out is not None else d
    _same_device(x, gamma, dest, residual, residual_out, q_out, scales_out, norm_out)
    with torch.cuda.device(x.device):
        _check(_get_lib().nq_fused_add_rmsnorm_quant_fp8_moe(
            _ptr(x), ld_x, _ptr(residual), _ptr(residual_out), ld_r, _ptr(gamma), _ptr(dest), topk, rows,
            _ptr(q_out), ld_q, _ptr(scales_out), ld_s, _ptr(norm_out), ld_n, M, d, group, eps, flags,
            _stream(stream)), "nq_fused_add_rmsnorm_quant_fp8_moe")
    return q_out, scales_out, residual_out, norm_out
