"""Python access to the CPU oracle (``oracle/nq_oracle.cpp``) through ctypes.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference arm of ``bench.py`` may import this package.  The product
path (``fp4_activation_quantization_b200``) never imports it and has no CPU
fallback.

Arrays: bf16 tensors are numpy ``uint16`` bit patterns; e4m3 codes, packed
e2m1 bytes and e4m3 block scales are ``uint8``; everything else is
``float32``.  Row strides are in elements of the array's own type.  Each
function documents the page passage it restates in ``nq_oracle.cpp``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nq_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_CXXFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c++17"]

# The oracle's own flag values (see nq_oracle.cpp).
DIV = 1
RECIP = 2
UE8M0 = 4
NORM_BF16_ROUND = 8
SUM_PLAIN = 16
E5M2 = 32

E4M3_MAX = 448.0
E2M1_MAX = 6.0

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to its source when missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", *_CXXFLAGS, "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P, I64, F, U32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_uint32
            sig = {
                "oracle_version": ([], ctypes.c_int),
                "oracle_bf16_from_f32": ([P, P, I64], None),
                "oracle_e4m3_encode": ([P, P, I64], None),
                "oracle_e4m3_decode": ([P, P, I64], None),
                "oracle_e5m2_encode": ([P, P, I64], None),
                "oracle_e5m2_decode": ([P, P, I64], None),
                "oracle_sf_swizzled_size": ([I64, I64], I64),
                "oracle_sf_swizzle": ([P, I64, I64, I64, P], None),
                "oracle_group_scales_layout": ([P, I64, I64, ctypes.c_int, ctypes.c_int, I64, P], ctypes.c_int),
                "oracle_e2m1_encode": ([P, P, I64], None),
                "oracle_e2m1_decode": ([P, P, I64], None),
                "oracle_ue8m0_ceil": ([P, P, I64], None),
                "oracle_canonical_sum": ([P, I64, ctypes.c_int], F),
                "oracle_rms_y": ([P, I64, P, I64, P, P, I64, I64, I64, F, U32], None),
                "oracle_ln_y": ([P, I64, P, P, P, I64, I64, I64, F, U32], None),
                "oracle_fused_add_rmsnorm_quant_fp8":
                    ([P, I64, P, P, I64, P, P, I64, P, P, I64, I64, I64, F, U32], ctypes.c_int),
                "oracle_rmsnorm_quant_fp8_static":
                    ([P, I64, P, P, I64, P, F, P, I64, P, I64, I64, I64, F, U32], ctypes.c_int),
                "oracle_layernorm_quant_fp8":
                    ([P, I64, P, P, F, P, I64, I64, I64, F, U32], ctypes.c_int),
                "oracle_per_token_group_quant_fp8":
                    ([P, I64, P, I64, P, I64, I64, I64, ctypes.c_int32, U32], ctypes.c_int),
                "oracle_rmsnorm_quant_fp8_group":
                    ([P, I64, P, P, I64, P, P, I64, P, I64, P, I64, I64, I64, ctypes.c_int32, F, U32],
                     ctypes.c_int),
                "oracle_rmsnorm_quant_nvfp4":
                    ([P, I64, P, P, I64, P, F, P, I64, P, I64, P, I64, I64, I64, F, U32],
                     ctypes.c_int),
            }
            for name, (args, res) in sig.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = res
            _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.asarray(a)
    if a.dtype != dtype:
        a = a.astype(dtype)
    return np.ascontiguousarray(a)


def _ld(a):
    return a.shape[-1] if a.ndim == 2 else a.shape[0]


# ---------------------------------------------------------------- codecs ----
def bf16_from_f32(v) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint16)
    _load().oracle_bf16_from_f32(_p(v), _p(out), v.size)
    return out


def bf16_to_f32(b) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def e4m3_encode(v) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    _load().oracle_e4m3_encode(_p(v), _p(out), v.size)
    return out


def e4m3_decode(c) -> np.ndarray:
    c = _c(c, np.uint8)
    out = np.empty(c.shape, np.float32)
    _load().oracle_e4m3_decode(_p(c), _p(out), c.size)
    return out


def e5m2_encode(v) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    _load().oracle_e5m2_encode(_p(v), _p(out), v.size)
    return out


def e5m2_decode(c) -> np.ndarray:
    c = _c(c, np.uint8)
    out = np.empty(c.shape, np.float32)
    _load().oracle_e5m2_decode(_p(c), _p(out), c.size)
    return out


def e2m1_encode(v) -> np.ndarray:
    """One e2m1 code per output byte (low nibble)."""
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    _load().oracle_e2m1_encode(_p(v), _p(out), v.size)
    return out


def e2m1_decode(c) -> np.ndarray:
    c = _c(c, np.uint8)
    out = np.empty(c.shape, np.float32)
    _load().oracle_e2m1_decode(_p(c), _p(out), c.size)
    return out


def ue8m0_ceil(s) -> np.ndarray:
    s = _c(s, np.float32)
    out = np.empty(s.shape, np.float32)
    _load().oracle_ue8m0_ceil(_p(s), _p(out), s.size)
    return out


def canonical_sum(v, squares: bool = False) -> np.float32:
    v = _c(v, np.float32)
    return np.float32(_load().oracle_canonical_sum(_p(v), v.size, int(squares)))


def unpack_e2m1(q: np.ndarray, d: int) -> np.ndarray:
    """Packed bytes [M, >= d/2] -> one code per element [M, d] (low nibble first)."""
    q = np.asarray(q, np.uint8)
    out = np.empty(q.shape[:-1] + (d,), np.uint8)
    out[..., 0::2] = q[..., : d // 2] & 0xF
    out[..., 1::2] = q[..., : d // 2] >> 4
    return out


# ------------------------------------------------------------ norm rows ----
def rms_y(x, gamma, residual=None, eps=1e-6, d=None, flags=0) -> np.ndarray:
    """fp32 RMSNorm output y [M, d] (residual added first when given)."""
    x = _c(x, np.uint16)
    M = x.shape[0]
    d = x.shape[1] if d is None else d
    g = _c(gamma, np.uint16)
    r = None if residual is None else _c(residual, np.uint16)
    y = np.empty((M, d), np.float32)
    _load().oracle_rms_y(_p(x), _ld(x), _p(r), 0 if r is None else _ld(r), _p(g), _p(y), d,
                         M, d, eps, flags)
    return y


def ln_y(x, gamma, beta, eps=1e-5, flags=0) -> np.ndarray:
    x = _c(x, np.uint16)
    M, d = x.shape
    g, b = _c(gamma, np.float32), _c(beta, np.float32)
    y = np.empty((M, d), np.float32)
    _load().oracle_ln_y(_p(x), _ld(x), _p(g), _p(b), _p(y), d, M, d, eps, flags)
    return y


# ------------------------------------------------------------ the five ----
def fused_add_rmsnorm_quant_fp8(x, residual, gamma, eps=1e-6, flags=0, d=None,
                                want_norm=False):
    """Residual-add + RMSNorm + dynamic per-token e4m3.

    Returns ``(q uint8 [M,d], scale float32 [M], residual_out uint16 [M,d],
    norm_out uint16 [M,d] or None)``.  ``x`` may be wider than ``d`` (a
    row-strided slice starting at column 0).
    """
    x = _c(x, np.uint16)
    M = x.shape[0]
    d = x.shape[1] if d is None else d
    res = _c(residual, np.uint16)
    g = _c(gamma, np.uint16)
    q = np.empty((M, d), np.uint8)
    s = np.empty((M,), np.float32)
    ro = np.empty((M, d), np.uint16)
    no = np.empty((M, d), np.uint16) if want_norm else None
    rc = _load().oracle_fused_add_rmsnorm_quant_fp8(
        _p(x), _ld(x), _p(res), _p(ro), d, _p(g), _p(q), d, _p(s), _p(no), d, M, d, eps, flags)
    assert rc == 0
    return q, s, ro, no


def rmsnorm_quant_fp8_static(x, gamma, scale, residual=None, eps=1e-6, flags=0, d=None,
                             want_norm=False):
    """RMSNorm (optional residual) + e4m3 with a static scale value.

    Returns ``(q, residual_out or None, norm_out or None)``.
    """
    x = _c(x, np.uint16)
    M = x.shape[0]
    d = x.shape[1] if d is None else d
    res = None if residual is None else _c(residual, np.uint16)
    g = _c(gamma, np.uint16)
    q = np.empty((M, d), np.uint8)
    ro = None if res is None else np.empty((M, d), np.uint16)
    no = np.empty((M, d), np.uint16) if want_norm else None
    rc = _load().oracle_rmsnorm_quant_fp8_static(
        _p(x), _ld(x), _p(res), _p(ro), d, _p(g), float(scale), _p(q), d, _p(no), d, M, d,
        eps, flags)
    assert rc == 0
    return q, ro, no


def layernorm_quant_fp8(x, gamma, beta, scale, eps=1e-5, flags=0):
    x = _c(x, np.uint16)
    M, d = x.shape
    g, b = _c(gamma, np.float32), _c(beta, np.float32)
    q = np.empty((M, d), np.uint8)
    rc = _load().oracle_layernorm_quant_fp8(_p(x), d, _p(g), _p(b), float(scale), _p(q), d,
                                            M, d, eps, flags)
    assert rc == 0
    return q


def per_token_group_quant_fp8(x, group=128, flags=0):
    """Returns ``(q uint8 [M,K], scales float32 [M, K/group])``."""
    x = _c(x, np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.uint8)
    s = np.empty((M, K // group), np.float32)
    rc = _load().oracle_per_token_group_quant_fp8(_p(x), K, _p(q), K, _p(s), K // group, M, K,
                                                  group, flags)
    assert rc == 0
    return q, s


def rmsnorm_quant_fp8_group(x, gamma, residual=None, group=128, eps=1e-6, flags=0, d=None,
                            want_norm=False):
    """RMSNorm (optional residual) + per-token-group e4m3 of y.

    Returns ``(q uint8 [M, d], scales float32 [M, d/group], residual_out or
    None, norm_out or None)``.
    """
    x = _c(x, np.uint16)
    M = x.shape[0]
    d = x.shape[1] if d is None else d
    res = None if residual is None else _c(residual, np.uint16)
    g = _c(gamma, np.uint16)
    q = np.empty((M, d), np.uint8)
    s = np.empty((M, d // group), np.float32)
    ro = None if res is None else np.empty((M, d), np.uint16)
    no = np.empty((M, d), np.uint16) if want_norm else None
    rc = _load().oracle_rmsnorm_quant_fp8_group(
        _p(x), _ld(x), _p(res), _p(ro), d, _p(g), _p(q), d, _p(s), d // group, _p(no), d, M, d, group,
        eps, flags)
    assert rc == 0
    return q, s, ro, no


def rmsnorm_quant_nvfp4(x, gamma, global_scale, residual=None, eps=1e-6, flags=0, d=None,
                        want_norm=False):
    """RMSNorm (optional residual) + NVFP4.

    Returns ``(q uint8 [M, d/2] packed, sf uint8 [M, d/16], residual_out or
    None, norm_out or None)``.
    """
    x = _c(x, np.uint16)
    M = x.shape[0]
    d = x.shape[1] if d is None else d
    res = None if residual is None else _c(residual, np.uint16)
    g = _c(gamma, np.uint16)
    q = np.empty((M, d // 2), np.uint8)
    sf = np.empty((M, d // 16), np.uint8)
    ro = None if res is None else np.empty((M, d), np.uint16)
    no = np.empty((M, d), np.uint16) if want_norm else None
    rc = _load().oracle_rmsnorm_quant_nvfp4(
        _p(x), _ld(x), _p(res), _p(ro), d, _p(g), float(global_scale), _p(q), d // 2, _p(sf),
        d // 16, _p(no), d, M, d, eps, flags)
    assert rc == 0
    return q, sf, ro, no


def nvfp4_global_scale(x, gamma, residual=None, eps=1e-6, d=None) -> float:
    """Stand-in for a calibrated static NVFP4 input scale: max|y| / (6 * 448)."""
    y = rms_y(x, gamma, residual, eps, d)
    amax = float(np.max(np.abs(y))) if y.size else 0.0
    return float(np.float32(amax / (E2M1_MAX * E4M3_MAX))) if amax > 0 else 1.0


def sf_swizzle(sf) -> np.ndarray:
    """Row-major block scales [rows, n] (uint8) -> the swizzled 128 x 4-tile
    layout of block-scaled GEMMs, zero padded (flat uint8 array)."""
    sf = _c(sf, np.uint8)
    rows, n = sf.shape
    out = np.empty(int(_load().oracle_sf_swizzled_size(rows, n)), np.uint8)
    _load().oracle_sf_swizzle(_p(sf), n, rows, n, _p(out))
    return out


def group_scales_layout(s, col_major=False, packed=False, ld=None) -> np.ndarray:
    """Row-major group scales [M, G] float32 -> the requested layout.

    fp32: [M, G] (row-major) or [G, ld] (col_major, ld >= M).  packed (UE8M0
    scales): uint32 words of four exponent bytes, [M, ld] with ld >= ceil(G/4)
    or [ceil(G/4), ld] with ld >= M when col_major.
    """
    s = _c(s, np.float32)
    M, G = s.shape
    W = (G + 3) // 4
    if ld is None:
        ld = M if col_major else (W if packed else G)
    shape = ((W if packed else G), ld) if col_major else (M, ld)
    out = np.zeros(shape, np.uint32 if packed else np.float32)
    rc = _load().oracle_group_scales_layout(_p(s), M, G, int(col_major), int(packed), ld, _p(out))
    if rc != 0:
        raise ValueError("packed UE8M0 layout needs power-of-two scales in [2^-127, 2^127]")
    return out


def moe_scatter(q, scales, dest, rows):
    """Rows of a per-token result in the experts' permuted order: row
    dest[t, j] of the output is token t's row, for every slot j with
    dest[t, j] >= 0 (the definition of the dispatch; rows nobody targets stay
    zero).  q [M, n] -> [rows, n]; scales [M] or [M, G] likewise."""
    q = np.asarray(q)
    s = np.asarray(scales)
    dest = np.asarray(dest)
    qo = np.zeros((rows,) + q.shape[1:], q.dtype)
    so = np.zeros((rows,) + s.shape[1:], s.dtype)
    t, j = np.nonzero(dest >= 0)
    qo[dest[t, j]] = q[t]
    so[dest[t, j]] = s[t]
    return qo, so
