"""Seeded synthetic inputs shared by the CUDA path's tests and by the oracle.

This module holds no arithmetic of the method (no norm, no scale, no
quantizer). It only draws numbers: every tensor is a pure function of
``(seed, stream_id, shape)``, so the oracle and the GPU path can be fed the
same bits.

Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014), used counter-style: output ``i`` of a
stream is ``mix(base + (i + 1) * golden)`` where ``base`` is derived from the
seed and stream id.  Normals come from the Box–Muller transform in float64,
then are rounded to float32 and from there to bf16 (round to nearest even on
the bit pattern).  The bf16 conversion here is part of *making inputs*; the
oracle and the kernels each have their own rounding code for *outputs*.

Workload recipes (shapes and distributions of the pages' configurations):

* ``x``, ``residual``: bf16 N(0, 1);
* RMSNorm gamma: bf16 ``1 + 0.1 * N(0, 1)``; LayerNorm gamma (fp32) the same,
  beta fp32 ``0.02 * N(0, 1)``;
* group-quant outliers: each element independently multiplied by 50 with
  probability 0.001;
* sweep outliers: channels ``floor((2k + 1) * d / 8) + 1``, k = 0..3, of ``x``
  multiplied by 100.
"""
from __future__ import annotations

import concurrent.futures as cf
import os

import numpy as np

__all__ = [
    "splitmix64_stream",
    "uniform01",
    "normal_f64",
    "f64_to_bf16_bits",
    "bf16_bits_to_f32",
    "bf16_normal",
    "f32_normal",
    "bernoulli",
    "outlier_channels",
    "Workload",
    "make_rms_inputs",
    "make_ln_inputs",
    "make_group_inputs",
]

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _base(seed: int, stream_id: int) -> np.uint64:
    s = np.array([(seed * 0x100000001B3 + stream_id * 0x9E3779B1 + 0x5851F42D4C957F2D)
                  & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(s + _GOLDEN)[0]


def splitmix64_stream(seed: int, stream_id: int, n: int, offset: int = 0) -> np.ndarray:
    """``n`` raw 64-bit outputs of stream ``(seed, stream_id)`` starting at ``offset``."""
    base = _base(seed, stream_id)
    out = np.empty(n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        for lo in range(0, n, _CHUNK):
            hi = min(n, lo + _CHUNK)
            idx = np.arange(offset + lo + 1, offset + hi + 1, dtype=np.uint64)
            out[lo:hi] = _mix(base + idx * _GOLDEN)
    return out


def uniform01(seed: int, stream_id: int, n: int, offset: int = 0) -> np.ndarray:
    """Uniform float64 in (0, 1]: the top 53 bits plus one, times 2**-53."""
    z = splitmix64_stream(seed, stream_id, n, offset)
    return ((z >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)


def _normal_block(seed: int, stream_id: int, lo: int, hi: int, out: np.ndarray) -> None:
    u = uniform01(seed, stream_id, 2 * (hi - lo), offset=2 * lo)
    u1, u2 = u[0::2], u[1::2]
    rad = np.sqrt(-2.0 * np.log(u1))
    ang = 2.0 * np.pi * u2
    out[2 * lo:2 * hi:2] = rad * np.cos(ang)
    out[2 * lo + 1:2 * hi:2] = rad * np.sin(ang)


def normal_f64(seed: int, stream_id: int, n: int) -> np.ndarray:
    """Standard normals by Box–Muller, both branches used (cos for even, sin for odd).

    Pair ``i`` uses uniforms ``2i`` and ``2i + 1`` of the stream, so blocks of
    pairs are independent and are generated on a few threads (numpy releases
    the GIL); the result does not depend on the blocking.
    """
    half = (n + 1) // 2
    out = np.empty(2 * half, dtype=np.float64)
    block = 1 << 20
    spans = [(lo, min(half, lo + block)) for lo in range(0, half, block)]
    if len(spans) <= 1:
        for lo, hi in spans:
            _normal_block(seed, stream_id, lo, hi, out)
    else:
        with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            list(ex.map(lambda sp: _normal_block(seed, stream_id, sp[0], sp[1], out), spans))
    return out[:n]


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """float64 -> float32 (numpy RNE) -> bf16 bit pattern (RNE on the 16 dropped bits)."""
    b = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    r = ((b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_normal(seed: int, stream_id: int, shape, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    """bf16 bit patterns (uint16 array of ``shape``) of ``mean + std * N(0, 1)``."""
    n = int(np.prod(shape)) if len(shape) else 1
    v = mean + std * normal_f64(seed, stream_id, n)
    return f64_to_bf16_bits(v).reshape(shape)


def f32_normal(seed: int, stream_id: int, shape, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    n = int(np.prod(shape)) if len(shape) else 1
    return (mean + std * normal_f64(seed, stream_id, n)).astype(np.float32).reshape(shape)


def bernoulli(seed: int, stream_id: int, shape, p: float) -> np.ndarray:
    n = int(np.prod(shape))
    return (uniform01(seed, stream_id, n) <= p).reshape(shape)


def outlier_channels(d: int) -> list[int]:
    """The four outlier channels of the sweep: floor((2k+1) d / 8) + 1, clipped to d-1."""
    return sorted({min(d - 1, (2 * k + 1) * d // 8 + 1) for k in range(4)})


# Stream ids: one per tensor role, so that changing one tensor's shape never
# changes another tensor's bits.
SID_X, SID_RES, SID_GAMMA, SID_BETA, SID_OUTLIER = 1, 2, 3, 4, 5


class Workload(dict):
    """A dict of named numpy arrays (bf16 as uint16 bit patterns) plus metadata."""


def make_rms_inputs(M: int, d: int, seed: int = 0, residual: bool = True,
                    ld_x: int | None = None, x_outlier_channels: bool = False) -> Workload:
    """Inputs of the residual-add + RMSNorm configurations.

    ``x`` is ``[M, ld_x]`` bf16 (the kernel reads the first ``d`` columns, or a
    column slice chosen by the caller); ``residual`` is ``[M, d]``; ``gamma``
    is bf16 ``[d]`` = 1 + 0.1 N(0, 1).
    """
    ld_x = d if ld_x is None else ld_x
    w = Workload()
    x = bf16_normal(seed, SID_X, (M, ld_x))
    if x_outlier_channels:
        xf = bf16_bits_to_f32(x).copy()
        for c in outlier_channels(d):
            xf[:, c] *= 100.0
        x = f64_to_bf16_bits(xf.astype(np.float64))
    w["x"] = x
    if residual:
        w["residual"] = bf16_normal(seed, SID_RES, (M, d))
    w["gamma"] = bf16_normal(seed, SID_GAMMA, (d,), mean=1.0, std=0.1)
    w.update(M=M, d=d, ld_x=ld_x, seed=seed)
    return w


def make_ln_inputs(M: int, d: int, seed: int = 0) -> Workload:
    """Inputs of the LayerNorm configuration: bf16 x, fp32 gamma = 1 + 0.1 N, fp32 beta = 0.02 N."""
    w = Workload()
    w["x"] = bf16_normal(seed, SID_X, (M, d))
    w["gamma"] = f32_normal(seed, SID_GAMMA, (d,), mean=1.0, std=0.1)
    w["beta"] = f32_normal(seed, SID_BETA, (d,), mean=0.0, std=0.02)
    w.update(M=M, d=d, seed=seed)
    return w


def make_group_inputs(M: int, K: int, seed: int = 0, outlier_p: float = 0.001,
                      outlier_mult: float = 50.0) -> Workload:
    """Inputs of the per-token-group configuration: bf16 N(0, 1) with rare x50 outliers."""
    w = Workload()
    v = normal_f64(seed, SID_X, M * K)
    if outlier_p > 0:
        mask = bernoulli(seed, SID_OUTLIER, (M * K,), outlier_p)
        v = np.where(mask, v * outlier_mult, v)
    w["x"] = f64_to_bf16_bits(v).reshape(M, K)
    w.update(M=M, K=K, seed=seed)
    return w


SID_ROUTE = 6


def make_moe_routing(M: int, E: int, topk: int, seed: int = 0, drop_p: float = 0.0) -> Workload:
    """Synthetic MoE routing: each token picks `topk` distinct experts (uniform,
    seeded), and every (token, slot) gets the row it occupies in the experts'
    permuted input: expert-major, and by (token, slot) within an expert.  With
    drop_p > 0, that fraction of (token, slot) pairs is dropped (row -1), as a
    capacity limit would.  This is routing data for the tests and the sweep, not
    part of the method."""
    keys = uniform01(seed, SID_ROUTE, M * E).reshape(M, E)
    topk_ids = np.argsort(keys, axis=1, kind="stable")[:, :topk].astype(np.int32)
    flat_e = topk_ids.reshape(-1).astype(np.int64)
    keep = np.ones(M * topk, bool)
    if drop_p > 0:
        keep = uniform01(seed, SID_ROUTE + 1, M * topk) > drop_p
    order = np.lexsort((np.arange(M * topk), flat_e))  # by expert, then (token, slot)
    order = order[keep[order]]
    dest = np.full(M * topk, -1, np.int64)
    dest[order] = np.arange(order.size)
    counts = np.bincount(flat_e[keep], minlength=E)
    w = Workload()
    w["topk_ids"] = topk_ids
    w["dest"] = dest.reshape(M, topk).astype(np.int32)
    w["expert_offsets"] = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    w.update(M=M, E=E, topk=topk, rows=int(order.size), seed=seed)
    return w
