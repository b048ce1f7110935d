"""GEMM-ready scale layouts of the CUDA path vs the oracle (needs a B200).

Swizzled NVFP4 block scales: the whole buffer, padding included, equals the
oracle's swizzle of its row-major block scales (padding is defined as zero; the
buffer is pre-filled with 0xFF and guarded past its end).  Codes, residual and
norm outputs are those of the row-major call.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from gpu_helpers import dev_bf16, host_u8, host_u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp4_activation_quantization_b200 as nq
    return nq


def all_schedules(d):
    C = (d + 7) // 8
    return [(lt, lk) for lt in range(5, 11) for lk in range(0, 4) if lt + lk <= 11 and (1 << (lt + lk)) >= C]


def run_swizzled(nq, w, d, gn, residual, flags=0, xoff=0, want_norm=False):
    M = w["x"].shape[0]
    x = dev_bf16(w["x"])[:, xoff:xoff + d]
    size = nq.sf_swizzled_size(M, d)
    guard = 64
    raw = torch.full((size + guard,), 0xFF, dtype=torch.uint8, device="cuda")
    sf = raw[:size].view(torch.float8_e4m3fn)
    gs = torch.tensor([gn], dtype=torch.float32, device="cuda")
    res = dev_bf16(w["residual"]) if residual else None
    q, sf, ro, no = nq.nq_rmsnorm_quant_nvfp4(x, dev_bf16(w["gamma"]), gs, 1e-6, residual=res, sf_out=sf,
                                              want_norm=want_norm, flags=flags | nq.FLAG_SF_SWIZZLED)
    torch.cuda.synchronize()
    tail = raw[size:].cpu().numpy()
    assert np.all(tail == 0xFF), "write past the swizzled buffer"
    return (host_u8(q), host_u8(sf), None if ro is None else host_u16(ro), None if no is None else host_u16(no))


@pytest.mark.parametrize("residual", [False, True])
@pytest.mark.parametrize("M,d", [(1, 7168), (64, 1536), (127, 512), (128, 48), (129, 2064), (300, 16),
                                 (8192, 7168)])
def test_nvfp4_swizzled_sf_bit_exact(nq, M, d, residual):
    w = S.make_rms_inputs(M, d, seed=M + d, residual=residual, x_outlier_channels=True)
    gn = oracle.nvfp4_global_scale(w["x"], w["gamma"], w.get("residual"))
    eq, esf, er, en = oracle.rmsnorm_quant_nvfp4(w["x"], w["gamma"], gn, w.get("residual"), want_norm=True)
    q, sf, ro, no = run_swizzled(nq, w, d, gn, residual, want_norm=True)
    assert np.array_equal(q, eq)
    assert np.array_equal(sf, oracle.sf_swizzle(esf))
    assert np.array_equal(no, en)
    if residual:
        assert np.array_equal(ro, er)


@pytest.mark.parametrize("d", [16, 112, 2064, 8208])
def test_nvfp4_swizzled_every_schedule_and_variant(nq, d):
    M = 37
    w = S.make_rms_inputs(M, d, seed=d + 2, residual=False)
    gn = oracle.nvfp4_global_scale(w["x"], w["gamma"])
    eq, esf, _, _ = oracle.rmsnorm_quant_nvfp4(w["x"], w["gamma"], gn)
    esw = oracle.sf_swizzle(esf)
    flags = [0] + [nq.flag_schedule(*s_) for s_ in all_schedules(d)] + [nq.flag_variant(v) for v in (1, 2, 3)]
    if (d + 7) // 8 <= 512:
        flags.append(nq.flag_variant(2) | nq.flag_schedule(5, 4))
    for f in flags:
        q, sf, _, _ = run_swizzled(nq, w, d, gn, False, flags=f)
        assert np.array_equal(q, eq), hex(f)
        assert np.array_equal(sf, esw), hex(f)


def test_nvfp4_swizzled_misaligned_slice_and_div(nq):
    M, d = 140, 1536
    w = S.make_rms_inputs(M, d, seed=4, residual=True, ld_x=2112)
    xs = w["x"][:, 1:1 + d]
    gn = oracle.nvfp4_global_scale(xs, w["gamma"], w["residual"])
    eq, esf, er, _ = oracle.rmsnorm_quant_nvfp4(xs, w["gamma"], gn, w["residual"], flags=oracle.DIV)
    q, sf, ro, _ = run_swizzled(nq, w, d, gn, True, flags=nq.FLAG_SCALE_DIV, xoff=1)
    assert np.array_equal(q, eq) and np.array_equal(ro, er)
    assert np.array_equal(sf, oracle.sf_swizzle(esf))


# ------------------------------------------------- group-scale layouts ----
LAYOUTS = [("col", True, False), ("packed", False, True), ("packed_col", True, True)]


def scales_buffer(nq, M, G, col, packed, pad):
    """A sentinel-filled buffer for the layout, with `pad` spare elements per
    leading-dimension line; returns (buffer, the [M, n] view the binding takes, ld)."""
    n = (G + 3) // 4 if packed else G
    dt = torch.int32 if packed else torch.float32
    ld = (M if col else n) + pad
    buf = torch.full((n, ld) if col else (M, ld), -7, dtype=dt, device="cuda")
    view = buf[:, :M].t() if col else buf[:, :n]
    return buf, view, ld


def expect_layout(es, col, packed, ld):
    exp = oracle.group_scales_layout(es, col_major=col, packed=packed, ld=ld)
    return exp.view(np.int32) if packed else exp


def check_layout_buffer(buf, exp, M, G, col, packed):
    got = buf.cpu().numpy()
    n = (G + 3) // 4 if packed else G
    inner = got[:, :M] if col else got[:, :n]
    want = exp[:, :M] if col else exp[:, :n]
    assert np.array_equal(inner.view(np.uint32), want.view(np.uint32))
    spare = got[:, M:] if col else got[:, n:]
    assert np.all(spare == -7), "write outside the scale layout"


@pytest.mark.parametrize("name,col,packed", LAYOUTS)
@pytest.mark.parametrize("group,K", [(128, 4096), (128, 2816), (64, 960), (128, 384)])
def test_group_scale_layouts_standalone(nq, name, col, packed, group, K):
    M = 301
    G = K // group
    w = S.make_group_inputs(M, K, seed=K + group)
    x = dev_bf16(w["x"])
    of = oracle.UE8M0 if packed else 0
    eq, es = oracle.per_token_group_quant_fp8(w["x"], group, of)
    flags = (nq.FLAG_SCALES_COL_MAJOR if col else 0) | (nq.FLAG_SCALES_PACKED_UE8M0 if packed else 0)
    scheds = [None] + [(lt, lu) for lt in range(1, 5 if group == 128 else 4) for lu in range(3)]
    for sched in scheds:
        buf, view, ld = scales_buffer(nq, M, G, col, packed, pad=3)
        f = flags | (0 if sched is None else nq.flag_group_schedule(*sched))
        q, s = nq.nq_per_token_group_quant_fp8(x, group, scales_out=view, flags=f)
        torch.cuda.synchronize()
        assert np.array_equal(host_u8(q), eq), (name, sched)
        check_layout_buffer(buf, expect_layout(es, col, packed, ld), M, G, col, packed)


def test_group_scale_layouts_default_allocation(nq):
    """The binding's own buffers: a column-major [M, G] view and packed int32 words."""
    M, K = 70, 2048
    w = S.make_group_inputs(M, K, seed=3)
    _, es = oracle.per_token_group_quant_fp8(w["x"], 128, 0)
    _, s = nq.nq_per_token_group_quant_fp8(dev_bf16(w["x"]), 128, flags=nq.FLAG_SCALES_COL_MAJOR)
    assert s.shape == (M, 16) and s.stride() == (1, M)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), es.view(np.uint32))
    _, eu = oracle.per_token_group_quant_fp8(w["x"], 128, oracle.UE8M0)
    _, p = nq.nq_per_token_group_quant_fp8(dev_bf16(w["x"]), 128, flags=nq.FLAG_SCALES_PACKED_UE8M0)
    assert p.dtype == torch.int32 and p.shape == (M, 4)
    assert np.array_equal(p.cpu().numpy().view(np.uint32), oracle.group_scales_layout(eu, packed=True))


@pytest.mark.parametrize("name,col,packed", LAYOUTS)
@pytest.mark.parametrize("residual", [False, True])
@pytest.mark.parametrize("d,M", [(4096, 300), (2816, 40), (7168, 9), (1024, 77)])
def test_group_scale_layouts_fused(nq, name, col, packed, residual, d, M):
    group = 128
    G = d // group
    w = S.make_rms_inputs(M, d, seed=d + M, residual=residual, x_outlier_channels=True)
    x, g = dev_bf16(w["x"]), dev_bf16(w["gamma"])
    res = dev_bf16(w["residual"]) if residual else None
    of = oracle.UE8M0 if packed else 0
    for e5 in (False, True):
        eq, es, er, _ = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"], w.get("residual"), group=group,
                                                       flags=of | (oracle.E5M2 if e5 else 0))
        flags = (nq.FLAG_SCALES_COL_MAJOR if col else 0) | (nq.FLAG_SCALES_PACKED_UE8M0 if packed else 0)
        flags |= nq.FLAG_E5M2 if e5 else 0
        variants = [0] + [nq.flag_schedule(*s_) for s_ in all_schedules(d)]
        if not residual:
            variants += [nq.flag_variant(v) for v in (2, 3)]
        for v in variants:
            buf, view, ld = scales_buffer(nq, M, G, col, packed, pad=2)
            q, s, ro, _ = nq.nq_rmsnorm_quant_fp8_group(x, g, 1e-6, group=group, residual=res, scales_out=view,
                                                        flags=flags | v)
            torch.cuda.synchronize()
            assert np.array_equal(host_u8(q), eq), (name, e5, hex(v))
            check_layout_buffer(buf, expect_layout(es, col, packed, ld), M, G, col, packed)
            if residual:
                assert np.array_equal(host_u16(ro), er)
