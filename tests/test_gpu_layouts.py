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
