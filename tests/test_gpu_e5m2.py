"""e5m2 outputs of the FP8 calls vs the CPU oracle (needs a B200).

With e5m2 the codes saturate at 57344 and the dynamic / group scales are
absmax / 57344 (FlashInfer PR #3962 Description: the output tensor's FP8 type
picks the format).  Every case is bit-exact: codes, scales, residual and norm
outputs; every schedule and kernel variant gives the same bits.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from gpu_helpers import Guarded, dev_bf16, dev_f32, host_u8, host_u16

pytestmark = pytest.mark.gpu
F8 = torch.float8_e5m2


@pytest.fixture(scope="module")
def nq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp4_activation_quantization_b200 as nq
    return nq


def all_schedules(d):
    C = (d + 7) // 8
    return [(lt, lk) for lt in range(5, 11) for lk in range(0, 4) if lt + lk <= 11 and (1 << (lt + lk)) >= C]


def u32(a):
    return np.ascontiguousarray(a).view(np.uint32)


@pytest.mark.parametrize("div", [False, True])
def test_fused_dynamic_e5m2_config(nq, div):
    M, d = 64, 2816
    w = S.make_rms_inputs(M, d, seed=0)
    gq = Guarded(M, d, F8)
    q, s, ro, no = nq.nq_fused_add_rmsnorm_quant_fp8(
        dev_bf16(w["x"]), dev_bf16(w["residual"]), dev_bf16(w["gamma"]), 1e-6, q_out=gq.view, want_norm=True,
        flags=nq.FLAG_SCALE_DIV if div else 0)
    torch.cuda.synchronize()
    assert q.dtype == F8 and gq.guards_intact()
    eq, es, er, en = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"], eps=1e-6,
                                                        flags=oracle.E5M2 | (oracle.DIV if div else 0),
                                                        want_norm=True)
    assert np.array_equal(u32(s.cpu().numpy()), u32(es))
    assert np.array_equal(host_u8(q), eq)
    assert np.array_equal(host_u16(ro), er) and np.array_equal(host_u16(no), en)
    # the row maximum maps to the largest finite e5m2 code
    assert np.all((eq[np.arange(M), np.argmax(np.abs(oracle.e5m2_decode(eq)), axis=1)] & 0x7F) == 0x7B)


@pytest.mark.parametrize("d", [1, 111, 1024, 2816, 8208])
def test_fused_dynamic_e5m2_every_schedule(nq, d):
    M = 11
    w = S.make_rms_inputs(M, d, seed=d + 1, x_outlier_channels=d >= 8)
    w["x"][3] = 0  # with a zero residual row below, a zero row: scale 0, codes are y's signed zeros
    w["residual"][3] = 0
    eq, es, er, _ = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"], flags=oracle.E5M2)
    assert es[3] == 0
    x, r, g = dev_bf16(w["x"]), dev_bf16(w["residual"]), dev_bf16(w["gamma"])
    for sched in [None, *all_schedules(d)]:
        f = nq.FLAG_E5M2 | (0 if sched is None else nq.flag_schedule(*sched))
        q, s, ro, _ = nq.nq_fused_add_rmsnorm_quant_fp8(x, r, g, 1e-6, flags=f)
        assert np.array_equal(host_u8(q), eq), sched
        assert np.array_equal(u32(s.cpu().numpy()), u32(es)), sched
        assert np.array_equal(host_u16(ro), er), sched


@pytest.mark.parametrize("scale", [0.05, 1e-5])
def test_static_e5m2_config(nq, scale):
    """4096 x 4096 RMSNorm (with and without residual) and LayerNorm; scale 1e-5
    drives most codes into e5m2 saturation (|y| / scale > 57344)."""
    M, d = 4096, 4096
    w = S.make_rms_inputs(M, d, seed=0, residual=True)
    lw = S.make_ln_inputs(M, d, seed=0)
    sc = torch.tensor([scale], dtype=torch.float32, device="cuda")
    x, g = dev_bf16(w["x"]), dev_bf16(w["gamma"])
    for res in (None, dev_bf16(w["residual"])):
        q, ro, _ = nq.nq_rmsnorm_quant_fp8_static(x, g, sc, 1e-5, residual=res, flags=nq.FLAG_E5M2)
        eq, er, _ = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], scale,
                                                    residual=None if res is None else w["residual"], eps=1e-5,
                                                    flags=oracle.E5M2)
        assert q.dtype == F8
        assert np.array_equal(host_u8(q), eq)
        if res is not None:
            assert np.array_equal(host_u16(ro), er)
    ql = nq.nq_layernorm_quant_fp8(dev_bf16(lw["x"]), dev_f32(lw["gamma"]), dev_f32(lw["beta"]), sc, 1e-5,
                                   flags=nq.FLAG_E5M2)
    el = oracle.layernorm_quant_fp8(lw["x"], lw["gamma"], lw["beta"], scale, eps=1e-5, flags=oracle.E5M2)
    assert np.array_equal(host_u8(ql), el)
    if scale == 1e-5:
        assert np.mean((el & 0x7F) == 0x7B) > 0.3


@pytest.mark.parametrize("d", [7, 989, 4096])
def test_static_e5m2_every_schedule_and_variant(nq, d):
    M = 13
    w = S.make_rms_inputs(M, d, seed=d, residual=False)
    lw = S.make_ln_inputs(M, d, seed=d)
    sc = torch.tensor([0.01], dtype=torch.float32, device="cuda")
    eq, _, _ = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], 0.01, flags=oracle.E5M2)
    el = oracle.layernorm_quant_fp8(lw["x"], lw["gamma"], lw["beta"], 0.01, eps=1e-6, flags=oracle.E5M2)
    flags = [nq.flag_schedule(*s_) for s_ in all_schedules(d)]
    if d % 8 == 0:
        flags += [nq.flag_variant(v) for v in (1, 2, 3)]
    for f in [0, *flags]:
        q, _, _ = nq.nq_rmsnorm_quant_fp8_static(dev_bf16(w["x"]), dev_bf16(w["gamma"]), sc, 1e-6,
                                                 flags=f | nq.FLAG_E5M2)
        assert np.array_equal(host_u8(q), eq), hex(f)
        ql = nq.nq_layernorm_quant_fp8(dev_bf16(lw["x"]), dev_f32(lw["gamma"]), dev_f32(lw["beta"]), sc, 1e-6,
                                       flags=f | nq.FLAG_E5M2)
        assert np.array_equal(host_u8(ql), el), hex(f)


@pytest.mark.parametrize("group", [64, 128])
def test_group_e5m2_every_team_size(nq, group):
    M, K = 333, 2048
    w = S.make_group_inputs(M, K, seed=group + 5)
    x = dev_bf16(w["x"])
    for flags, of in ((0, 0), (nq.FLAG_UE8M0, oracle.UE8M0), (nq.FLAG_SCALE_DIV, oracle.DIV)):
        eq, es = oracle.per_token_group_quant_fp8(w["x"], group, of | oracle.E5M2)
        for sched in [None] + [(lt, lu) for lt in range(1, 5 if group == 128 else 4) for lu in range(3)]:
            f = flags | nq.FLAG_E5M2 | (0 if sched is None else nq.flag_group_schedule(*sched))
            q, s = nq.nq_per_token_group_quant_fp8(x, group, flags=f)
            assert q.dtype == F8
            assert np.array_equal(host_u8(q), eq), (flags, sched)
            assert np.array_equal(u32(s.cpu().numpy()), u32(es)), (flags, sched)


def test_group_e5m2_config_and_e5m2_q_out_selects_format(nq):
    """32768 x 4096 group 128; a float8_e5m2 q_out picks e5m2 without the flag."""
    M, K = 32768, 4096
    w = S.make_group_inputs(M, K, seed=0)
    q = torch.empty(M, K, dtype=F8, device="cuda")
    _, s = nq.nq_per_token_group_quant_fp8(dev_bf16(w["x"]), 128, q_out=q)
    torch.cuda.synchronize()
    eq, es = oracle.per_token_group_quant_fp8(w["x"], 128, oracle.E5M2)
    assert np.array_equal(host_u8(q), eq)
    assert np.array_equal(u32(s.cpu().numpy()), u32(es))


def test_group_e5m2_cvt_over_all_bf16_values(nq):
    """Groups whose absmax is 57344 have scale 1: their codes are the hardware
    e5m2 conversion of every finite bf16 value in [-57344, 57344]."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = oracle.bf16_to_f32(bits)
    vals = bits[np.isfinite(f) & (np.abs(f) <= 57344)]
    n_per = 127
    G = (len(vals) + n_per - 1) // n_per
    rows = np.zeros((G, 128), np.uint16)
    rows[:, 0] = 0x4760  # 57344.0 in bf16
    flat = np.zeros(G * n_per, np.uint16)
    flat[: len(vals)] = vals
    rows[:, 1:] = flat.reshape(G, n_per)
    q, s = nq.nq_per_token_group_quant_fp8(dev_bf16(rows), 128, flags=nq.FLAG_E5M2)
    eq, es = oracle.per_token_group_quant_fp8(rows, 128, oracle.E5M2)
    assert np.all(es == 1.0)
    assert np.array_equal(host_u8(q), eq)
    assert np.array_equal(u32(s.cpu().numpy()), u32(es))


@pytest.mark.parametrize("residual", [False, True])
@pytest.mark.parametrize("d", [512, 4096, 7168])
def test_rms_group_e5m2(nq, d, residual):
    M = 37
    w = S.make_rms_inputs(M, d, seed=d + 9, residual=residual, x_outlier_channels=True)
    x, g = dev_bf16(w["x"]), dev_bf16(w["gamma"])
    res = dev_bf16(w["residual"]) if residual else None
    for flags, of in ((0, 0), (nq.FLAG_UE8M0, oracle.UE8M0)):
        eq, es, er, en = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"], w.get("residual"), flags=of | oracle.E5M2,
                                                        want_norm=True)
        variants = [0, *[nq.flag_schedule(*s_) for s_ in all_schedules(d)]]
        if not residual:
            variants += [nq.flag_variant(v) for v in (2, 3)]
        for v in variants:
            q, s, ro, no = nq.nq_rmsnorm_quant_fp8_group(x, g, 1e-6, residual=res, want_norm=True,
                                                         flags=flags | v | nq.FLAG_E5M2)
            assert np.array_equal(host_u8(q), eq), (flags, hex(v))
            assert np.array_equal(u32(s.cpu().numpy()), u32(es)), (flags, hex(v))
            assert np.array_equal(host_u16(no), en)
            if residual:
                assert np.array_equal(host_u16(ro), er)


def test_nvfp4_rejects_e5m2(nq):
    w = S.make_rms_inputs(4, 64, seed=1, residual=False)
    gs = torch.tensor([1.0], dtype=torch.float32, device="cuda")
    with pytest.raises(nq.NQError):
        nq.nq_rmsnorm_quant_nvfp4(dev_bf16(w["x"]), dev_bf16(w["gamma"]), gs, 1e-6, flags=nq.FLAG_E5M2)
