"""Every norm call on the GPU against the oracle's plain definition of the row
sums (needs a B200).

The pages fix no summation order.  The bit-exact tests elsewhere compare the
kernels with the oracle's canonical chunked order; these compare them with the
oracle's SUM_PLAIN mode, where every row sum (sum of squares, LayerNorm mean
and variance) is a float64 sequential sum rounded once to float32, the plain
definition of the mean.  The tolerance is the one stated for a differing
reduction order:

* per-token and per-group float32 scales within 1e-6 relative (zero scales
  equal);
* FP8 / e2m1 codes and NVFP4 e4m3 block-scale codes: at most 1 ulp apart
  (adjacent codes in magnitude order within one sign), on at most 0.1 % of
  them;
* the residual update, which does not depend on any sum: bit-exact.

The element-mismatch fraction as the accuracy check follows FlashInfer PR
#3962 (review thread: a mismatch fraction rather than a loose rtol / atol);
the 1-ulp bound follows vLLM PR #61343 (Validation: casts flip by one step on a
few hundredths of a percent of elements when the arithmetic changes).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from gpu_helpers import dev_bf16, dev_f32, e2m1_rank, e4m3_rank, host_u8, host_u16

pytestmark = pytest.mark.gpu

MAX_FRAC = 1e-3   # at most 0.1 % of codes may differ ...
MAX_ULP = 1       # ... and by at most one code
SCALE_RTOL = 1e-6


@pytest.fixture(scope="module")
def nq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp4_activation_quantization_b200 as nq
    return nq


def assert_codes_close(got, exp, rank, what):
    diff = np.abs(rank(got).astype(np.int64) - rank(exp).astype(np.int64))
    assert diff.max(initial=0) <= MAX_ULP, f"{what}: codes {diff.max()} apart at {np.argwhere(diff > MAX_ULP)[:4]}"
    frac = float((diff > 0).mean()) if diff.size else 0.0
    assert frac <= MAX_FRAC, f"{what}: {frac:.3e} of codes differ"
    return frac


def assert_scales_close(got, exp, what):
    got = np.asarray(got, np.float64)
    exp = np.asarray(exp, np.float64)
    zero = exp == 0
    assert np.array_equal(got[zero], exp[zero]), f"{what}: zero scales differ"
    rel = np.abs(got[~zero] / exp[~zero] - 1.0)
    assert rel.max(initial=0.0) <= SCALE_RTOL, f"{what}: relative scale error {rel.max():.3e}"


def bf16_rank(u16):
    """Signed position of a bf16 bit pattern on the number line (as e4m3_rank)."""
    u = np.asarray(u16, np.int64)
    mag = u & 0x7FFF
    return np.where(u & 0x8000, -mag, mag)


# ---------------------------------------------- dynamic per-token FP8 ----
@pytest.mark.parametrize("M,d", [(64, 2816), (4096, 8192), (4096, 2816)])
def test_fused_dynamic_plain_order(nq, M, d):
    """Residual-add + RMSNorm + dynamic e4m3 at the small configuration and two sweep cells."""
    w = S.make_rms_inputs(M, d, seed=11, x_outlier_channels=M > 64)
    res = dev_bf16(w["residual"])
    q, s, ro, no = nq.nq_fused_add_rmsnorm_quant_fp8(dev_bf16(w["x"]), res, dev_bf16(w["gamma"]), 1e-6,
                                                     want_norm=True)
    torch.cuda.synchronize()
    eq, es, er, en = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"], flags=oracle.SUM_PLAIN,
                                                        want_norm=True)
    assert np.array_equal(host_u16(ro), er), "residual_out"
    assert_scales_close(s.cpu().numpy(), es, "per-token scales")
    assert_codes_close(host_u8(q), eq, e4m3_rank, "e4m3 codes")
    assert_codes_close(host_u16(no), en, bf16_rank, "bf16 norm_out")


# ----------------------------------------------------- static FP8 ----
@pytest.mark.parametrize("residual", [False, True])
def test_rms_static_plain_order(nq, residual):
    """RMSNorm (with and without residual) -> e4m3, static scale 0.05, 4096 x 4096, eps 1e-5."""
    M, d = 4096, 4096
    w = S.make_rms_inputs(M, d, seed=12, residual=residual)
    sc = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    q, ro, _ = nq.nq_rmsnorm_quant_fp8_static(dev_bf16(w["x"]), dev_bf16(w["gamma"]), sc, 1e-5,
                                              residual=dev_bf16(w["residual"]) if residual else None)
    torch.cuda.synchronize()
    eq, er, _ = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], 0.05, residual=w.get("residual"), eps=1e-5,
                                                flags=oracle.SUM_PLAIN)
    if residual:
        assert np.array_equal(host_u16(ro), er), "residual_out"
    assert_codes_close(host_u8(q), eq, e4m3_rank, "e4m3 codes")


@pytest.mark.parametrize("M,d", [(4096, 4096), (2048, 7168), (1024, 16384)])
def test_layernorm_plain_order(nq, M, d):
    """LayerNorm -> e4m3 (static scale 0.05, eps 1e-5): the two-pass mean / variance is the most
    order-sensitive sum here (the variance sums squares of centred values)."""
    w = S.make_ln_inputs(M, d, seed=13)
    sc = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    q = nq.nq_layernorm_quant_fp8(dev_bf16(w["x"]), dev_f32(w["gamma"]), dev_f32(w["beta"]), sc, 1e-5)
    torch.cuda.synchronize()
    eq = oracle.layernorm_quant_fp8(w["x"], w["gamma"], w["beta"], 0.05, eps=1e-5, flags=oracle.SUM_PLAIN)
    assert_codes_close(host_u8(q), eq, e4m3_rank, "e4m3 codes")


# ------------------------------------------------------------ NVFP4 ----
@pytest.mark.parametrize("residual", [False, True])
@pytest.mark.parametrize("d,ld", [(7168, 7168), (1536, 2112), (512, 512)])
def test_nvfp4_plain_order(nq, d, ld, residual):
    """RMSNorm (+ residual) -> NVFP4 at M = 8192 (d = 1536 is a column slice of a [M, 2112] tensor):
    e4m3 block-scale codes and e2m1 codes within one code on at most 0.1 %."""
    M = 8192
    w = S.make_rms_inputs(M, d, seed=14, residual=residual, ld_x=ld)
    g = oracle.nvfp4_global_scale(w["x"], w["gamma"], w.get("residual"), d=d)
    xs = dev_bf16(w["x"])[:, :d]
    gs = torch.tensor([g], dtype=torch.float32, device="cuda")
    q, sf, ro, _ = nq.nq_rmsnorm_quant_nvfp4(xs, dev_bf16(w["gamma"]), gs, 1e-6,
                                             residual=dev_bf16(w["residual"]) if residual else None)
    torch.cuda.synchronize()
    eq, esf, er, _ = oracle.rmsnorm_quant_nvfp4(w["x"], w["gamma"], g, residual=w.get("residual"), d=d,
                                                flags=oracle.SUM_PLAIN)
    if residual:
        assert np.array_equal(host_u16(ro), er), "residual_out"
    assert_codes_close(host_u8(sf), esf, e4m3_rank, "e4m3 block scales")
    assert_codes_close(oracle.unpack_e2m1(host_u8(q), d), oracle.unpack_e2m1(eq, d), e2m1_rank, "e2m1 codes")


# ----------------------------------------- fused RMSNorm + group FP8 ----
@pytest.mark.parametrize("residual", [False, True])
def test_rms_group_plain_order(nq, residual):
    """RMSNorm (+ residual) -> per-token-group e4m3 (group 128) at 32768 x 4096."""
    M, d = 32768, 4096
    w = S.make_rms_inputs(M, d, seed=15, residual=residual, x_outlier_channels=True)
    q, s, ro, _ = nq.nq_rmsnorm_quant_fp8_group(dev_bf16(w["x"]), dev_bf16(w["gamma"]), 1e-6, group=128,
                                                residual=dev_bf16(w["residual"]) if residual else None)
    torch.cuda.synchronize()
    eq, es, er, _ = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"], w.get("residual"), group=128,
                                                   flags=oracle.SUM_PLAIN)
    if residual:
        assert np.array_equal(host_u16(ro), er), "residual_out"
    assert_scales_close(s.cpu().numpy(), es, "group scales")
    assert_codes_close(host_u8(q), eq, e4m3_rank, "e4m3 codes")


# ------------------------------------------------------- MoE dispatch ----
@pytest.mark.parametrize("group", [0, 128])
def test_moe_dispatch_plain_order(nq, group):
    """Add + RMSNorm -> e4m3 stored into the experts' permuted rows (2048 tokens, d = 7168, 256 experts,
    top-8): every targeted row against the plain-order oracle result of its token."""
    M, d, E, topk = 2048, 7168, 256, 8
    w = S.make_rms_inputs(M, d, seed=16, x_outlier_channels=True)
    r = S.make_moe_routing(M, E, topk, seed=16, drop_p=0.02)
    rows = r["rows"]
    G = d // group if group else 1
    dest = torch.from_numpy(r["dest"]).cuda()
    qo, so, ro, _ = nq.nq_fused_add_rmsnorm_quant_fp8_moe(
        dev_bf16(w["x"]), dev_bf16(w["gamma"]), dest, rows, 1e-6, group=group, residual=dev_bf16(w["residual"]))
    torch.cuda.synchronize()
    if group == 0:
        eq, es, er, _ = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"], flags=oracle.SUM_PLAIN)
    else:
        eq, es, er, _ = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"], w["residual"], group=group,
                                                       flags=oracle.SUM_PLAIN)
    xq, xs = oracle.moe_scatter(eq, es, r["dest"], rows)
    kept = np.unique(r["dest"][r["dest"] >= 0])
    assert np.array_equal(host_u16(ro), er), "residual_out"
    got_s = so.cpu().numpy().reshape(rows, G) if group else so.cpu().numpy()
    assert_scales_close(got_s[kept], xs[kept], "scales")
    assert_codes_close(host_u8(qo)[kept], xq[kept], e4m3_rank, "e4m3 codes")
