"""CUDA path vs the CPU oracle on the same seeded inputs (needs a B200).

Bar (stated per test):
* canonical mode: bit-exact for residual_out, norm_out, scales and codes;
* against the oracle's plain float64-order mode: scales within 1e-6
  relative, codes at most 1 ulp apart on at most 0.1% of elements;
* every schedule the planner can pick gives identical bits;
* outputs never write outside their rows (sentinel guard bands).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from gpu_helpers import (Guarded, dev_bf16, dev_f32, e2m1_rank, e4m3_rank, host_u8, host_u16,
                         same_codes_e4m3)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp4_activation_quantization_b200 as nq
    return nq


def all_schedules(d):
    """Every built (log2 threads, log2 chunks) schedule that covers a row of d elements."""
    C = (d + 7) // 8
    return [(lt, lk) for lt in range(5, 11) for lk in range(0, 4) if lt + lk <= 11 and (1 << (lt + lk)) >= C]


# ------------------------------------------------ dynamic per-token FP8 ----
def run_fused(nq, w, d=None, flags=0, eps=1e-6, want_norm=False, inplace=False, guarded=False):
    x = dev_bf16(w["x"])
    d = x.shape[1] if d is None else d
    xs = x[:, :d]
    res = dev_bf16(w["residual"])
    g = dev_bf16(w["gamma"])
    M = xs.shape[0]
    kw = {}
    guards = []
    if guarded:
        gq = Guarded(M, d, torch.float8_e4m3fn)
        gr = Guarded(M, d, torch.bfloat16)
        gr.view.copy_(res)
        res = gr.view
        kw.update(q_out=gq.view, residual_out=gr.view)
        guards = [gq, gr]
    if inplace:
        kw["residual_out"] = res
    q, s, ro, no = nq.nq_fused_add_rmsnorm_quant_fp8(xs, res, g, eps, flags=flags, want_norm=want_norm, **kw)
    torch.cuda.synchronize()
    for gd in guards:
        assert gd.guards_intact()
    return host_u8(q), s.cpu().numpy(), host_u16(ro), (host_u16(no) if no is not None else None)


def oracle_fused(w, d=None, flags=0, eps=1e-6, want_norm=False):
    return oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"], eps=eps, flags=flags, d=d,
                                              want_norm=want_norm)


def assert_fused_equal(got, exp):
    assert np.array_equal(got[2], exp[2]), "residual_out"
    assert np.array_equal(got[1].view(np.uint32), exp[1].view(np.uint32)), "scales"
    assert np.array_equal(got[0], exp[0]), f"codes differ at {np.argwhere(got[0] != exp[0])[:5]}"
    if exp[3] is not None:
        assert np.array_equal(got[3], exp[3]), "norm_out"


@pytest.mark.parametrize("flags_name", ["default", "div", "recip"])
def test_fused_dynamic_small_config_bit_exact(nq, flags_name):
    """64 tokens x 2816, seed 0, eps 1e-6: bit-exact codes, scales, residual and bf16 norm output."""
    flags = {"default": 0, "div": nq.FLAG_SCALE_DIV, "recip": nq.FLAG_SCALE_RECIP}[flags_name]
    oflags = {"default": 0, "div": oracle.DIV, "recip": oracle.RECIP}[flags_name]
    w = S.make_rms_inputs(64, 2816, seed=0)
    got = run_fused(nq, w, flags=flags, want_norm=True, guarded=True)
    assert_fused_equal(got, oracle_fused(w, flags=oflags, want_norm=True))


@pytest.mark.parametrize("d", [1, 7, 8, 32, 111, 128, 1000, 1024, 2816, 4104, 8192, 8208, 16384])
def test_fused_dynamic_every_schedule(nq, d):
    """Every built schedule covering the row gives the oracle's bits (ragged d included)."""
    M = 19
    w = S.make_rms_inputs(M, d, seed=d, x_outlier_channels=d >= 8)
    exp = oracle_fused(w)
    for lt, lk in all_schedules(d):
        got = run_fused(nq, w, flags=nq.flag_schedule(lt, lk))
        assert_fused_equal(got, exp)
    assert_fused_equal(run_fused(nq, w), exp)


@pytest.mark.parametrize("M", [1, 16, 256, 4096])
@pytest.mark.parametrize("d", [2816, 4096, 7168, 8192])
def test_sweep_cells_bit_exact(nq, M, d):
    """Sweep cells (x with four x100 outlier channels) at the planner's schedule, M <= 4096."""
    w = S.make_rms_inputs(M, d, seed=0, x_outlier_channels=True)
    assert_fused_equal(run_fused(nq, w), oracle_fused(w))


@pytest.mark.parametrize("d", [2816, 8192])
def test_sweep_largest_m_sampled_rows(nq, d):
    """M = 65536 sweep cells: device-generated inputs, sampled rows checked one by one."""
    M = 65536
    gen = torch.Generator(device="cuda").manual_seed(1234 + d)
    x = torch.randn(M, d, device="cuda", generator=gen).to(torch.bfloat16)
    for c in S.outlier_channels(d):
        x[:, c] *= 100
    res = torch.randn(M, d, device="cuda", generator=gen).to(torch.bfloat16)
    g = (1 + 0.1 * torch.randn(d, device="cuda", generator=gen)).to(torch.bfloat16)
    rows = np.unique(np.concatenate([[0, 1, M // 2, M - 2, M - 1],
                                     np.random.default_rng(d).integers(0, M, 59)]))
    res_rows = host_u16(res[rows])
    q, s, ro, _ = nq.nq_fused_add_rmsnorm_quant_fp8(x, res, g, 1e-6)
    torch.cuda.synchronize()
    w = {"x": host_u16(x[rows]), "residual": res_rows, "gamma": host_u16(g)}
    exp = oracle_fused(w)
    got = (host_u8(q[rows]), s[rows].cpu().numpy(), host_u16(ro[rows]), None)
    assert_fused_equal(got, exp)


def test_fused_inplace_residual(nq):
    w = S.make_rms_inputs(33, 4096, seed=3)
    got = run_fused(nq, w, inplace=True)
    assert_fused_equal(got, oracle_fused(w))


def test_fused_plain_order_tolerance(nq):
    """GPU vs the oracle's float64-order sums: scales within 1e-6 relative; codes <= 1 ulp on <= 0.1%."""
    w = S.make_rms_inputs(512, 4096, seed=9, x_outlier_channels=True)
    q, s, ro, _ = run_fused(nq, w)
    eq, es, er, _ = oracle_fused(w, flags=oracle.SUM_PLAIN)
    assert np.array_equal(ro, er)
    assert np.all(np.abs(s.astype(np.float64) / es - 1) <= 1e-6)
    diff = np.abs(e4m3_rank(q) - e4m3_rank(eq))
    assert diff.max() <= 1 and (diff > 0).mean() <= 1e-3


def test_fused_vs_unfused_on_gpu(nq):
    """The bf16 double-rounding emulation matches the oracle's, and differs from fused on ~2-3% of codes."""
    w = S.make_rms_inputs(128, 2816, seed=5)
    fused = run_fused(nq, w)
    unf = run_fused(nq, w, flags=nq.FLAG_NORM_BF16_ROUND)
    assert_fused_equal(unf, oracle_fused(w, flags=oracle.NORM_BF16_ROUND))
    frac = (fused[0] != unf[0]).mean()
    assert 0.015 <= frac <= 0.045


def test_fused_misaligned_column_slice(nq):
    """x starting one element into a wider tensor takes the scalar path; same bits as the oracle."""
    M, d = 40, 1024
    w = S.make_rms_inputs(M, d, seed=4, ld_x=d + 8)
    xfull = dev_bf16(w["x"])
    xs = xfull[:, 1:1 + d]
    res = dev_bf16(w["residual"])
    g = dev_bf16(w["gamma"])
    q, s, ro, _ = nq.nq_fused_add_rmsnorm_quant_fp8(xs, res, g, 1e-6)
    exp = oracle.fused_add_rmsnorm_quant_fp8(w["x"][:, 1:1 + d], w["residual"], w["gamma"])
    assert_fused_equal((host_u8(q), s.cpu().numpy(), host_u16(ro), None), exp)


def test_zero_rows_and_m0(nq):
    d = 256
    x = torch.zeros(9, d, dtype=torch.bfloat16, device="cuda")
    res = torch.zeros_like(x)
    g = torch.ones(d, dtype=torch.bfloat16, device="cuda")
    q, s, ro, _ = nq.nq_fused_add_rmsnorm_quant_fp8(x, res, g, 1e-6)
    assert (s == 0).all() and (host_u8(q) == 0).all()
    e = torch.empty(0, d, dtype=torch.bfloat16, device="cuda")
    q0, s0, r0, _ = nq.nq_fused_add_rmsnorm_quant_fp8(e, torch.empty_like(e), g, 1e-6)
    assert q0.shape == (0, d)


def test_pdl_flag_same_bits(nq):
    w = S.make_rms_inputs(300, 4096, seed=8)
    a = run_fused(nq, w)
    b = run_fused(nq, w, flags=nq.FLAG_PDL)
    assert_fused_equal(b, a)


# ---------------------------------------------------- static-scale FP8 ----
@pytest.mark.parametrize("residual", [False, True])
@pytest.mark.parametrize("flags_name", ["default", "div"])
def test_rms_static_config_bit_exact(nq, residual, flags_name):
    """4096 x 4096, scale 0.05 in device memory, eps 1e-5: bit-exact."""
    M, d = 4096, 4096
    w = S.make_rms_inputs(M, d, seed=0, residual=residual)
    flags = nq.FLAG_SCALE_DIV if flags_name == "div" else 0
    oflags = oracle.DIV if flags_name == "div" else 0
    sc = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    gq = Guarded(M, d, torch.float8_e4m3fn)
    q, ro, no = nq.nq_rmsnorm_quant_fp8_static(dev_bf16(w["x"]), dev_bf16(w["gamma"]), sc, 1e-5,
                                               residual=dev_bf16(w["residual"]) if residual else None,
                                               q_out=gq.view, want_norm=True, flags=flags)
    torch.cuda.synchronize()
    assert gq.guards_intact()
    eq, er, en = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], 0.05, residual=w.get("residual"),
                                                 eps=1e-5, flags=oflags, want_norm=True)
    assert np.array_equal(host_u8(q), eq)
    assert np.array_equal(host_u16(no), en)
    if residual:
        assert np.array_equal(host_u16(ro), er)


@pytest.mark.parametrize("flags_name", ["default", "div"])
def test_layernorm_static_config_bit_exact(nq, flags_name):
    M, d = 4096, 4096
    w = S.make_ln_inputs(M, d, seed=0)
    flags = nq.FLAG_SCALE_DIV if flags_name == "div" else 0
    oflags = oracle.DIV if flags_name == "div" else 0
    sc = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    q = nq.nq_layernorm_quant_fp8(dev_bf16(w["x"]), dev_f32(w["gamma"]), dev_f32(w["beta"]), sc, 1e-5, flags=flags)
    eq = oracle.layernorm_quant_fp8(w["x"], w["gamma"], w["beta"], 0.05, eps=1e-5, flags=oflags)
    assert np.array_equal(host_u8(q), eq)


@pytest.mark.parametrize("d", [1, 7, 111, 128, 989, 2816, 8208, 16384])
def test_static_paths_every_schedule(nq, d):
    """Odd and wide hidden sizes, every schedule, RMSNorm and LayerNorm, three scales."""
    M = 13
    w = S.make_rms_inputs(M, d, seed=d, residual=True)
    lw = S.make_ln_inputs(M, d, seed=d)
    for scale in (0.01, 1.0, 10.0):
        sc = torch.tensor([scale], dtype=torch.float32, device="cuda")
        eq, er, _ = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], scale, residual=w["residual"])
        el = oracle.layernorm_quant_fp8(lw["x"], lw["gamma"], lw["beta"], scale, eps=1e-6)
        for sched in [None, *all_schedules(d)]:
            f = 0 if sched is None else nq.flag_schedule(*sched)
            q, ro, _ = nq.nq_rmsnorm_quant_fp8_static(dev_bf16(w["x"]), dev_bf16(w["gamma"]), sc, 1e-6,
                                                      residual=dev_bf16(w["residual"]), flags=f)
            assert np.array_equal(host_u8(q), eq) and np.array_equal(host_u16(ro), er), (scale, sched)
            ql = nq.nq_layernorm_quant_fp8(dev_bf16(lw["x"]), dev_f32(lw["gamma"]), dev_f32(lw["beta"]), sc,
                                           1e-6, flags=f)
            assert np.array_equal(host_u8(ql), el), (scale, sched)


def test_static_zero_scale_ieee(nq):
    w = S.make_rms_inputs(4, 64, seed=1, residual=False)
    x = w["x"].copy()
    x[0, :8] = 0  # zeros give 0 * inf = NaN codes
    sc = torch.zeros(1, dtype=torch.float32, device="cuda")
    q, _, _ = nq.nq_rmsnorm_quant_fp8_static(dev_bf16(x), dev_bf16(w["gamma"]), sc, 1e-6)
    eq, _, _ = oracle.rmsnorm_quant_fp8_static(x, w["gamma"], 0.0)
    assert same_codes_e4m3(host_u8(q), eq)


def test_static_scale_graph_replay(nq):
    """The scale is read at execution time: a captured graph follows scale updates."""
    w = S.make_rms_inputs(256, 4096, seed=2, residual=False)
    x, g = dev_bf16(w["x"]), dev_bf16(w["gamma"])
    sc = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    q = torch.empty(256, 4096, dtype=torch.float8_e4m3fn, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        nq.nq_rmsnorm_quant_fp8_static(x, g, sc, 1e-6, q_out=q)  # warm-up outside capture
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        nq.nq_rmsnorm_quant_fp8_static(x, g, sc, 1e-6, q_out=q)
    for scale in (0.05, 0.5, 0.013):
        sc.fill_(scale)
        graph.replay()
        torch.cuda.synchronize()
        eq, _, _ = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], scale)
        assert np.array_equal(host_u8(q), eq), scale


# ------------------------------------------------------- group FP8 ----
@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("M", [1, 32768])
def test_group_config_bit_exact(nq, M, ue8m0):
    """bf16 [M, 4096] with 0.1% x50 outliers, group 128, fp32 or UE8M0 scales, x * (1/s)."""
    K = 4096
    w = S.make_group_inputs(M, K, seed=0)
    flags = nq.FLAG_UE8M0 if ue8m0 else 0
    q, s = nq.nq_per_token_group_quant_fp8(dev_bf16(w["x"]), 128, flags=flags)
    torch.cuda.synchronize()
    eq, es = oracle.per_token_group_quant_fp8(w["x"], 128, oracle.UE8M0 if ue8m0 else 0)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), es.view(np.uint32))
    assert np.array_equal(host_u8(q), eq)


@pytest.mark.parametrize("group", [64, 128])
@pytest.mark.parametrize("flags_name", ["div", "recip", "ue8m0"])
def test_group_variants_and_strides(nq, group, flags_name):
    M, K = 77, 1024
    w = S.make_group_inputs(M, K + 64, seed=group)
    f = {"div": nq.FLAG_SCALE_DIV, "recip": 0, "ue8m0": nq.FLAG_UE8M0}[flags_name]
    of = {"div": oracle.DIV, "recip": 0, "ue8m0": oracle.UE8M0}[flags_name]
    xfull = dev_bf16(w["x"])
    for off in (0, 8, 1):  # aligned slice, 16-byte-aligned offset, misaligned (scalar path)
        xs = xfull[:, off:off + K]
        gq = Guarded(M, K, torch.float8_e4m3fn)
        gs = Guarded(M, K // group, torch.float32)
        q, s = nq.nq_per_token_group_quant_fp8(xs, group, q_out=gq.view, scales_out=gs.view, flags=f)
        torch.cuda.synchronize()
        assert gq.guards_intact() and gs.guards_intact()
        eq, es = oracle.per_token_group_quant_fp8(w["x"][:, off:off + K], group, of)
        assert np.array_equal(host_u8(q), eq), off
        assert np.array_equal(s.cpu().numpy().view(np.uint32), es.view(np.uint32)), off


@pytest.mark.parametrize("group", [64, 128])
def test_group_every_team_size(nq, group):
    """Every built (lanes per group, groups per thread) mapping gives the oracle's bits."""
    M, K = 333, 2048
    w = S.make_group_inputs(M, K, seed=group + 11)
    x = dev_bf16(w["x"])
    for flags, of in ((0, 0), (nq.FLAG_UE8M0, oracle.UE8M0), (nq.FLAG_SCALE_DIV, oracle.DIV)):
        eq, es = oracle.per_token_group_quant_fp8(w["x"], group, of)
        for lt in range(1, (5 if group == 128 else 4)):
            for lu in range(0, 3):
                q, s = nq.nq_per_token_group_quant_fp8(x, group, flags=flags | nq.flag_group_schedule(lt, lu))
                assert np.array_equal(host_u8(q), eq), (flags, lt, lu)
                assert np.array_equal(s.cpu().numpy().view(np.uint32), es.view(np.uint32)), (flags, lt, lu)


def test_group_cvt_over_all_bf16_values(nq):
    """Groups whose absmax is 448 have scale 1, so their codes are the hardware
    e4m3 conversion of every finite bf16 value in [-448, 448]: compare with the oracle."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = oracle.bf16_to_f32(bits)
    vals = bits[np.isfinite(f) & (np.abs(f) <= 448)]
    n_per = 127
    G = (len(vals) + n_per - 1) // n_per
    rows = np.zeros((G, 128), np.uint16)
    rows[:, 0] = 0x43E0  # 448.0 in bf16
    flat = np.zeros(G * n_per, np.uint16)
    flat[: len(vals)] = vals
    rows[:, 1:] = flat.reshape(G, n_per)
    q, s = nq.nq_per_token_group_quant_fp8(dev_bf16(rows), 128)
    eq, es = oracle.per_token_group_quant_fp8(rows, 128)
    assert np.all(es == 1.0)
    assert np.array_equal(host_u8(q), eq)


# ------------------------------------------------------------ NVFP4 ----
def run_nvfp4(nq, w, d, g, residual, flags=0, want_norm=False, xoff=0):
    xfull = dev_bf16(w["x"])
    xs = xfull[:, xoff:xoff + d]
    M = xs.shape[0]
    gs = torch.tensor([g], dtype=torch.float32, device="cuda")
    gq = Guarded(M, d // 2, torch.uint8)
    gsf = Guarded(M, d // 16, torch.float8_e4m3fn)
    q, sf, ro, no = nq.nq_rmsnorm_quant_nvfp4(xs, dev_bf16(w["gamma"]), gs, 1e-6,
                                              residual=dev_bf16(w["residual"]) if residual else None,
                                              q_out=gq.view, sf_out=gsf.view, want_norm=want_norm, flags=flags)
    torch.cuda.synchronize()
    assert gq.guards_intact() and gsf.guards_intact()
    return (host_u8(q), host_u8(sf), host_u16(ro) if ro is not None else None,
            host_u16(no) if no is not None else None)


@pytest.mark.parametrize("residual", [False, True])
@pytest.mark.parametrize("M", [1, 64, 8192])
@pytest.mark.parametrize("d", [7168, 1536, 512])
def test_nvfp4_configs_bit_exact(nq, d, M, residual):
    """d in {7168, 1536 (column slice of a [M, 2112] tensor), 512}, M in {1, 64, 8192}."""
    ld = 2112 if d == 1536 else d
    w = S.make_rms_inputs(M, d, seed=0, residual=residual, ld_x=ld)
    g = oracle.nvfp4_global_scale(w["x"], w["gamma"], w.get("residual"), d=d)
    got = run_nvfp4(nq, w, d, g, residual, want_norm=True)
    eq, esf, er, en = oracle.rmsnorm_quant_nvfp4(w["x"], w["gamma"], g, residual=w.get("residual"), d=d,
                                                 want_norm=True)
    assert np.array_equal(got[1], esf), "block scales"
    assert np.array_equal(got[0], eq), "codes"
    assert np.array_equal(got[3], en), "norm_out"
    if residual:
        assert np.array_equal(got[2], er), "residual_out"


@pytest.mark.parametrize("d", [16, 32, 128, 8208, 16384])
def test_nvfp4_every_schedule_and_partial_warps(nq, d):
    """Hidden sizes that leave warps partially active (32, 128, 8208) on every schedule."""
    M = 11
    w = S.make_rms_inputs(M, d, seed=d)
    g = oracle.nvfp4_global_scale(w["x"], w["gamma"], w["residual"])
    exp = oracle.rmsnorm_quant_nvfp4(w["x"], w["gamma"], g, residual=w["residual"])
    for sched in [None, *all_schedules(d)]:
        f = 0 if sched is None else nq.flag_schedule(*sched)
        got = run_nvfp4(nq, w, d, g, True, flags=f)
        assert np.array_equal(got[0], exp[0]) and np.array_equal(got[1], exp[1]), sched
        assert np.array_equal(got[2], exp[2]), sched


def test_nvfp4_div_misaligned_and_bf16_round(nq):
    M, d = 21, 1536
    w = S.make_rms_inputs(M, d, seed=6, residual=False, ld_x=2112)
    g = oracle.nvfp4_global_scale(w["x"][:, 1:1 + d], w["gamma"])
    for flags, oflags in [(nq.FLAG_SCALE_DIV, oracle.DIV), (nq.FLAG_NORM_BF16_ROUND, oracle.NORM_BF16_ROUND)]:
        got = run_nvfp4(nq, w, d, g, False, flags=flags, xoff=1)
        eq, esf, _, _ = oracle.rmsnorm_quant_nvfp4(w["x"][:, 1:1 + d], w["gamma"], g, flags=oflags)
        assert np.array_equal(got[1], esf) and np.array_equal(got[0], eq)


def test_nvfp4_zero_blocks(nq):
    M, d = 3, 64
    w = S.make_rms_inputs(M, d, seed=2, residual=False)
    x = w["x"].copy()
    x[1] = 0
    x[2, :16] = 0
    w["x"] = x
    got = run_nvfp4(nq, w, d, 0.01, False)
    eq, esf, _, _ = oracle.rmsnorm_quant_nvfp4(x, w["gamma"], 0.01)
    assert np.array_equal(got[0], eq) and np.array_equal(got[1], esf)
    assert not got[0][1].any() and not got[1][1].any()


# ------------------------------------------------ kernel variants ----
@pytest.mark.parametrize("d,M,ld", [(512, 3000, 512), (1536, 2000, 2112), (2816, 1500, 2816), (4096, 4096, 4096),
                                    (7168, 700, 7168), (16384, 300, 16384)])
def test_variants_without_residual_bit_exact(nq, d, M, ld):
    """Raw-row and persistent raw-row variants (static RMSNorm, LayerNorm, NVFP4 without residual)
    give the oracle's bits for the default and forced schedules."""
    w = S.make_rms_inputs(M, d, seed=d + 5, residual=False, ld_x=ld, x_outlier_channels=True)
    lw = S.make_ln_inputs(M, d, seed=d + 6)
    x = dev_bf16(w["x"])[:, :d]
    g = dev_bf16(w["gamma"])
    sc = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    gn = oracle.nvfp4_global_scale(w["x"], w["gamma"], d=d)
    gs = torch.tensor([gn], dtype=torch.float32, device="cuda")
    e_st, _, _ = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], 0.05, d=d, eps=1e-6)
    e_ln = oracle.layernorm_quant_fp8(lw["x"], lw["gamma"], lw["beta"], 0.05, eps=1e-6)
    e_fp4 = oracle.rmsnorm_quant_nvfp4(w["x"], w["gamma"], gn, d=d)
    sch = [s for s in all_schedules(d) if s[0] > 5]
    if (d + 7) // 8 <= 512:
        sch.append((5, 4))  # one warp per row, 16 chunks per lane (raw variants only)
    for var in (2, 3):
        for sched in [None] + sch[:2] + sch[-1:]:
            f = nq.flag_variant(var) | (0 if sched is None else nq.flag_schedule(*sched))
            q, _, _ = nq.nq_rmsnorm_quant_fp8_static(x, g, sc, 1e-6, flags=f)
            assert np.array_equal(host_u8(q), e_st), (var, sched)
            q = nq.nq_layernorm_quant_fp8(dev_bf16(lw["x"]), dev_f32(lw["gamma"]), dev_f32(lw["beta"]), sc, 1e-6,
                                          flags=f)
            assert np.array_equal(host_u8(q), e_ln), (var, sched)
            q, sf, _, _ = nq.nq_rmsnorm_quant_nvfp4(x, g, gs, 1e-6, flags=f)
            assert np.array_equal(host_u8(q), e_fp4[0]) and np.array_equal(host_u8(sf), e_fp4[1]), (var, sched)


@pytest.mark.parametrize("d", [10240, 16384])
def test_residual_rows_512_threads(nq, d):
    """Rows of 8193 ... 16384 elements with a residual at M >= 384 run on 512 threads x 4 chunks
    under the two-CTA launch bound (the predicate-free copy at d = 16384, the one that skips
    dead chunk slots at 10240): dynamic, static RMSNorm, NVFP4 and the fused group path,
    bit-exact with the oracle, residual_out included."""
    M = 400
    w = S.make_rms_inputs(M, d, seed=d + 3, x_outlier_channels=True)
    assert nq.nq_query_schedule(0, M, d) == (512, 4, 1)
    assert_fused_equal(run_fused(nq, w), oracle_fused(w))
    x, g = dev_bf16(w["x"]), dev_bf16(w["gamma"])
    sc = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    q, ro, _ = nq.nq_rmsnorm_quant_fp8_static(x, g, sc, 1e-6, residual=dev_bf16(w["residual"]))
    eq, er, _ = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], 0.05, w["residual"])
    assert np.array_equal(host_u8(q), eq) and np.array_equal(host_u16(ro), er)
    gn = oracle.nvfp4_global_scale(w["x"], w["gamma"], w["residual"])
    q4, sf, ro4, _ = nq.nq_rmsnorm_quant_nvfp4(x, g, torch.tensor([gn], dtype=torch.float32, device="cuda"), 1e-6,
                                               residual=dev_bf16(w["residual"]))
    e4, esf, er4, _ = oracle.rmsnorm_quant_nvfp4(w["x"], w["gamma"], gn, w["residual"])
    assert np.array_equal(host_u8(q4), e4) and np.array_equal(host_u8(sf), esf) and np.array_equal(host_u16(ro4), er4)
    qg, sg, rog, _ = nq.nq_rmsnorm_quant_fp8_group(x, g, 1e-6, residual=dev_bf16(w["residual"]))
    eg, esg, erg, _ = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"], w["residual"])
    assert np.array_equal(host_u8(qg), eg) and np.array_equal(host_u16(rog), erg)
    assert np.array_equal(sg.cpu().numpy().view(np.uint32), esg.view(np.uint32))


@pytest.mark.parametrize("M,d", [(1000, 8192), (800, 2816), (1000, 7168), (1000, 4096)])
def test_lean_raw_rows_automatic(nq, M, d):
    """The automatic raw-row kernels of NVFP4 and the fused group path without residual at the
    shapes where they run on their lean register budget (8 chunks per thread at d = 2816, 7168
    and 8192, where ptxas spills a few words; 4 chunks at 4096): bit-exact with the oracle."""
    w = S.make_rms_inputs(M, d, seed=M * 7 + d, residual=False, x_outlier_channels=True)
    x, g = dev_bf16(w["x"]), dev_bf16(w["gamma"])
    gn = oracle.nvfp4_global_scale(w["x"], w["gamma"])
    e4, esf, _, _ = oracle.rmsnorm_quant_nvfp4(w["x"], w["gamma"], gn)
    q4, sf, _, _ = nq.nq_rmsnorm_quant_nvfp4(x, g, torch.tensor([gn], dtype=torch.float32, device="cuda"), 1e-6)
    assert np.array_equal(host_u8(q4), e4) and np.array_equal(host_u8(sf), esf)
    if d % 128 == 0:
        eg, esg, _, _ = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"])
        qg, sg, _, _ = nq.nq_rmsnorm_quant_fp8_group(x, g, 1e-6)
        assert np.array_equal(host_u8(qg), eg)
        assert np.array_equal(sg.cpu().numpy().view(np.uint32), esg.view(np.uint32))


# ------------------------------------- fused RMSNorm + per-token-group FP8 ----
@pytest.mark.parametrize("group", [64, 128])
@pytest.mark.parametrize("residual", [False, True])
@pytest.mark.parametrize("d,M", [(128, 37), (512, 64), (2048, 9), (4096, 300), (7168, 20), (8192, 5)])
def test_rms_group_bit_exact(nq, d, M, residual, group):
    w = S.make_rms_inputs(M, d, seed=d + M, residual=residual, x_outlier_channels=True)
    x, g = dev_bf16(w["x"]), dev_bf16(w["gamma"])
    res = dev_bf16(w["residual"]) if residual else None
    for flags, of in ((0, 0), (nq.FLAG_UE8M0, oracle.UE8M0), (nq.FLAG_SCALE_DIV, oracle.DIV)):
        eq, es, er, en = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"], w.get("residual"), group=group,
                                                        flags=of, want_norm=True)
        gq = Guarded(M, d, torch.float8_e4m3fn)
        gs = Guarded(M, d // group, torch.float32)
        q, s, ro, no = nq.nq_rmsnorm_quant_fp8_group(x, g, 1e-6, group=group, residual=res, q_out=gq.view,
                                                     scales_out=gs.view, want_norm=True, flags=flags)
        torch.cuda.synchronize()
        assert gq.guards_intact() and gs.guards_intact()
        assert np.array_equal(host_u8(q), eq), flags
        assert np.array_equal(s.cpu().numpy().view(np.uint32), es.view(np.uint32)), flags
        assert np.array_equal(host_u16(no), en)
        if residual:
            assert np.array_equal(host_u16(ro), er)


@pytest.mark.parametrize("d", [1024, 4096, 8192])
def test_rms_group_every_schedule_and_variant(nq, d):
    M = 17
    w = S.make_rms_inputs(M, d, seed=d + 3, residual=False)
    x, g = dev_bf16(w["x"]), dev_bf16(w["gamma"])
    eq, es, _, _ = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"])
    scheds = all_schedules(d)
    flags = [nq.flag_schedule(*s_) for s_ in scheds] + [nq.flag_variant(v) for v in (1, 2, 3)]
    if (d + 7) // 8 <= 512:
        flags.append(nq.flag_variant(2) | nq.flag_schedule(5, 4))
    for f in flags:
        q, s, _, _ = nq.nq_rmsnorm_quant_fp8_group(x, g, 1e-6, flags=f)
        assert np.array_equal(host_u8(q), eq), hex(f)
        assert np.array_equal(s.cpu().numpy().view(np.uint32), es.view(np.uint32)), hex(f)


def test_rms_group_misaligned_slice(nq):
    M, d = 19, 1024
    w = S.make_rms_inputs(M, d, seed=8, residual=True, ld_x=d + 8)
    x = dev_bf16(w["x"])[:, 1:1 + d]
    q, s, ro, _ = nq.nq_rmsnorm_quant_fp8_group(x, dev_bf16(w["gamma"]), 1e-6, residual=dev_bf16(w["residual"]))
    eq, es, er, _ = oracle.rmsnorm_quant_fp8_group(w["x"][:, 1:1 + d], w["gamma"], w["residual"])
    assert np.array_equal(host_u8(q), eq) and np.array_equal(host_u16(ro), er)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), es.view(np.uint32))


def test_unbuilt_variants_rejected(nq):
    """Variants 4, 5 and 7 are not built: the call fails on the host and launches nothing."""
    x = torch.zeros(4, 256, dtype=torch.bfloat16, device="cuda")
    g = torch.ones(256, dtype=torch.bfloat16, device="cuda")
    sc = torch.tensor([1.0], dtype=torch.float32, device="cuda")
    for v in (4, 5, 7):
        with pytest.raises(nq.NQError, match="not built"):
            nq.nq_rmsnorm_quant_fp8_static(x, g, sc, 1e-6, flags=nq.flag_variant(v))


@pytest.mark.parametrize("d,M", [(512, 7), (1024, 1), (2816, 301), (4096, 4097), (7168, 64), (16384, 33)])
def test_two_row_variant_every_schedule(nq, d, M):
    """NQ_FLAG_VARIANT(6): two rows per CTA on the same columns (static RMSNorm and LayerNorm),
    every schedule with at least 64 threads, odd and even M."""
    w = S.make_rms_inputs(M, d, seed=d * 3 + M, residual=False, x_outlier_channels=True)
    lw = S.make_ln_inputs(M, d, seed=d * 3 + M + 1)
    x, g = dev_bf16(w["x"]), dev_bf16(w["gamma"])
    sc = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    e_st, _, e_no = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], 0.05, want_norm=True)
    e_ln = oracle.layernorm_quant_fp8(lw["x"], lw["gamma"], lw["beta"], 0.05, eps=1e-6)
    e_div, _, _ = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], 0.05, flags=oracle.DIV)
    lx, lgam, lbet = dev_bf16(lw["x"]), dev_f32(lw["gamma"]), dev_f32(lw["beta"])
    for var, sched in [(v, s_) for v in (6,) for s_ in [None] + [s_ for s_ in all_schedules(d) if s_[0] > 5]]:
        f = nq.flag_variant(var) | (0 if sched is None else nq.flag_schedule(*sched))
        q, _, no = nq.nq_rmsnorm_quant_fp8_static(x, g, sc, 1e-6, want_norm=True, flags=f)
        assert np.array_equal(host_u8(q), e_st) and np.array_equal(host_u16(no), e_no), ("rms", var, sched)
        q, _, _ = nq.nq_rmsnorm_quant_fp8_static(x, g, sc, 1e-6, flags=f | nq.FLAG_SCALE_DIV)
        assert np.array_equal(host_u8(q), e_div), ("rms div", var, sched)
        q = nq.nq_layernorm_quant_fp8(lx, lgam, lbet, sc, 1e-6, flags=f)
        assert np.array_equal(host_u8(q), e_ln), ("ln", var, sched)


# -------------------------------------- rows narrower than the schedule ----
@pytest.mark.parametrize("residual", [False, True])
def test_narrow_rows_partial_warps_every_schedule(nq, residual):
    """Rows narrower than their power-of-two schedule, with a chunk count that is not a multiple
    of 32, so that one warp of a chunk slot is partly inside the row and the warps after it are
    wholly past it (the slots the register-row and raw-row kernels skip).  NVFP4 (d = 2832),
    group 64 (d = 2880) and group 128 (d = 2944), every schedule, bit-exact with the oracle."""
    M = 37
    for d, kind, group in ((2832, "nvfp4", 0), (2880, "group", 64), (2944, "group", 128)):
        assert ((d // 8) % 32) != 0
        w = S.make_rms_inputs(M, d, seed=d + residual, residual=residual, x_outlier_channels=True)
        x, gam = dev_bf16(w["x"]), dev_bf16(w["gamma"])
        res = dev_bf16(w["residual"]) if residual else None
        if kind == "nvfp4":
            g = oracle.nvfp4_global_scale(w["x"], w["gamma"], w.get("residual"), d=d)
            eq, esf, er, _ = oracle.rmsnorm_quant_nvfp4(w["x"], w["gamma"], g, residual=w.get("residual"), d=d)
            gs = torch.tensor([g], dtype=torch.float32, device="cuda")
        else:
            eq, es, er, _ = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"], w.get("residual"), group=group)
        for sched in [None, *all_schedules(d)]:
            f = 0 if sched is None else nq.flag_schedule(*sched)
            if kind == "nvfp4":
                q, sf, ro, _ = nq.nq_rmsnorm_quant_nvfp4(x, gam, gs, 1e-6, residual=res, flags=f)
                assert np.array_equal(host_u8(sf), esf), (d, sched, "block scales")
            else:
                q, s, ro, _ = nq.nq_rmsnorm_quant_fp8_group(x, gam, 1e-6, group=group, residual=res, flags=f)
                assert np.array_equal(s.cpu().numpy().view(np.uint32), es.view(np.uint32)), (d, sched, "scales")
            assert np.array_equal(host_u8(q), eq), (d, sched, "codes")
            if residual:
                assert np.array_equal(host_u16(ro), er), (d, sched, "residual_out")


@pytest.mark.parametrize("M", [700, 1000])
@pytest.mark.parametrize("d", [11264, 12288, 16384])
def test_static_persistent_wide_rows(nq, d, M):
    """Persistent raw rows keep gamma as fp32 in dynamic shared memory (4 d bytes: 44, 48 and
    64 KB here, on top of the kernel's static buffers).  Static RMSNorm, NVFP4 and the fused
    group path without residual, automatic (512 threads x 4 chunks at 700 rows, 256 x 8 at
    1000 rows below 16384 elements) and forced persistent variant, bit-exact with the oracle."""
    w = S.make_rms_inputs(M, d, seed=d + M, residual=False)
    x, gam = dev_bf16(w["x"]), dev_bf16(w["gamma"])
    sc = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    eq, _, _ = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], 0.05)
    g = oracle.nvfp4_global_scale(w["x"], w["gamma"], d=d)
    e4, esf, _, _ = oracle.rmsnorm_quant_nvfp4(w["x"], w["gamma"], g, d=d)
    eg, esg, _, _ = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"])
    gs = torch.tensor([g], dtype=torch.float32, device="cuda")
    for f in (0, nq.flag_variant(3)):
        q, _, _ = nq.nq_rmsnorm_quant_fp8_static(x, gam, sc, 1e-6, flags=f)
        assert np.array_equal(host_u8(q), eq), f
        q4, sf, _, _ = nq.nq_rmsnorm_quant_nvfp4(x, gam, gs, 1e-6, flags=f)
        assert np.array_equal(host_u8(q4), e4) and np.array_equal(host_u8(sf), esf), f
        qg, sg, _, _ = nq.nq_rmsnorm_quant_fp8_group(x, gam, 1e-6, flags=f)
        assert np.array_equal(host_u8(qg), eg) and np.array_equal(sg.cpu().numpy().view(np.uint32),
                                                                 esg.view(np.uint32)), f


@pytest.mark.parametrize("M", [100, 700, 1000])
@pytest.mark.parametrize("d", [8200, 11264, 16384])
def test_layernorm_wide_rows(nq, d, M):
    """LayerNorm rows wider than 8192 elements: raw rows (100 rows); persistent CTAs that keep
    the fp32 gamma and beta in dynamic shared memory (8 d bytes: up to 128 KB) once each CTA
    walks two or more rows (700 rows; 1000 rows of 16384); two rows per CTA at 256 threads x 8
    chunks (1000 rows narrower than 16384).  Automatic and forced persistent, e4m3 and e5m2,
    bit-exact; d = 8200 leaves most chunk slots of the last warps past the row."""
    lw = S.make_ln_inputs(M, d, seed=d + 17)
    x, gl, bl = dev_bf16(lw["x"]), dev_f32(lw["gamma"]), dev_f32(lw["beta"])
    sc = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    e4 = oracle.layernorm_quant_fp8(lw["x"], lw["gamma"], lw["beta"], 0.05, eps=1e-5)
    e5 = oracle.layernorm_quant_fp8(lw["x"], lw["gamma"], lw["beta"], 0.05, eps=1e-5, flags=oracle.E5M2)
    for f in (0, nq.flag_variant(3), nq.flag_variant(3) | nq.FLAG_PDL):
        q = nq.nq_layernorm_quant_fp8(x, gl, bl, sc, 1e-5, flags=f)
        assert np.array_equal(host_u8(q), e4), f
        q = nq.nq_layernorm_quant_fp8(x, gl, bl, sc, 1e-5, flags=f | nq.FLAG_E5M2)
        assert np.array_equal(host_u8(q), e5), f
