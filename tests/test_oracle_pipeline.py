"""Pins of the oracle's norm + quantization pipelines.

What each test ties the oracle to (never to itself):
* golden rows with closed forms (tests/golden/rows.json, canonical_sum.json);
* the canonical sum's error bound against an exact (math.fsum) sum;
* the residual update against torch's float32 add + bf16 cast;
* invariants: the row absmax maps to +-448; NVFP4 block absmax maps to +-6
  when its block scale is a normal unsaturated e4m3; UE8M0 absmax codes land
  in [224, 448]; every non-saturated code is within half an ulp of its input;
* statistics the pages report: fused vs unfused (bf16 double rounding) codes
  differ on a few percent of elements, and the per-token scale by < 0.3%
  (netraruntime blog, "Gating a numerics-changing fusion"); reciprocal vs
  division codes differ by one ulp on a few hundredths of a percent (vLLM
  PR #61343, Overview and the trainer note);
* closed forms: RMS of a constant row, LayerNorm output moments;
* the plain-order (float64) mode stays within the stated tolerance.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf(v):
    return torch.tensor(v, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def e4m3_rank(codes):
    """Signed position of an e4m3 code on the number line (adjacent codes differ by 1; +-0 equal)."""
    c = np.asarray(codes, np.int32)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def e2m1_rank(codes):
    c = np.asarray(codes, np.int32)
    mag = c & 7
    return np.where(c & 8, -mag, mag)


# ------------------------------------------------------------- golden ----
def test_canonical_sum_golden():
    for c in json.load(open(os.path.join(GOLDEN, "canonical_sum.json")))["cases"]:
        got = oracle.canonical_sum(np.array(c["v"], np.float32), c["squares"])
        assert float(got) == c["sum"], c["why"]


def test_canonical_sum_error_bound_and_exact_integers():
    rng = np.random.default_rng(5)
    for n in [1, 7, 8, 9, 100, 2816, 4096, 7168, 16384]:
        v = rng.standard_normal(n).astype(np.float32)
        for sq in (False, True):
            exact = math.fsum((float(a) * float(a) if sq else float(a)) for a in v)
            absum = math.fsum((float(a) * float(a) if sq else abs(float(a))) for a in v)
            levels = 8 + max(1, math.ceil(math.log2(max(1, (n + 7) // 8))))
            bound = levels * 2.0 ** -24 * absum * 1.01
            assert abs(float(oracle.canonical_sum(v, sq)) - exact) <= bound
        ints = rng.integers(-1000, 1000, n).astype(np.float32)
        assert float(oracle.canonical_sum(ints)) == float(ints.astype(np.int64).sum())


def test_golden_rms_dynamic():
    for c in json.load(open(os.path.join(GOLDEN, "rows.json")))["rms_dynamic"]:
        x, res, g = bf([c["x"]]), bf([c["residual"]]), bf(c["gamma"])
        for flags in (0, oracle.DIV, oracle.RECIP):
            q, s, ro, no = oracle.fused_add_rmsnorm_quant_fp8(x, res, g, eps=c["eps"], flags=flags,
                                                              want_norm=True)
            assert list(q[0]) == c["codes"], c["why"]
            assert s[0] == np.float32(c["absmax"]) / np.float32(448.0)
            assert np.array_equal(ro[0], bf(c["residual_out"]))
            assert np.array_equal(no[0], bf(c["y"]))


def test_golden_rms_static_and_ln():
    rows = json.load(open(os.path.join(GOLDEN, "rows.json")))
    for c in rows["rms_static"]:
        for flags in (0, oracle.DIV, oracle.RECIP):
            q, ro, _ = oracle.rmsnorm_quant_fp8_static(bf([c["x"]]), bf(c["gamma"]), c["scale"],
                                                       residual=bf([c["residual"]]), eps=c["eps"],
                                                       flags=flags)
            assert list(q[0]) == c["codes"], c["why"]
    for c in rows["ln_static"]:
        y = oracle.ln_y(bf([c["x"]]), np.array(c["gamma"], np.float32),
                        np.array(c["beta"], np.float32), eps=c["eps"])
        assert list(y[0]) == c["y"]
        for flags in (0, oracle.DIV, oracle.RECIP):
            q = oracle.layernorm_quant_fp8(bf([c["x"]]), np.array(c["gamma"], np.float32),
                                           np.array(c["beta"], np.float32), c["scale"],
                                           eps=c["eps"], flags=flags)
            assert list(q[0]) == c["codes"], c["why"]


def test_golden_nvfp4():
    for c in json.load(open(os.path.join(GOLDEN, "rows.json")))["nvfp4"]:
        q, sf, _, _ = oracle.rmsnorm_quant_nvfp4(bf([c["x"]]), bf(c["gamma"]), c["global_scale"],
                                                 eps=c["eps"])
        assert list(sf[0]) == c["sf"] and list(q[0]) == c["packed"], c["why"]


def test_golden_group():
    for c in json.load(open(os.path.join(GOLDEN, "rows.json")))["group"]:
        row = np.zeros(128, np.float32)
        row[: len(c["x_head"])] = c["x_head"]
        flags = oracle.UE8M0 if c["ue8m0"] else 0
        q, s = oracle.per_token_group_quant_fp8(bf(row[None, :]), 128, flags)
        if "scale" in c:
            assert s[0, 0] == np.float32(c["scale"]), c["why"]
        else:
            assert s[0, 0] == np.float32(max(abs(v) for v in c["x_head"])) / np.float32(448)
        n = len(c["codes_head"])
        assert list(q[0, :n]) == c["codes_head"], c["why"]
        assert not q[0, n:].any()


# ---------------------------------------------------------- residual ----
def test_residual_update_matches_torch():
    w = S.make_rms_inputs(8, 2816)
    _, _, ro, _ = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"])
    xt = torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).float()
    rt = torch.from_numpy(w["residual"].view(np.int16)).view(torch.bfloat16).float()
    exp = (xt + rt).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ro, exp)


# -------------------------------------------------------- invariants ----
@pytest.mark.parametrize("flags", [0, oracle.RECIP])
def test_dynamic_absmax_maps_to_448(flags):
    w = S.make_rms_inputs(64, 2816, x_outlier_channels=True)
    q, s, _, _ = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"], flags=flags)
    y = oracle.rms_y(w["x"], w["gamma"], w["residual"])
    am = np.argmax(np.abs(y), axis=1)
    top = q[np.arange(64), am]
    assert np.all((top == 0x7E) | (top == 0xFE))
    assert np.array_equal(s, (np.abs(y).max(axis=1) / np.float32(448)).astype(np.float32))


def _ulp_e4m3(t):
    a = np.abs(t.astype(np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -30)))
    return np.exp2(np.maximum(e, -6) - 3)


def _ulp_e2m1(t):
    a = np.abs(t.astype(np.float64))
    return np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))


@pytest.mark.parametrize("flags", [oracle.DIV, oracle.RECIP])
def test_dequant_error_bound_dynamic(flags):
    w = S.make_rms_inputs(16, 4096)
    q, s, _, _ = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"], flags=flags)
    y = oracle.rms_y(w["x"], w["gamma"], w["residual"])
    if flags == oracle.DIV:
        t = (y / s[:, None]).astype(np.float32)
    else:
        t = (y * (np.float32(1) / s)[:, None]).astype(np.float32)
    dq = oracle.e4m3_decode(q).astype(np.float64)
    ok = np.abs(t) < 448
    assert np.all(np.abs(t[ok] - dq[ok]) <= 0.5 * _ulp_e4m3(t[ok]))


def test_nvfp4_invariants():
    M, d = 32, 7168
    w = S.make_rms_inputs(M, d)
    g = oracle.nvfp4_global_scale(w["x"], w["gamma"], w["residual"])
    q, sf, _, _ = oracle.rmsnorm_quant_nvfp4(w["x"], w["gamma"], g, residual=w["residual"])
    y = oracle.rms_y(w["x"], w["gamma"], w["residual"])
    codes = oracle.unpack_e2m1(q, d)
    yb = y.reshape(M, d // 16, 16)
    cb = codes.reshape(M, d // 16, 16)
    sfv = oracle.e4m3_decode(sf)
    # block absmax -> +-6 when the block scale is a normal, unsaturated e4m3
    am = np.argmax(np.abs(yb), axis=2)
    top = np.take_along_axis(cb, am[..., None], axis=2)[..., 0]
    normal = (sfv >= 2.0 ** -6) & (sfv < 448)
    assert normal.mean() > 0.99
    assert np.all((top[normal] & 7) == 7)
    # half-ulp bound for every element given its block multiplier
    S_ = (sfv.astype(np.float32) * np.float32(g)).astype(np.float32)
    mult = np.where(S_ == 0, np.float32(0), np.float32(1) / S_).astype(np.float32)
    t = (yb * mult[..., None]).astype(np.float32)
    dq = oracle.e2m1_decode(cb).astype(np.float64)
    ok = np.abs(t) < 6
    assert np.all(np.abs(t[ok] - dq[ok]) <= 0.5 * _ulp_e2m1(t[ok]))
    # sf is the e4m3 of amax / 6 / g
    amax = np.abs(yb).max(axis=2)
    assert np.array_equal(sf, oracle.e4m3_encode((amax / np.float32(6)) / np.float32(g)))


def test_group_ue8m0_absmax_codes_in_range():
    w = S.make_group_inputs(64, 4096)
    q, s = oracle.per_token_group_quant_fp8(w["x"], 128, oracle.UE8M0)
    xs = oracle.bf16_to_f32(w["x"]).reshape(64, 32, 128)
    am = np.argmax(np.abs(xs), axis=2)
    top = np.take_along_axis(q.reshape(64, 32, 128), am[..., None], axis=2)[..., 0]
    dec = np.abs(oracle.e4m3_decode(top))
    assert np.all((dec >= 224) & (dec <= 448))
    m, e = np.frexp(s)
    assert np.all(m == 0.5)  # powers of two


# -------------------------------------------------- page statistics ----
def test_div_vs_recip_statistics():
    """Scales identical; codes differ by <= 1 ulp on a few hundredths of a percent."""
    w = S.make_group_inputs(512, 4096)
    qd, sd = oracle.per_token_group_quant_fp8(w["x"], 128, oracle.DIV)
    qr, sr = oracle.per_token_group_quant_fp8(w["x"], 128, oracle.RECIP)
    assert np.array_equal(sd, sr)
    diff = np.abs(e4m3_rank(qd) - e4m3_rank(qr))
    assert diff.max() <= 1
    frac = (diff > 0).mean()
    assert 1e-4 <= frac <= 2e-3, frac  # pages: ~0.05% (0.03-0.08%)


def test_fused_vs_unfused_statistics():
    """Single rounding vs bf16 double rounding: 2-3% of codes differ, scale within 0.3%."""
    w = S.make_rms_inputs(256, 2816)
    qf, sf_, _, _ = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"])
    qu, su, _, _ = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"],
                                                      flags=oracle.NORM_BF16_ROUND)
    frac = (qf != qu).mean()
    assert 0.015 <= frac <= 0.045, frac
    rel = np.abs(su.astype(np.float64) / sf_ - 1)
    assert rel.max() <= 2.0 ** -8      # bf16 unit roundoff bounds every row
    assert rel.mean() < 0.003           # the page's "under 0.3%" per-token scale error
    assert np.abs(e4m3_rank(qf) - e4m3_rank(qu)).max() <= 1


def test_static_fused_codes_are_nearer():
    w = S.make_rms_inputs(64, 4096, residual=False)
    scale = 0.05
    qf, _, _ = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], scale, eps=1e-5)
    qu, _, _ = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], scale, eps=1e-5,
                                               flags=oracle.NORM_BF16_ROUND)
    y = oracle.rms_y(w["x"], w["gamma"], eps=1e-5)
    t = (y * (np.float32(1) / np.float32(scale))).astype(np.float64)
    dif = qf != qu
    assert dif.any()
    ef = np.abs(oracle.e4m3_decode(qf[dif]) - t[dif])
    eu = np.abs(oracle.e4m3_decode(qu[dif]) - t[dif])
    assert np.all(ef <= eu)


# ------------------------------------------------------- closed forms ----
def test_constant_row_rstd_closed_form():
    for c in [0.5, 1.0, 3.0, -2.0]:
        d = 2816
        x = bf(np.full((1, d), c))
        g = bf(np.ones(d))
        y = oracle.rms_y(x, g, eps=1e-6)
        exact = c / math.sqrt(c * c + 1e-6)
        assert np.all(np.abs(y.astype(np.float64) - exact) <= 4 * 2.0 ** -24 * abs(exact))
        q, s, _, _ = oracle.fused_add_rmsnorm_quant_fp8(x, bf(np.zeros((1, d))), g, eps=1e-6)
        assert np.all(q == (0xFE if c < 0 else 0x7E))


def test_layernorm_moments():
    w = S.make_ln_inputs(16, 4096)
    y = oracle.ln_y(w["x"], np.ones(4096, np.float32), np.zeros(4096, np.float32), eps=1e-5)
    assert np.all(np.abs(y.mean(axis=1)) < 1e-5)
    assert np.all(np.abs((y.astype(np.float64) ** 2).mean(axis=1) - 1) < 1e-4)


def test_plain_order_within_tolerance():
    """The float64 plain-order mode and the canonical order agree within the stated tolerance."""
    w = S.make_rms_inputs(256, 4096, x_outlier_channels=True)
    qa, sa, ra, _ = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"])
    qb, sb, rb, _ = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"],
                                                       flags=oracle.SUM_PLAIN)
    assert np.array_equal(ra, rb)
    assert np.all(np.abs(sa / sb - 1) <= 1e-6)
    diff = np.abs(e4m3_rank(qa) - e4m3_rank(qb))
    assert diff.max() <= 1 and (diff > 0).mean() <= 1e-3


# --------------------------------------------------------- degenerate ----
def test_zero_rows_and_groups():
    d = 64
    x = bf(np.zeros((2, d)))
    q, s, ro, _ = oracle.fused_add_rmsnorm_quant_fp8(x, bf(np.zeros((2, d))), bf(np.ones(d)))
    assert np.all(s == 0) and np.all(q == 0) and np.all(ro == 0)
    q, s = oracle.per_token_group_quant_fp8(bf(np.zeros((1, 256))), 128)
    assert np.all(s == 0) and np.all(q == 0)
    q, sf, _, _ = oracle.rmsnorm_quant_nvfp4(bf(np.zeros((1, 32))), bf(np.ones(32)), 1.0)
    assert np.all(q == 0) and np.all(sf == 0)


def test_static_zero_scale_is_ieee():
    """scale = 0: inverse is +inf, nonzero y saturates to +-448, y = 0 gives 0*inf = NaN."""
    x = bf([[1.0, -1.0, 0.0, 2.0]])
    q, _, _ = oracle.rmsnorm_quant_fp8_static(x, bf([1.0, 1.0, 0.0, 1.0]), 0.0, eps=1e-6)
    assert q[0, 0] == 0x7E and q[0, 1] == 0xFE and q[0, 3] == 0x7E
    assert q[0, 2] & 0x7F == 0x7F


# ------------------------------------------- fused RMSNorm + group FP8 ----
def test_golden_rms_group():
    c = json.load(open(os.path.join(GOLDEN, "rows.json")))["rms_group"][0]
    d = c["d"]
    gamma = np.zeros(d, np.float32)
    gamma[: len(c["gamma_head"])] = c["gamma_head"]
    gamma[128] = c["gamma_at_128"]
    x = bf(np.ones((1, d)))
    for flags in (0, oracle.RECIP, oracle.DIV):
        q, s, _, _ = oracle.rmsnorm_quant_fp8_group(x, bf(gamma), eps=c["eps"], flags=flags)
        assert s[0, 0] == np.float32(c["scales"][0])
        assert s[0, 1] == np.float32(c["gamma_at_128"]) / np.float32(448)
        assert list(q[0, :4]) == c["codes_head"], c["why"]
        assert q[0, 128] == c["code_at_128"]
        assert not q[0, 4:128].any() and not q[0, 129:].any()


@pytest.mark.parametrize("flags", [0, oracle.UE8M0, oracle.DIV])
@pytest.mark.parametrize("residual", [False, True])
def test_rms_group_composes_pinned_pieces(flags, residual):
    """The fused result equals the pinned pieces composed in numpy: y from the
    RMSNorm pin, per-group s = RN(absmax / 448) (or its UE8M0 ceil), the pinned
    e4m3 encoder of RN(y * RN(1 / s)) (or RN(y / s))."""
    M, d, G = 24, 1024, 128
    w = S.make_rms_inputs(M, d, seed=3, residual=residual, x_outlier_channels=True)
    q, s, ro, _ = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"], w.get("residual"), flags=flags)
    y = oracle.rms_y(w["x"], w["gamma"], w.get("residual"))
    yg = y.reshape(M, d // G, G)
    es = (np.abs(yg).max(axis=2) / np.float32(448)).astype(np.float32)
    if flags & oracle.UE8M0:
        es = oracle.ue8m0_ceil(es)
    assert np.array_equal(s, es)
    if flags & oracle.DIV:
        t = (yg / es[..., None]).astype(np.float32)
    else:
        inv = np.where(es == 0, np.float32(0), np.float32(1) / es).astype(np.float32)
        t = (yg * inv[..., None]).astype(np.float32)
    assert np.array_equal(q, oracle.e4m3_encode(t).reshape(M, d))
    if residual:
        _, _, er, _ = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"])
        assert np.array_equal(ro, er)


def test_rms_group_fused_vs_unfused():
    """Quantizing fp32 y vs bf16-rounded y: a few percent of codes move by one ulp."""
    w = S.make_rms_inputs(128, 4096, seed=4)
    qf, sf_, _, _ = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"], w["residual"])
    qu, su, _, _ = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"], w["residual"], flags=oracle.NORM_BF16_ROUND)
    frac = (qf != qu).mean()
    assert 0.01 <= frac <= 0.05
    assert np.abs(e4m3_rank(qf) - e4m3_rank(qu)).max() <= 1


def test_e5m2_outputs_compose_pinned_pieces():
    """With e5m2 output the dynamic scale is absmax / 57344 and the codes are the
    pinned e5m2 encoder of RN(y / s); static and group paths likewise."""
    w = S.make_rms_inputs(16, 1024, seed=21)
    q, s, _, _ = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"], flags=oracle.E5M2)
    y = oracle.rms_y(w["x"], w["gamma"], w["residual"])
    es = (np.abs(y).max(axis=1) / np.float32(57344)).astype(np.float32)
    assert np.array_equal(s, es)
    assert np.array_equal(q, oracle.e5m2_encode((y / es[:, None]).astype(np.float32)))
    top = q[np.arange(16), np.argmax(np.abs(y), axis=1)]
    assert np.all((top & 0x7F) == 0x7B)
    qs, _, _ = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], 0.05, flags=oracle.E5M2)
    y0 = oracle.rms_y(w["x"], w["gamma"])
    assert np.array_equal(qs, oracle.e5m2_encode((y0 * (np.float32(1) / np.float32(0.05))).astype(np.float32)))
    gw = S.make_group_inputs(8, 512, seed=2)
    qg, sg = oracle.per_token_group_quant_fp8(gw["x"], 128, oracle.E5M2)
    xf = oracle.bf16_to_f32(gw["x"]).reshape(8, 4, 128)
    esg = (np.abs(xf).max(axis=2) / np.float32(57344)).astype(np.float32)
    assert np.array_equal(sg, esg)
    inv = (np.float32(1) / esg).astype(np.float32)
    assert np.array_equal(qg, oracle.e5m2_encode((xf * inv[..., None]).astype(np.float32)).reshape(8, 512))


# --------------------------------------------------- MoE dispatch scatter ----
def test_moe_scatter_golden_dispatch():
    """The oracle's MoE dispatch against a dispatch worked by hand
    (tests/golden/moe_dispatch.json: 3 tokens, top-2, one dropped slot, one
    row nobody targets).  A transposed destination index, a gather in place
    of the scatter, or a dropped slot (-1) wrapping to the last row each fail
    it."""
    c = json.load(open(os.path.join(GOLDEN, "moe_dispatch.json")))
    dest = np.array(c["dest"], np.int32)
    q = np.array(c["q"], np.uint8)
    for key, exp_key, dtype in (("scale", "expected_scale", np.float32),
                                ("group_scales", "expected_group_scales", np.float32)):
        qo, so = oracle.moe_scatter(q, np.array(c[key], dtype), dest, c["rows"])
        assert qo.dtype == np.uint8 and qo.shape == (c["rows"], q.shape[1])
        assert np.array_equal(qo, np.array(c["expected_q"], np.uint8))
        assert np.array_equal(so, np.array(c[exp_key], dtype))


def test_moe_scatter_counts_against_routing():
    """Every row the router assigns receives exactly one token's row: rows that
    several slots name cannot occur (the routing is a permutation of the kept
    slots), and each kept slot's row equals its token's row."""
    r = S.make_moe_routing(50, 16, 4, seed=5, drop_p=0.1)
    dest = r["dest"]
    kept = dest[dest >= 0]
    assert len(np.unique(kept)) == len(kept) and kept.max() < r["rows"]
    q = np.arange(50 * 8, dtype=np.uint8).reshape(50, 8) % 251
    s = np.arange(50, dtype=np.float32) + 1
    qo, so = oracle.moe_scatter(q, s, dest, r["rows"])
    for t in range(50):
        for j in range(4):
            if dest[t, j] >= 0:
                assert np.array_equal(qo[dest[t, j]], q[t]) and so[dest[t, j]] == s[t]
    untouched = np.setdiff1d(np.arange(r["rows"]), kept)
    assert not qo[untouched].any() and not so[untouched].any()
