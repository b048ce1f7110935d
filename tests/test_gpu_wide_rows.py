"""Rows wider than 16384 elements (up to NQ_MAX_D = 65536), split over a
thread-block cluster of 4 or 8 CTAs per row, against the oracle (needs a B200).

The row sums cross the cluster through distributed shared memory in the same
canonical order as one CTA would use, so every output is bit-exact with the
oracle's canonical mode: residual_out, norm_out, scales, codes, block scales.
Widths cover both cluster sizes, rows that fill the cluster (d = 32768,
65536), rows narrower than it (whole warps of chunk slots past the row), a
width that is not a multiple of 8 (the scalar path) and a misaligned column
slice.  The plain float64-order tolerance is checked at d = 65536 too.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from gpu_helpers import Guarded, dev_bf16, dev_f32, e4m3_rank, host_u8, host_u16

pytestmark = pytest.mark.gpu

WIDTHS = [16392, 20000, 32768, 32776, 49152, 65536]


@pytest.fixture(scope="module")
def nq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp4_activation_quantization_b200 as nq
    return nq


def test_query_reports_clusters(nq):
    for d, n in ((16384, 0), (16392, 4), (32768, 4), (32776, 8), (65536, 8)):
        t, k, r = nq.nq_query_schedule(nq.OP_RMS_DYN_FP8, 64, d)
        assert (t == 256 * n and k == 4 and r == 1) if n else t <= 1024, (d, t, k, r)


@pytest.mark.parametrize("d", WIDTHS + [65535])
def test_wide_fused_dynamic_bit_exact(nq, d):
    M = 5
    w = S.make_rms_inputs(M, d, seed=d, x_outlier_channels=True)
    gq, gr = Guarded(M, d, torch.float8_e4m3fn), Guarded(M, d, torch.bfloat16)
    gr.view.copy_(dev_bf16(w["residual"]))
    for flags, of in ((0, 0), (nq.FLAG_SCALE_RECIP, oracle.RECIP)):
        gr.view.copy_(dev_bf16(w["residual"]))
        q, s, ro, no = nq.nq_fused_add_rmsnorm_quant_fp8(dev_bf16(w["x"]), gr.view, dev_bf16(w["gamma"]), 1e-6,
                                                         residual_out=gr.view, q_out=gq.view, want_norm=True,
                                                         flags=flags)
        torch.cuda.synchronize()
        assert gq.guards_intact() and gr.guards_intact()
        eq, es, er, en = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"], flags=of,
                                                            want_norm=True)
        assert np.array_equal(host_u16(ro), er), (d, "residual_out (in place)")
        assert np.array_equal(s.cpu().numpy().view(np.uint32), es.view(np.uint32)), (d, "scales")
        assert np.array_equal(host_u8(q), eq), (d, "codes")
        assert np.array_equal(host_u16(no), en), (d, "norm_out")


@pytest.mark.parametrize("d", WIDTHS)
def test_wide_static_and_layernorm_bit_exact(nq, d):
    M = 6
    w = S.make_rms_inputs(M, d, seed=d + 1)
    lw = S.make_ln_inputs(M, d, seed=d + 2)
    sc = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    for residual in (False, True):
        q, ro, _ = nq.nq_rmsnorm_quant_fp8_static(dev_bf16(w["x"]), dev_bf16(w["gamma"]), sc, 1e-5,
                                                  residual=dev_bf16(w["residual"]) if residual else None,
                                                  flags=nq.flag_variant(3))  # a variant is ignored here
        eq, er, _ = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], 0.05, eps=1e-5,
                                                    residual=w["residual"] if residual else None)
        assert np.array_equal(host_u8(q), eq), (d, residual)
        if residual:
            assert np.array_equal(host_u16(ro), er), (d, "residual_out")
    q = nq.nq_layernorm_quant_fp8(dev_bf16(lw["x"]), dev_f32(lw["gamma"]), dev_f32(lw["beta"]), sc, 1e-5)
    assert np.array_equal(host_u8(q), oracle.layernorm_quant_fp8(lw["x"], lw["gamma"], lw["beta"], 0.05, eps=1e-5))
    qe = nq.nq_layernorm_quant_fp8(dev_bf16(lw["x"]), dev_f32(lw["gamma"]), dev_f32(lw["beta"]), sc, 1e-5,
                                   flags=nq.FLAG_E5M2)
    assert np.array_equal(host_u8(qe), oracle.layernorm_quant_fp8(lw["x"], lw["gamma"], lw["beta"], 0.05, eps=1e-5,
                                                                  flags=oracle.E5M2))


@pytest.mark.parametrize("d", [16400, 32768, 40960, 65536])
def test_wide_nvfp4_bit_exact(nq, d):
    M = 4
    for residual in (False, True):
        w = S.make_rms_inputs(M, d, seed=d + 3, residual=residual)
        g = oracle.nvfp4_global_scale(w["x"], w["gamma"], w.get("residual"))
        gs = torch.tensor([g], dtype=torch.float32, device="cuda")
        eq, esf, er, _ = oracle.rmsnorm_quant_nvfp4(w["x"], w["gamma"], g, residual=w.get("residual"))
        res = dev_bf16(w["residual"]) if residual else None
        q, sf, ro, _ = nq.nq_rmsnorm_quant_nvfp4(dev_bf16(w["x"]), dev_bf16(w["gamma"]), gs, 1e-6, residual=res)
        assert np.array_equal(host_u8(sf), esf) and np.array_equal(host_u8(q), eq), (d, residual)
        if residual:
            assert np.array_equal(host_u16(ro), er)
        n = nq.sf_swizzled_size(M, d)
        sw = torch.full((n,), 0x5A, dtype=torch.uint8, device="cuda")
        nq.nq_rmsnorm_quant_nvfp4(dev_bf16(w["x"]), dev_bf16(w["gamma"]), gs, 1e-6, residual=res,
                                  sf_out=sw.view(torch.float8_e4m3fn), flags=nq.FLAG_SF_SWIZZLED)
        assert np.array_equal(sw.cpu().numpy(), oracle.sf_swizzle(esf)), (d, "swizzled, zero padding")


@pytest.mark.parametrize("d", [16512, 32768, 65536])
def test_wide_group_bit_exact(nq, d):
    M = 4
    for residual in (False, True):
        w = S.make_rms_inputs(M, d, seed=d + 4, residual=residual, x_outlier_channels=True)
        res = dev_bf16(w["residual"]) if residual else None
        for group, flags, of in ((128, 0, 0), (64, nq.FLAG_UE8M0, oracle.UE8M0)):
            eq, es, er, _ = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"], w.get("residual"), group=group,
                                                           flags=of)
            q, s, ro, _ = nq.nq_rmsnorm_quant_fp8_group(dev_bf16(w["x"]), dev_bf16(w["gamma"]), 1e-6, group=group,
                                                        residual=res, flags=flags)
            assert np.array_equal(host_u8(q), eq), (d, residual, group)
            assert np.array_equal(s.cpu().numpy().view(np.uint32), es.view(np.uint32)), (d, residual, group)
            if residual:
                assert np.array_equal(host_u16(ro), er)
    # GEMM-ready layout: packed UE8M0 words, column-major
    w = S.make_rms_inputs(M, d, seed=d + 5, residual=False)
    eq, es, _, _ = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"], flags=oracle.UE8M0)
    q, s, _, _ = nq.nq_rmsnorm_quant_fp8_group(dev_bf16(w["x"]), dev_bf16(w["gamma"]), 1e-6,
                                               flags=nq.FLAG_SCALES_PACKED_UE8M0 | nq.FLAG_SCALES_COL_MAJOR)
    assert np.array_equal(host_u8(q), eq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32),
                          oracle.group_scales_layout(es, col_major=True, packed=True).T)


def test_wide_moe_dispatch_bit_exact(nq):
    M, d, E, topk = 9, 32768, 8, 2
    w = S.make_rms_inputs(M, d, seed=77)
    r = S.make_moe_routing(M, E, topk, seed=77)
    dest = torch.from_numpy(r["dest"]).cuda()
    for group in (0, 128):
        qo, so, ro, _ = nq.nq_fused_add_rmsnorm_quant_fp8_moe(dev_bf16(w["x"]), dev_bf16(w["gamma"]), dest,
                                                              r["rows"], 1e-6, group=group,
                                                              residual=dev_bf16(w["residual"]))
        if group == 0:
            eq, es, er, _ = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"])
        else:
            eq, es, er, _ = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"], w["residual"], group=group)
        xq, xs = oracle.moe_scatter(eq, es, r["dest"], r["rows"])
        kept = np.unique(r["dest"][r["dest"] >= 0])
        assert np.array_equal(host_u8(qo)[kept], xq[kept]), group
        assert np.array_equal(so.cpu().numpy()[kept].view(np.uint32), xs[kept].view(np.uint32)), group
        assert np.array_equal(host_u16(ro), er)


def test_wide_misaligned_slice_and_many_rows(nq):
    """A column slice starting one element in (scalar path) and M = 600 rows (600 clusters)."""
    d = 24000
    w = S.make_rms_inputs(3, d, seed=12, ld_x=d + 8)
    x = dev_bf16(w["x"])[:, 1:1 + d]
    q, s, ro, _ = nq.nq_fused_add_rmsnorm_quant_fp8(x, dev_bf16(w["residual"]), dev_bf16(w["gamma"]), 1e-6)
    eq, es, er, _ = oracle.fused_add_rmsnorm_quant_fp8(w["x"][:, 1:1 + d], w["residual"], w["gamma"])
    assert np.array_equal(host_u8(q), eq) and np.array_equal(host_u16(ro), er)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), es.view(np.uint32))
    w = S.make_rms_inputs(600, 40960, seed=13, residual=False)
    sc = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    q, _, _ = nq.nq_rmsnorm_quant_fp8_static(dev_bf16(w["x"]), dev_bf16(w["gamma"]), sc, 1e-6, flags=nq.FLAG_PDL)
    eq, _, _ = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], 0.05)
    assert np.array_equal(host_u8(q), eq)


def test_wide_plain_order_tolerance(nq):
    """d = 65536 against the oracle's float64 sequential sums: scales within 1e-6 relative, codes
    at most 1 ulp apart on at most 0.1 % of elements, residual bit-exact."""
    M, d = 64, 65536
    w = S.make_rms_inputs(M, d, seed=21, x_outlier_channels=True)
    q, s, ro, _ = nq.nq_fused_add_rmsnorm_quant_fp8(dev_bf16(w["x"]), dev_bf16(w["residual"]),
                                                    dev_bf16(w["gamma"]), 1e-6)
    eq, es, er, _ = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"], w["gamma"], flags=oracle.SUM_PLAIN)
    assert np.array_equal(host_u16(ro), er)
    assert np.all(np.abs(s.cpu().numpy().astype(np.float64) / es - 1) <= 1e-6)
    diff = np.abs(e4m3_rank(host_u8(q)) - e4m3_rank(eq))
    assert diff.max() <= 1 and (diff > 0).mean() <= 1e-3


def test_wide_rows_in_a_cuda_graph(nq):
    """Cluster launches captured in a CUDA graph (with programmatic dependent launch) and
    replayed: the static scale is read at execution time, so updating it between replays
    changes the codes, and each replay matches the oracle for the scale it saw."""
    M, d = 7, 30000
    w = S.make_rms_inputs(M, d, seed=31, residual=False)
    x, g = dev_bf16(w["x"]), dev_bf16(w["gamma"])
    sc = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    q = torch.empty(M, d, dtype=torch.float8_e4m3fn, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        nq.nq_rmsnorm_quant_fp8_static(x, g, sc, 1e-6, q_out=q, flags=nq.FLAG_PDL)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        nq.nq_rmsnorm_quant_fp8_static(x, g, sc, 1e-6, q_out=q, flags=nq.FLAG_PDL)
    for scale in (0.05, 0.2, 0.01):
        sc.fill_(scale)
        graph.replay()
        torch.cuda.synchronize()
        eq, _, _ = oracle.rmsnorm_quant_fp8_static(w["x"], w["gamma"], scale)
        assert np.array_equal(host_u8(q), eq), scale
