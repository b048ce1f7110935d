"""Norm + FP8 quantization stored straight into a MoE layer's permuted input
(nq_fused_add_rmsnorm_quant_fp8_moe) vs the oracle: the token-order oracle
result (dynamic per-token or per-token-group e4m3), dispatched by the oracle's
scatter to each (token, slot)'s destination row.  Bit-exact; rows no slot
targets stay untouched; an out-of-range destination is skipped and reported."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from gpu_helpers import dev_bf16, host_u8, host_u16

pytestmark = pytest.mark.gpu
SENT = 0x5A


@pytest.fixture(scope="module")
def nq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp4_activation_quantization_b200 as nq
    return nq


def run(nq, w, r, group, residual, want_norm=False, flags=0):
    M, d = w["x"].shape
    rows = r["rows"]
    q = torch.full((rows, d), SENT, dtype=torch.uint8, device="cuda")
    G = 1 if group == 0 else d // group
    s = torch.full((rows, G) if group else (rows,), -7.0, dtype=torch.float32, device="cuda")
    dest = torch.from_numpy(r["dest"]).cuda()
    res = dev_bf16(w["residual"]) if residual else None
    qo, so, ro, no = nq.nq_fused_add_rmsnorm_quant_fp8_moe(
        dev_bf16(w["x"]), dev_bf16(w["gamma"]), dest, rows, 1e-6, group=group, residual=res,
        q_out=q.view(torch.float8_e4m3fn), scales_out=s, want_norm=want_norm, flags=flags)
    torch.cuda.synchronize()
    return (q.cpu().numpy(), s.cpu().numpy(), None if ro is None else host_u16(ro),
            None if no is None else host_u16(no))


def expected(w, r, group, residual, flags=0):
    if group == 0:
        eq, es, er, en = oracle.fused_add_rmsnorm_quant_fp8(w["x"], w["residual"] if residual else
                                                            np.zeros_like(w["x"][:, :w["x"].shape[1]]),
                                                            w["gamma"], flags=flags, want_norm=True)
    else:
        eq, es, er, en = oracle.rmsnorm_quant_fp8_group(w["x"], w["gamma"], w["residual"] if residual else None,
                                                        group=group, flags=flags, want_norm=True)
    qo, so = oracle.moe_scatter(eq, es, r["dest"], r["rows"])
    return qo, so, er, en


@pytest.mark.parametrize("group", [0, 128, 64])
@pytest.mark.parametrize("residual", [True, False])
@pytest.mark.parametrize("M,d,E,topk", [(1, 4096, 8, 2), (37, 2816, 16, 4), (300, 7168, 256, 8),
                                        (64, 512, 64, 8), (1024, 4096, 64, 1)])
def test_moe_dispatch_bit_exact(nq, M, d, E, topk, residual, group):
    if group and d % group:
        pytest.skip("d not a multiple of the group")
    w = S.make_rms_inputs(M, d, seed=M + d + E, residual=True, x_outlier_channels=True)
    r = S.make_moe_routing(M, E, topk, seed=M + E)
    if group == 0 and not residual:
        w["residual"][:] = 0  # a zero residual: the dynamic path's oracle takes one
    got_q, got_s, got_r, got_n = run(nq, w, r, group, residual or group == 0, want_norm=True)
    eq, es, er, en = expected(w, r, group, residual or group == 0)
    assert np.array_equal(got_q, eq.view(np.uint8))
    assert np.array_equal(got_s.view(np.uint32), es.view(np.uint32))
    assert np.array_equal(got_n, en)
    if residual or group == 0:
        assert np.array_equal(got_r, er)


@pytest.mark.parametrize("group", [0, 128])
def test_moe_dropped_slots_leave_rows_untouched(nq, group):
    M, d, E, topk = 500, 4096, 32, 4
    w = S.make_rms_inputs(M, d, seed=9, residual=True)
    r = S.make_moe_routing(M, E, topk, seed=4, drop_p=0.2)
    rows_total = r["rows"] + 50  # spare rows that no slot targets
    r2 = dict(r, rows=rows_total)
    got_q, got_s, _, _ = run(nq, w, r2, group, True)
    eq, es, _, _ = expected(w, r, group, True)
    n = r["rows"]
    assert np.array_equal(got_q[:n], eq.view(np.uint8)[:n])
    assert np.array_equal(got_s[:n].view(np.uint32), es[:n].view(np.uint32))
    assert np.all(got_q[n:] == SENT) and np.all(got_s[n:] == -7.0)


def test_moe_out_of_range_destination_is_skipped_and_reported(nq):
    M, d, E, topk = 64, 1024, 8, 2
    w = S.make_rms_inputs(M, d, seed=2, residual=True)
    r = S.make_moe_routing(M, E, topk, seed=2)
    bad = r["dest"].copy()
    bad[5, 1] = r["rows"] + 1000  # out of range
    nq.nq_check_device_errors()
    got_q, got_s, _, _ = run(nq, w, dict(r, dest=bad), 0, True)
    with pytest.raises(nq.NQError, match="bit 1"):
        nq.nq_check_device_errors()
    eq, es, _, _ = expected(w, r, 0, True)
    ok = np.ones(r["rows"], bool)
    ok[r["dest"][5, 1]] = False  # the slot whose destination was replaced was not written
    assert np.array_equal(got_q[ok], eq.view(np.uint8)[ok])
    assert np.all(got_q[~ok] == SENT)


def test_error_word_seen_from_a_side_stream(nq):
    """A dispatch with an out-of-range destination launched on a non-default
    torch stream, with no synchronization before the check: the check waits
    for every stream of the device, reports bit 1 once, and leaves the word
    clear (the next check passes)."""
    M, d, E, topk = 256, 2048, 16, 4
    w = S.make_rms_inputs(M, d, seed=9, residual=True)
    r = S.make_moe_routing(M, E, topk, seed=9)
    bad = torch.from_numpy(r["dest"].copy())
    bad[M - 1, 0] = r["rows"] + 7
    nq.nq_check_device_errors()
    x, g, res = dev_bf16(w["x"]), dev_bf16(w["gamma"]), dev_bf16(w["residual"])
    dest = bad.cuda()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        for _ in range(20):  # queue work ahead of the reported launch
            nq.nq_fused_add_rmsnorm_quant_fp8(x, res, g, 1e-6)
        nq.nq_fused_add_rmsnorm_quant_fp8_moe(x, g, dest, r["rows"], 1e-6, residual=res)
    with pytest.raises(nq.NQError, match="bit 1"):
        nq.nq_check_device_errors()
    nq.nq_check_device_errors()


def test_moe_ue8m0_and_forced_schedules(nq):
    M, d, E, topk = 129, 4096, 64, 8
    w = S.make_rms_inputs(M, d, seed=5, residual=True)
    r = S.make_moe_routing(M, E, topk, seed=5)
    eq, es, _, _ = expected(w, r, 128, True, flags=oracle.UE8M0)
    for sched in [None, (7, 2), (8, 1), (9, 0)]:
        f = nq.FLAG_UE8M0 | (0 if sched is None else nq.flag_schedule(*sched))
        got_q, got_s, _, _ = run(nq, w, r, 128, True, flags=f)
        assert np.array_equal(got_q, eq.view(np.uint8)), sched
        assert np.array_equal(got_s.view(np.uint32), es.view(np.uint32)), sched
