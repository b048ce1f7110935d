"""The C-ABI library without a GPU: it loads, exports every declared symbol,
and its host-side validation and planner answer without touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nq.h")


@pytest.fixture(scope="module")
def nq():
    from fp4_activation_quantization_b200 import build as b
    b.build()
    import fp4_activation_quantization_b200 as nq
    return nq


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nq_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(nq):
    names = declared_functions()
    assert {"nq_fused_add_rmsnorm_quant_fp8", "nq_rmsnorm_quant_fp8_static", "nq_layernorm_quant_fp8",
            "nq_per_token_group_quant_fp8", "nq_rmsnorm_quant_nvfp4"} <= set(names)
    raw = ctypes.CDLL(nq.library_path())
    for n in names:
        assert hasattr(raw, n), n


def test_version_and_strings(nq):
    assert nq.version() >= 100
    assert nq.lib.nq_status_string(0) == b"NQ_OK"
    assert nq.lib.nq_status_string(1) == b"NQ_ERR_INVALID_ARGUMENT"
    assert nq.lib.nq_status_string(2) == b"NQ_ERR_UNSUPPORTED"
    assert nq.lib.nq_status_string(3) == b"NQ_ERR_CUDA"


def test_flag_values_match_header(nq):
    text = open(HEADER).read()
    assert "#define NQ_MAX_D 65536" in text and nq.NQ_MAX_D == 65536
    for name, val in [("NQ_FLAG_PDL", nq.FLAG_PDL), ("NQ_FLAG_SCALE_DIV", nq.FLAG_SCALE_DIV),
                      ("NQ_FLAG_SCALE_RECIP", nq.FLAG_SCALE_RECIP), ("NQ_FLAG_UE8M0", nq.FLAG_UE8M0),
                      ("NQ_FLAG_NORM_BF16_ROUND", nq.FLAG_NORM_BF16_ROUND), ("NQ_FLAG_E5M2", nq.FLAG_E5M2),
                      ("NQ_FLAG_SF_SWIZZLED", nq.FLAG_SF_SWIZZLED),
                      ("NQ_FLAG_SCALES_COL_MAJOR", nq.FLAG_SCALES_COL_MAJOR),
                      ("NQ_FLAG_SCALES_PACKED_UE8M0", nq.FLAG_SCALES_PACKED_UE8M0)]:
        m = re.search(rf"#define {name} \(1u << (\d+)\)", text)
        assert m and (1 << int(m.group(1))) == val, name


FAKE = 0x10000  # a non-null address that validation rejects before any CUDA use


def call_fused(nq, M=4, d=64, x=FAKE, res=FAKE, res_out=FAKE, gamma=FAKE, q=FAKE, s=FAKE, ld_x=None,
               eps=1e-6, flags=0):
    ld_x = d if ld_x is None else ld_x
    return nq.lib.nq_fused_add_rmsnorm_quant_fp8(x, ld_x, res, res_out, d, gamma, q, d, s, None, d, M, d,
                                                 eps, flags, None)


def test_validation_without_gpu(nq):
    INV, UNS = nq.NQ_ERR_INVALID_ARGUMENT, nq.NQ_ERR_UNSUPPORTED
    assert call_fused(nq, x=None) == INV
    assert b"required" in nq.lib.nq_last_error()
    assert call_fused(nq, q=None) == INV
    assert call_fused(nq, s=None) == INV
    assert call_fused(nq, M=-1) == INV
    assert call_fused(nq, d=0) == INV
    assert call_fused(nq, d=65537) == UNS and b"NQ_MAX_D" in nq.lib.nq_last_error()
    # rows wider than 16384 take a cluster per row: a forced schedule cannot cover them
    assert call_fused(nq, d=16392, flags=nq.flag_schedule(10, 1)) == INV
    assert call_fused(nq, ld_x=32) == INV
    assert call_fused(nq, eps=float("nan")) == INV
    assert call_fused(nq, eps=-1.0) == INV
    assert call_fused(nq, flags=nq.FLAG_SCALE_DIV | nq.FLAG_SCALE_RECIP) == INV
    assert call_fused(nq, flags=nq.FLAG_UE8M0) == INV
    assert call_fused(nq, flags=1 << 30) == INV
    # M == 0 is a no-op, even with null pointers
    assert call_fused(nq, M=0, x=None, res=None, res_out=None, gamma=None, q=None, s=None) == nq.NQ_OK
    # schedule too small for the row
    assert call_fused(nq, d=1024, flags=nq.flag_schedule(5, 0)) == INV
    # static: residual pair must be both or neither
    L = nq.lib
    # variants 4, 5 and 7 are not built: rejected on the host, nothing launched
    for v in (4, 5, 7):
        assert L.nq_rmsnorm_quant_fp8_static(FAKE, 64, None, None, 64, FAKE, FAKE, FAKE, 64, None, 64, 4, 64,
                                             1e-6, nq.flag_variant(v), None) == UNS, v
        assert b"not built" in L.nq_last_error()
    assert L.nq_rmsnorm_quant_fp8_static(FAKE, 64, FAKE, None, 64, FAKE, FAKE, FAKE, 64, None, 64, 4, 64,
                                         1e-6, 0, None) == INV
    # NVFP4 needs d % 16 == 0, and has no e5m2 form
    assert L.nq_rmsnorm_quant_nvfp4(FAKE, 24, None, None, 24, FAKE, FAKE, FAKE, 12, FAKE, 1, None, 24, 4, 24,
                                    1e-6, 0, None) == INV
    assert L.nq_rmsnorm_quant_nvfp4(FAKE, 32, None, None, 32, FAKE, FAKE, FAKE, 16, FAKE, 2, None, 32, 4, 32,
                                    1e-6, nq.FLAG_E5M2, None) == INV
    assert b"E5M2" in L.nq_last_error()
    # swizzled block scales: NVFP4 only; the buffer must be 4-byte aligned; ld_sf is not checked
    assert call_fused(nq, flags=nq.FLAG_SF_SWIZZLED) == INV
    assert L.nq_rmsnorm_quant_nvfp4(FAKE, 32, None, None, 32, FAKE, FAKE, FAKE, 16, FAKE + 2, 0, None, 32, 4, 32,
                                    1e-6, nq.FLAG_SF_SWIZZLED, None) == INV
    assert b"4-byte" in L.nq_last_error()
    assert nq.sf_swizzled_size(1, 16) == 128 * 4 and nq.sf_swizzled_size(129, 7168) == 256 * 448
    # MoE dispatch: topk, group and the unsupported flags are checked on the host
    def moe(topk=2, group=0, flags=0, rows=8, dest=FAKE):
        return L.nq_fused_add_rmsnorm_quant_fp8_moe(FAKE, 256, FAKE, FAKE, 256, FAKE, dest, topk, rows, FAKE, 256,
                                                    FAKE, 2, None, 256, 4, 256, group, 1e-6, flags, None)
    assert moe(topk=0) == INV and moe(topk=65) == INV
    assert moe(group=32) == UNS and moe(flags=nq.FLAG_E5M2) == UNS
    assert moe(flags=nq.FLAG_UE8M0) == INV  # UE8M0 needs group scales
    assert moe(dest=None) == INV and moe(rows=-1) == INV
    # group-scale layouts: group calls only; ld_s checked per layout (M = 4, K = 640 -> 5 groups, 2 words)
    assert call_fused(nq, flags=nq.FLAG_SCALES_COL_MAJOR) == INV
    col, packed = nq.FLAG_SCALES_COL_MAJOR, nq.FLAG_SCALES_PACKED_UE8M0
    for flags, ld_ok, ld_bad in ((0, 5, 4), (col, 4, 3), (packed, 2, 1), (col | packed, 4, 3)):
        assert L.nq_per_token_group_quant_fp8(FAKE, 640, FAKE, 640, FAKE, ld_bad, 4, 640, 128, flags,
                                              None) == INV, flags
        assert b"ld_s" in L.nq_last_error()
        assert L.nq_per_token_group_quant_fp8(None, 640, None, 640, None, ld_ok, 0, 640, 128, flags,
                                              None) == nq.NQ_OK, flags
        assert L.nq_rmsnorm_quant_fp8_group(FAKE, 640, None, None, 640, FAKE, FAKE, 640, FAKE, ld_bad, None, 640,
                                            4, 640, 128, 1e-6, flags, None) == INV, flags
    # group: K % group, group size, schedule flag not allowed
    assert L.nq_per_token_group_quant_fp8(FAKE, 200, FAKE, 200, FAKE, 2, 4, 200, 128, 0, None) == INV
    assert L.nq_per_token_group_quant_fp8(FAKE, 96, FAKE, 96, FAKE, 3, 4, 96, 32, 0, None) == UNS
    assert L.nq_per_token_group_quant_fp8(FAKE, 256, FAKE, 256, FAKE, 2, 4, 256, 128,
                                          nq.flag_group_schedule(5, 0), None) == UNS
    assert L.nq_per_token_group_quant_fp8(FAKE, 256, FAKE, 256, FAKE, 2, 4, 256, 128,
                                          nq.flag_variant(2), None) == INV
    assert L.nq_per_token_group_quant_fp8(None, 256, None, 256, None, 2, 0, 256, 128, 0, None) == nq.NQ_OK
    # LayerNorm rejects the bf16 double-rounding flag only when there is no norm: it has one, so fine;
    # it rejects UE8M0
    assert L.nq_layernorm_quant_fp8(FAKE, 64, FAKE, FAKE, FAKE, FAKE, 64, 4, 64, 1e-5, nq.FLAG_UE8M0,
                                    None) == INV


@pytest.mark.parametrize("op,M,d,exp", [
    (0, 64, 2816, (512, 1, 1)),      # fewer rows than SMs: one chunk per thread
    (0, 4096, 4096, (256, 2, 1)),    # residual-add dynamic, d <= 4096: two chunks per thread at any M ...
    (0, 4096, 2816, (128, 4, 1)),    # ... except rows narrower than the 512-chunk schedule: four
    (0, 4096, 2048, (128, 2, 1)),
    (0, 65536, 8192, (256, 4, 1)),   # wider rows: four chunks per thread
    (0, 8192, 7168, (256, 4, 1)),
    (0, 8192, 512, (32, 2, 8)),      # narrow rows: one warp per row, 8 rows per CTA
    (0, 8192, 1536, (128, 2, 1)),
    (0, 1, 8192, (512, 2, 1)),       # a single row: 512 threads with two chunks each ...
    (0, 100, 4096, (512, 1, 1)),     # ... or one
    (0, 16, 16384, (1024, 2, 1)),
    (0, 1, 100, (32, 1, 8)),
    (1, 4096, 4096, (128, 4, 1)),    # static RMSNorm: four chunks once there are many rows per SM
    (1, 600, 4096, (256, 2, 1)),     # ... two below 768 rows
    (1, 160, 4096, (512, 1, 1)),     # ... one below 192 rows
    (1, 300, 7168, (512, 2, 1)),     # two below 384 rows
    (2, 512, 4096, (256, 2, 1)),
    (4, 600, 4096, (128, 4, 1)),     # fused group: four chunks from 384 rows
    (2, 8192, 7168, (128, 8, 1)),    # LayerNorm, P = 1024: eight chunks per thread
    (3, 8192, 7168, (128, 8, 1)),    # NVFP4 without residual, rows narrower than P = 512: eight
    (3, 8192, 2816, (64, 8, 1)),
    (3, 8192, 8192, (128, 8, 1)),    # ... and at P = 1024 whatever the width
    (3, 8192, 4096, (128, 4, 1)),    # ... but four on rows that fill P = 512
    (3, 8192, 1536, (64, 4, 1)),
    # rows of 8193 ... 16384 elements without residual: eight chunks per thread from 768 rows
    (1, 4096, 10240, (256, 8, 1)),
    (2, 4096, 12288, (256, 8, 1)),
    (3, 4096, 12288, (256, 8, 1)),
    (4, 4096, 10240, (256, 8, 1)),
    (2, 700, 12288, (512, 4, 1)),
    (1, 4096, 16384, (256, 8, 1)),   # ... on full rows too for static RMSNorm,
    (3, 4096, 16384, (256, 8, 1)),   # ... and NVFP4 and the fused group from 4096 rows
    (4, 4096, 16384, (256, 8, 1)),
    (3, 1024, 16384, (512, 4, 1)),
    (4, 1024, 16384, (512, 4, 1)),
    (2, 4096, 16384, (512, 4, 1)),
    (0, 4096, 12288, (512, 4, 1)),   # the residual-add path keeps four
])
def test_planner(nq, op, M, d, exp):
    assert nq.nq_query_schedule(op, M, d) == exp


def test_planner_forced_schedules(nq):
    assert nq.nq_query_schedule(0, 100, 4096, nq.flag_schedule(9, 0)) == (512, 1, 1)
    assert nq.nq_query_schedule(3, 100, 1024, nq.flag_schedule(5, 2)) == (32, 4, 8)
    with pytest.raises(nq.NQError):
        nq.nq_query_schedule(0, 100, 4096, nq.flag_schedule(5, 2))   # 32 * 4 * 8 < 4096
    with pytest.raises(nq.NQError):
        nq.nq_query_schedule(0, 100, 64, nq.flag_schedule(10, 2))    # not built (t + k > 11)
    assert nq.nq_query_schedule(0, 100, 8192, nq.flag_schedule(7, 3)) == (128, 8, 1)


def test_planner_cluster_rows(nq):
    """Rows wider than 16384 elements: one cluster of 4 CTAs (up to 32768 elements) or 8 (up to
    65536) of 256 threads with 4 chunks each; the cluster covers the next power of two of chunks.
    A forced schedule cannot cover them."""
    for op in range(5):
        for d in (16400, 20480, 32768, 32784, 49152, 65536):
            T, K, R = nq.nq_query_schedule(op, 4096, d)
            C = (d + 7) // 8
            P = 1 << (C - 1).bit_length()
            assert (T, K, R) == (P // 4, 4, 1) and T in (1024, 2048), (op, d, T, K, R)
    with pytest.raises(nq.NQError):
        nq.nq_query_schedule(0, 100, 20000, nq.flag_schedule(10, 1))
    with pytest.raises(nq.NQError):
        nq.nq_query_schedule(0, 100, 65537)


def test_planner_properties(nq):
    """Over a grid of operations, row counts and widths, the automatic schedule covers the row
    with the fewest chunk slots a power-of-two schedule allows (or one warp with one chunk),
    stays within the built schedules, and puts eight rows in a CTA exactly when a warp owns a
    row."""
    Ms = [1, 16, 100, 147, 148, 191, 192, 383, 384, 767, 768, 4096, 65536]
    ds = [8, 64, 512, 1000, 1024, 1536, 2048, 2816, 4096, 4104, 7168, 8192, 12288, 16384]
    for op in range(5):
        for M in Ms:
            for d in ds:
                if op == 3 and d % 16:
                    continue
                T, K, R = nq.nq_query_schedule(op, M, d)
                C = (d + 7) // 8
                P = 1 << max(0, (C - 1).bit_length())
                assert T & (T - 1) == 0 and 32 <= T <= 1024, (op, M, d, T)
                assert K in (1, 2, 4, 8), (op, M, d, K)
                assert T * K >= C, (op, M, d, T, K)
                assert T * K == max(P, 32), (op, M, d, T, K)
                assert R == (8 if T == 32 else 1), (op, M, d, T, R)
