"""The seeded input generator: deterministic, stream-separated, right distributions."""
import numpy as np

import synthetic as S


def test_splitmix64_reference_values():
    # SplitMix64 with state 0: the first outputs of the published generator
    # (Vigna's splitmix64.c) are 0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F.
    z = np.array([1, 2, 3], dtype=np.uint64) * np.uint64(0x9E3779B97F4A7C15)
    with np.errstate(over="ignore"):
        out = S._mix(z)
    assert [int(v) for v in out] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_deterministic_and_offset_consistent():
    a = S.splitmix64_stream(0, 1, 1000)
    b = S.splitmix64_stream(0, 1, 1000)
    c = S.splitmix64_stream(0, 1, 500, offset=500)
    assert np.array_equal(a, b) and np.array_equal(a[500:], c)
    assert not np.array_equal(a, S.splitmix64_stream(0, 2, 1000))
    assert not np.array_equal(a, S.splitmix64_stream(1, 1, 1000))


def test_normal_moments_and_bf16():
    v = S.normal_f64(0, 7, 400_000)
    assert abs(v.mean()) < 0.01 and abs(v.std() - 1) < 0.01
    b = S.bf16_normal(0, 7, (1000,))
    f = S.bf16_bits_to_f32(b)
    assert np.all(np.abs(f - S.normal_f64(0, 7, 1000)) <= np.abs(f) * 2.0 ** -8 + 1e-30)


def test_workload_recipes():
    w = S.make_rms_inputs(64, 2816)
    assert w["x"].shape == (64, 2816) and w["residual"].shape == (64, 2816)
    g = S.bf16_bits_to_f32(w["gamma"])
    assert abs(g.mean() - 1) < 0.02 and abs(g.std() - 0.1) < 0.02
    w = S.make_rms_inputs(8, 1536, residual=False, ld_x=2112)
    assert w["x"].shape == (8, 2112) and "residual" not in w
    w = S.make_rms_inputs(16, 4096, x_outlier_channels=True)
    xf = np.abs(S.bf16_bits_to_f32(w["x"]))
    big = set(np.argsort(xf.mean(axis=0))[-4:].tolist())
    assert big == set(S.outlier_channels(4096))
    w = S.make_group_inputs(256, 4096)
    xf = np.abs(S.bf16_bits_to_f32(w["x"]))
    frac = (xf > 6).mean()
    assert 0.0004 < frac < 0.0016
    w = S.make_ln_inputs(4, 4096)
    assert w["gamma"].dtype == np.float32 and w["beta"].dtype == np.float32
    assert abs(w["beta"].std() - 0.02) < 0.003
