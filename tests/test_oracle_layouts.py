"""Pins of the oracle's GEMM-ready scale layouts, from their definitions read
in memory order (not from the oracle's index formula).

* Swizzled NVFP4 block scales (the 128 x 4 scale-factor tile of block-scaled
  tensor-core GEMMs, public PTX ISA / cuBLAS documentation): memory is a
  sequence of 512-byte tiles, row tiles outer, column tiles inner; a tile's
  bytes run over 32 row lanes, then 4 row quarters, then 4 columns.  The
  expected buffer is built by walking memory in that order.
* Group scales: the column-major layout is the transpose; a packed UE8M0 word
  decodes, byte by byte, to 2^(byte - 127) = the scale of consecutive groups.
"""
import numpy as np
import pytest

import oracle


def swizzled_by_walking_memory(sf: np.ndarray) -> np.ndarray:
    rows, n = sf.shape
    out = []
    for rt in range(-(-rows // 128)):
        for ct in range(-(-n // 4)):
            for lane in range(32):
                for quarter in range(4):
                    for col in range(4):
                        r, c = rt * 128 + quarter * 32 + lane, ct * 4 + col
                        out.append(int(sf[r, c]) if (r < rows and c < n) else 0)
    return np.array(out, np.uint8)


@pytest.mark.parametrize("rows,n", [(1, 1), (1, 7), (31, 4), (127, 4), (128, 4), (129, 5), (300, 112), (256, 8)])
def test_sf_swizzle_matches_memory_walk(rows, n):
    rng = np.random.default_rng(rows * 1000 + n)
    sf = rng.integers(1, 256, size=(rows, n), dtype=np.uint8)  # nonzero: padding is the only zero
    got = oracle.sf_swizzle(sf)
    assert got.size == (-(-rows // 128) * 128) * (-(-n // 4) * 4)
    assert np.array_equal(got, swizzled_by_walking_memory(sf))
    # every scale appears exactly once; everything else is zero padding
    assert np.count_nonzero(got) == rows * n
    assert np.array_equal(np.sort(got[got != 0]), np.sort(sf.ravel()))


def test_sf_swizzle_known_positions():
    sf = np.zeros((256, 8), np.uint8)
    sf[0, 0], sf[1, 0], sf[32, 0], sf[0, 1], sf[0, 4], sf[128, 0], sf[127, 3] = 1, 2, 3, 4, 5, 6, 7
    out = oracle.sf_swizzle(sf)
    # (row 0, col 0) first; next row 16 bytes on; row 32 one word on; col 1 next byte;
    # col 4 in the next tile; row 128 after a row tile of two column tiles; row 127 col 3 = last byte of tile 0
    assert out[0] == 1 and out[16] == 2 and out[4] == 3 and out[1] == 4
    assert out[512] == 5 and out[1024] == 6 and out[511] == 7


@pytest.mark.parametrize("M,G", [(1, 1), (5, 3), (7, 32), (64, 56), (33, 57)])
def test_group_scales_layouts(M, G):
    rng = np.random.default_rng(M * 100 + G)
    e = rng.integers(-127, 128, size=(M, G))
    s = np.ldexp(np.float32(1), e).astype(np.float32)
    assert np.array_equal(oracle.group_scales_layout(s), s)
    cm = oracle.group_scales_layout(s, col_major=True, ld=M + 3)
    assert cm.shape == (G, M + 3) and np.array_equal(cm[:, :M], s.T) and not cm[:, M:].any()
    W = -(-G // 4)
    for col_major in (False, True):
        p = oracle.group_scales_layout(s, col_major=col_major, packed=True)
        words = p.T if col_major else p
        assert words.shape == (M, W)
        b = np.ascontiguousarray(words).view(np.uint8).reshape(M, 4 * W).astype(np.int64)  # little-endian bytes
        assert np.array_equal(np.ldexp(1.0, b[:, :G] - 127), s.astype(np.float64))
        assert not b[:, G:].any()


def test_group_scales_packed_rejects_non_power_of_two():
    with pytest.raises(ValueError):
        oracle.group_scales_layout(np.array([[0.75]], np.float32), packed=True)
    with pytest.raises(ValueError):
        oracle.group_scales_layout(np.array([[0.0]], np.float32), packed=True)
