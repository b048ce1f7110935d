"""The dynamic FP8 path's bounded division RN(y / s) (a correctly rounded
reciprocal of the row scale, then two FMA remainder corrections; Markstein
1990), checked on the device against the correctly rounded quotient of CUDA's
__fdiv_rn, exhaustively over every float32 bit pattern of the dividend (both
signs, scalar and packed forms) for divisors chosen to stress the method.

Contract: bit-exact when |y / s| >= 2^-24; below (where the remainders leave
the normal range), the same sign and a magnitude < 2^-20, so the e4m3 / e5m2
code is the same signed zero.  A host emulation with IEEE fmaf found the
only bitwise differences at |y / s| < 4e-31."""
import struct

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp4_activation_quantization_b200 as nq
    return nq


def f32(bits):
    return struct.unpack("<f", struct.pack("<I", bits))[0]


def divisors():
    one = 0x3F800000
    v = [1.0, 2.0 ** -60, 2.0 ** 100, 6.0, 448.0, 57344.0, 1.0 / 448, 3.0, 7.0, 0.1, 1.0 / 3.0]
    v += [f32(one + k) for k in (1, 2, 3, 0x400000, 0x7FFFFE, 0x7FFFFF)]       # significands near 1 and 2
    v += [f32(one - k) for k in (1, 2)]                                          # just below 1
    v += [f32(0x20000000 + k) for k in (1, 0x7FFFFF)] + [f32(0x6E000000 + 0x555555)]
    rng = np.random.default_rng(5)
    v += list((np.float32(2.0) ** rng.uniform(-59, 99, 16) * rng.uniform(1, 2, 16)).astype(np.float32))
    # row scales as the kernel forms them: RN(amax / 448) for random amax
    amax = rng.uniform(0.5, 20, 8).astype(np.float32)
    v += list((amax / np.float32(448)).astype(np.float32))
    return np.array(v, np.float32)


def test_bounded_division_exhaustive(nq):
    d = torch.from_numpy(divisors()).cuda()
    assert nq.nq_selftest_division(d) == 0


def test_bounded_division_partial_range(nq):
    """A sub-range of dividends; a divisor outside the domain (2^-70) is skipped."""
    d = torch.tensor([3.0, 2.0 ** -70], dtype=torch.float32, device="cuda")
    assert nq.nq_selftest_division(d, a_bits_begin=0x3F800000, count=1 << 20) == 0
