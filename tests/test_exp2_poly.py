"""CPU check of the software exp2 used on the FMA pipe in the forward softmax:
the coefficients in sm100.cuh are the degree-4 polynomial interpolating 2^f at
the five Chebyshev nodes of [-1/2, 1/2] (derived here again in fp64 and
rounded to fp32), and, evaluated exactly as the kernel does (fp32 Horner after
the round-to-nearest split x = n + f), they stay within 4e-6 relative error of
2^x over the range the kernel feeds it, and the clamp keeps x >= -125."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "exact_attention_114_b200", "csrc", "sm100.cuh")


def coeffs():
    text = open(HDR, encoding="utf-8").read()
    c = [float(re.search(rf"kExp2P{i} = ([0-9.eE+-]+)f", text).group(1)) for i in range(5)]
    return np.array(c, dtype=np.float32)


def chebyshev_interpolant():
    """Coefficients (constant term first) of the degree-4 polynomial through
    (t_k, 2^t_k) at the Chebyshev nodes t_k = cos((2k + 1) pi / 10) / 2 of
    [-1/2, 1/2], k = 0..4, solved in fp64 from the Vandermonde system."""
    t = 0.5 * np.cos((2 * np.arange(5) + 1) * np.pi / 10)
    return np.linalg.solve(np.vander(t, 5, increasing=True), np.exp2(t))


def test_coefficients_are_the_chebyshev_interpolant():
    c = chebyshev_interpolant()
    # the middle node is t = 0, so the constant term is exactly 2^0 = 1
    assert abs(c[0] - 1.0) < 1e-15
    assert np.array_equal(c.astype(np.float32), coeffs()), (c, coeffs())
    # the fp64 interpolant itself is within the interpolation-error bound
    # max|(2^t)^(5)| / (5! 2^4) * (1/2)^5 = ln(2)^5 sqrt(2) / (120 * 16 * 32) on [-1/2, 1/2]
    t = np.linspace(-0.5, 0.5, 100_001)
    err = np.abs(np.polyval(c[::-1], t) - np.exp2(t)).max()
    assert err <= np.log(2) ** 5 * np.sqrt(2) / (120 * 16 * 32)


def exp2_like_kernel(x):
    c = coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = np.float32(c[4])
    for ci in c[3::-1]:
        q = (q * f + ci).astype(np.float32)
    bits = q.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_over_kernel_range():
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float64).astype(np.float32)
    y = exp2_like_kernel(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 4e-6, rel.max()


def test_clamp_and_integers():
    assert exp2_like_kernel(np.array([-1000.0], np.float32))[0] == np.float32(2.0 ** -125) * \
        np.float32(1.0) or abs(exp2_like_kernel(np.array([-1000.0], np.float32))[0] / 2.0 ** -125 - 1) < 4e-6
    ints = np.arange(-125, 9, dtype=np.float32)
    y = exp2_like_kernel(ints).astype(np.float64)
    assert np.max(np.abs(y / np.exp2(ints.astype(np.float64)) - 1)) < 4e-6
