"""CPU check of the software exp2 used on the FMA pipe in the forward softmax:
the coefficients in sm100.cuh, evaluated exactly as the kernel does (fp32 Horner
after the round-to-nearest split x = n + f), stay within 4e-6 relative error of
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
