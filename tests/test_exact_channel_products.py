"""The channel-importance products e = |k| * a (k fp16, a fp32) are exact in
fp64: an 11-bit times a 24-bit significand needs at most 35 bits, and the
exponents stay far inside the fp64 range.  Rounding e + acc once is then the
same whether e is formed first (the oracle) or fused into the add (the
channel-selection kernel's fused multiply-adds)."""
from fractions import Fraction

import numpy as np


def test_fp16_times_fp32_is_exact_in_fp64():
    rng = np.random.default_rng(3)
    k = rng.standard_normal(20000).astype(np.float16)
    a = np.abs(rng.standard_normal(20000)).astype(np.float32)
    # extremes: largest and smallest (subnormal) fp16, tiny and huge fp32
    k = np.concatenate([k, np.array([65504, 6.0e-8, 2.0 ** -24, 1.0], dtype=np.float16)])
    a = np.concatenate([a, np.array([3.0e38, 1.0e-45, 1.17549435e-38, 0.3], dtype=np.float32)])
    for kk, aa in zip(np.abs(k).tolist(), a.tolist()):
        prod = float(kk) * float(aa)
        assert Fraction(prod) == Fraction(kk) * Fraction(aa)
