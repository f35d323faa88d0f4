"""The FMA-pipe exp2 of the scoring epilogues (csrc/common.cuh: exp2_fma,
and exp2_fma2, the same steps on packed pairs with the same coefficients),
replayed step by step in numpy float32 (each multiply-add rounded once, as a
fused multiply-add is) and compared with the exact 2^x: relative error at
most 3e-7 on [-126, 0], the same order as the hardware approximation it
shares the work with (the kernels' score tolerance is 1e-4)."""
import re
import os

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coeffs():
    with open(os.path.join(ROOT, "kv_cache_compression_kv2d_b200", "csrc", "common.cuh")) as f:
        src = f.read()
    vals = [float(re.search(r"constexpr float kExp2P%d = ([0-9]\.[0-9]+e[-+][0-9]+)f;" % k, src).group(1))
            for k in range(5, -1, -1)]
    return np.float32(vals[0]), [np.float32(v) for v in vals[1:]]


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_fma_replay(x):
    top, rest = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    shifter = np.float32(12582912.0)
    t = (x + shifter).astype(np.float32)
    f = (x - (t - shifter).astype(np.float32)).astype(np.float32)
    p = np.full(x.shape, top, dtype=np.float32)
    for c in rest:
        p = _fma32(p, f, np.full(x.shape, c, dtype=np.float32))
    n = t.view(np.int32) - np.int32(0x4B400000)
    return (p.view(np.int32) + (n << 23)).view(np.float32)


def test_exp2_fma_relative_error():
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-126.0, 0.0, 2_000_001), -rng.exponential(4.0, 1_000_000),
                        np.array([0.0, -0.5, -1.5, -125.5, -126.0])]).astype(np.float32)
    got = exp2_fma_replay(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 3e-7, rel.max()


def test_exp2_fma_integer_points_exact_enough():
    x = np.arange(-126, 1, dtype=np.float32)
    got = exp2_fma_replay(x).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(x.astype(np.float64)) - 1) < 3e-7)
