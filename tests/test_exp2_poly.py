"""The FMA-pipe exponential used for part of the softmax (csrc/common.cuh, exp2_fma).

Replays its exact fp32 step sequence in NumPy (round-to-nearest via 1.5*2^23,
Cody-Waite split, cubic in Horner form with fp32 fused multiply-adds emulated by
an fp64 product rounded once) and checks the relative error against 2^x over
the range the softmax feeds it (the lazy rescale keeps x <= 8; masked keys never
reach it).  Bound: 1e-4 relative, below bf16 rounding of P (2^-9).
"""
import numpy as np

C = [np.float32(v) for v in (0.9999280572, 0.6932609677, 0.2426111251, 0.0551716685)]


def fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def exp2_fma(x):
    x = np.maximum(np.float32(x), np.float32(-126.0))
    t = np.float32(x + np.float32(12582912.0))
    f = np.float32(x - np.float32(t - np.float32(12582912.0)))
    p = fma32(fma32(fma32(C[3], f, C[2]), f, C[1]), f, C[0])
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return np.uint32(bits).view(np.float32)


def test_relative_error_over_softmax_range():
    xs = np.concatenate([np.linspace(-120, 8, 400001), np.arange(-20, 9, 0.5), -np.logspace(-8, 2, 1001)])
    got = np.array([exp2_fma(np.float32(v)) for v in xs.astype(np.float32)], dtype=np.float64)
    ref = np.exp2(xs.astype(np.float32).astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4, rel.max()


def test_exact_at_integers():
    for n in range(-100, 9):
        assert abs(float(exp2_fma(np.float32(n))) / 2.0 ** n - 1) < 1e-4
