"""CPU emulation of the attention kernel's FMA-pipe exponential (exp2_poly2 in k_attn_tc.cuh):
x is clamped at -126, n = round(x) is taken from x + 1.5 * 2^23, f = x - n in [-1/2, 1/2],
2^f by the degree-3 polynomial C0 + f (C1 + f (C2 + f C3)) evaluated with fused multiply-adds,
and n is added to the exponent field of the result. Checks the relative error claimed in the
kernel (7.5e-5, below the 2^-9 rounding of P to bf16) over the range the softmax feeds it
(running maximum at most 2^8 below the row maximum, so x <= 8)."""
import numpy as np

C0, C1, C2, C3 = (float.fromhex(h) for h in ("0x1.fff692p-1", "0x1.62f31cp-1", "0x1.f0de20p-3", "0x1.c3f704p-5"))
F32 = np.float32


def _fma(a, b, c):  # one rounding, like fma.rn.f32
    return F32(np.float64(a) * np.float64(b) + np.float64(c))


def exp2_poly(x):
    x = F32(max(F32(x), F32(-126.0)))
    t = F32(x + F32(12582912.0))            # round(x) in the low mantissa bits
    r = F32(t + F32(-12582912.0))           # round(x) as a float
    f = _fma(r, F32(-1.0), x)               # x - round(x), exact
    p = _fma(F32(C3), f, F32(C2))
    p = _fma(p, f, F32(C1))
    p = _fma(p, f, F32(C0))
    n = np.int32(np.array(t, dtype=np.float32).view(np.int32))
    bits = np.array(p, dtype=np.float32).view(np.int32) + np.int32(n << 23)
    return np.array(bits, dtype=np.int32).view(np.float32)[()]


def test_relative_error_over_the_softmax_range():
    """Normal results (x >= -125): relative error of the polynomial itself, 7.5e-5."""
    xs = np.concatenate([np.linspace(-125.0, 8.0, 200001), np.arange(-125, 9) + 0.5,
                         np.arange(-125, 9).astype(np.float64)])
    worst = 0.0
    for x in xs.astype(np.float32):
        got = np.float64(exp2_poly(x))
        ref = np.exp2(np.float64(x))
        worst = max(worst, abs(got / ref - 1.0))
    assert worst <= 7.6e-5, worst
    assert worst < 2.0 ** -9  # below the rounding of P to bf16


def test_tiny_and_masked_weights_stay_negligible():
    """Below -125 the exponent insertion lands at the bottom of the range (weights below 2^-124,
    against a row maximum's weight >= 1): inexact but harmless, never negative, never large.
    A masked key (-inf) is clamped there too."""
    for x in np.linspace(-126.0, -125.0, 2001).astype(np.float32):
        v = exp2_poly(x)
        assert 0.0 < v < 2.0 ** -124
    for x in (-np.inf, -1000.0, -127.0):
        v = exp2_poly(np.float32(x))
        assert 0.0 < v < 2.0 ** -125
