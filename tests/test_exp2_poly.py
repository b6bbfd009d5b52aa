"""The forward's exp2 on the FMA pipe (ex2_poly in csrc/msa_device.cuh),
restated step by step in float32 on the CPU: range reduction x = n + f with
the 1.5 * 2^23 rounding constant, the cubic for 2^f on [-1/2, 1/2], n added to
the exponent field.  Checked against the mathematical 2^x: relative error
below 1e-4 (the bf16 the weights are stored in carries 2^-9), and exactly 0
below 2^-125."""
import numpy as np

C = [np.float32(0.99992895), np.float32(0.69327623), np.float32(0.24260405), np.float32(0.05508868)]


def f32(x):
    return np.asarray(x, dtype=np.float32)


def fma32(a, b, c):
    # a*b is exact in float64 for float32 operands; one rounding to float32
    return f32(np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64))


def ex2_poly(x):
    x = f32(x)
    xc = np.maximum(x, f32(-125.0))
    r = f32(xc + f32(12582912.0))
    f = f32(xc - f32(r - f32(12582912.0)))
    q = fma32(fma32(fma32(C[3], f, C[2]), f, C[1]), f, C[0])
    bits = (q.view(np.int32).astype(np.int64) + (r.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    y = bits.astype(np.uint32).view(np.float32)
    return np.where(x < -125.0, f32(0.0), y)


def test_relative_error_over_the_weight_range():
    x = f32(np.concatenate([np.linspace(-125.0, 0.0, 400001), -np.logspace(-8, 2, 2001), [0.0, -0.5, -1.5]]))
    y = ex2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_exact_integers_and_underflow():
    n = np.arange(-125, 1)
    y = ex2_poly(n.astype(np.float32)).astype(np.float64)
    assert np.abs(y / np.exp2(n) - 1.0).max() < 1e-4
    assert (ex2_poly(f32([-125.5, -200.0, -np.inf])) == 0.0).all()
