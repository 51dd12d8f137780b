"""Coefficients of the software 2^x the attention softmax uses for part of its
elements (to share the work of the hardware exp unit with the FMA pipes).

Method: Cody-Waite range reduction x = n + f with n = rint(x), f in [-1/2, 1/2], then
2^f from a cubic p(f) fitted by weighted least squares on Chebyshev nodes of
[-1/2, 1/2] with weight 2^-f (minimising relative error: a near-minimax fit), with
p(0) = 1 imposed; finally 2^x = p(f) * 2^n by adding n to the exponent field.

The attention rounds every probability to bf16 (relative step 2^-8), so a relative
error of a few 1e-4 is below its resolution.  Run this file to print the constants
embedded in attn.cu (kExp2C1..C3).
"""
import numpy as np


def coefficients(degree: int = 3, nodes: int = 2001):
    k = np.arange(nodes)
    f = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * nodes))       # Chebyshev nodes in [-1/2, 1/2]
    target = np.exp2(f)
    w = 1.0 / target                                          # relative error
    # p(f) = 1 + c1 f + c2 f^2 + c3 f^3: fit (2^f - 1) with the monomials f..f^degree.
    A = np.stack([f ** j for j in range(1, degree + 1)], axis=1) * w[:, None]
    b = (target - 1.0) * w
    c, *_ = np.linalg.lstsq(A, b, rcond=None)
    return [1.0] + [float(x) for x in c]


def evaluate_f32(x, coef):
    """The device algorithm in float32 arithmetic (same operation order)."""
    x = np.maximum(np.float32(x), np.float32(-127.0)).astype(np.float32)
    magic = np.float32(12582912.0)                            # 1.5 * 2^23
    t = (x + magic).astype(np.float32)
    n_bits = t.view(np.int32)
    r = (x - (t - magic)).astype(np.float32)
    c = [np.float32(v) for v in coef]
    p = np.float32(c[3])
    p = (p * r + c[2]).astype(np.float32)
    p = (p * r + c[1]).astype(np.float32)
    p = (p * r + c[0]).astype(np.float32)
    bits = (p.view(np.int32).astype(np.int64) + (n_bits.astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    coef = coefficients()
    for j, v in enumerate(coef[1:], 1):
        print(f"constexpr float kExp2C{j} = {np.format_float_positional(np.float32(v))}f;")
    xs = np.linspace(-30, 8, 400001, dtype=np.float32)
    rel = np.abs(evaluate_f32(xs, coef).astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1)
    print("max relative error on [-30, 8]:", rel.max())
