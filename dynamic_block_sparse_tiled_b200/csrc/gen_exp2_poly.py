"""Coefficients of the polynomial that approximates 2**f on [-1/2, 1/2].

Method: Chebyshev interpolation (interpolate at the Chebyshev nodes of the
first kind, then convert to the monomial basis) of degree 3. For a function
whose (n+1)-th derivative is bounded by M on an interval of half-width h, the
interpolation error is at most M h^(n+1) / (2^n (n+1)!); here M = ln(2)^4 *
2^(1/2), h = 1/2, n = 3, i.e. about 1.1e-4 relative, far below the bf16
rounding (2^-9) applied to P. The kernel combines the polynomial with an
exact exponent add: 2^x = 2^n * 2^f, n = round(x), f = x - n.

Run: python gen_exp2_poly.py   (prints the float32 coefficients, c0 first)
"""
import numpy as np

DEG = 3


def coefficients(deg=DEG):
    k = np.arange(deg + 1)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (deg + 1)))  # Chebyshev nodes on [-1/2, 1/2]
    vals = np.exp2(nodes)
    V = np.vander(nodes, deg + 1, increasing=True)
    return np.linalg.solve(V, vals)


def max_rel_error(c):
    f = np.linspace(-0.5, 0.5, 200001)
    p = np.polyval(c[::-1], f)
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = coefficients()
    c32 = c.astype(np.float32)
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v):.9e}f  (0x{np.float32(v).view(np.uint32):08x})")
    print("max relative error (float64 eval):", max_rel_error(c))
    print("max relative error (float32 coeffs):", max_rel_error(c32.astype(np.float64)))
