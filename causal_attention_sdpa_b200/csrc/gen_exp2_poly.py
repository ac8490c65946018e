"""Fits the polynomial the kernels use to compute 2^f on the FMA pipe.

2^x = 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2].  This script finds
the degree-n polynomial p minimising max |p(f) / 2^f - 1| on that interval with a
Remez exchange (relative-error minimax, weight 2^-f) and prints its coefficients
rounded to float32, lowest order first, with the achieved error.

  python causal_attention_sdpa_b200/csrc/gen_exp2_poly.py [degree]
"""
import sys

import numpy as np


def remez_exp2(n, iters=40):
    a, b = -0.5, 0.5
    # initial reference: Chebyshev extrema
    k = np.arange(n + 2)
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * k[::-1] / (n + 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        f = np.exp2(x)
        # p(x_i) - f_i = (-1)^i E f_i   (relative error equioscillation)
        A = np.zeros((n + 2, n + 2))
        for i in range(n + 2):
            A[i, :n + 1] = x[i] ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * f[i]
        sol = np.linalg.solve(A, f)
        c, E = sol[:n + 1], sol[n + 1]
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        # new reference: extrema of err between sign changes
        idx = []
        s = np.sign(err)
        start = 0
        for i in range(1, len(grid)):
            if s[i] != s[i - 1] and s[i] != 0:
                seg = slice(start, i)
                idx.append(start + int(np.argmax(np.abs(err[seg]))))
                start = i
        idx.append(start + int(np.argmax(np.abs(err[start:]))))
        if len(idx) == n + 2:
            x = grid[idx]
    c32 = np.float32(c)
    err32 = np.polyval(np.float64(c32)[::-1], grid) / np.exp2(grid) - 1.0
    return c32, float(np.max(np.abs(err32)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_exp2(deg)
    print(f"degree {deg}: max relative error {e:.3e}")
    for i, ci in enumerate(c):
        print(f"  c{i} = {float(ci)!r}f  (0x{np.float32(ci).view(np.uint32):08x})")
