"""Minimax polynomial for 2**f on [-1/2, 1/2], relative error.

    python exact_io_aware_80_b200/csrc/gen_exp2_poly.py [degree]

Method: the Remez exchange algorithm (E. Remez, 1934) for the weighted
minimax problem  min_c max_f |p(f) / 2**f - 1|  with p(f) = c0 + c1 f + ... +
cn f^n.  The reference set (n + 2 points) starts at Chebyshev extrema; each
step solves the alternation system  p(x_i) - 2**x_i = (-1)**i E 2**x_i  for
(c0..cn, E), then moves the reference to the alternating extrema of the
error on a dense grid, until E stops changing.  The coefficients are rounded
to fp32 and the error of the rounded polynomial, evaluated in fp32 Horner
form, is reported.  (p(0) = c0 differs from 1 by about E; the kernels round
p to 16 bits, whose spacing below 1 is far larger, so the largest weight of a
row still rounds to exactly 1.)

The kernels evaluate 2**x for x <= 8 as 2**n * p(f): n = round(x) with the
1.5 * 2**23 shifter, f = x - n, and 2**n applied by adding n << 23 to the
bits of p(f).  The printed coefficients are pasted into sm100.cuh.
"""
import sys

import numpy as np


def remez_exp2(deg: int, iters: int = 60):
    a, b = -0.5, 0.5
    m = deg + 2  # unknowns c0..cn and E
    x = 0.5 * (a + b) - 0.5 * (b - a) * np.cos(np.pi * np.arange(m) / (m - 1))
    grid = np.linspace(a, b, 200001)
    E = None
    c = None
    for _ in range(iters):
        A = np.zeros((m, m))
        for k in range(deg + 1):
            A[:, k] = x ** k
        A[:, deg + 1] = -((-1.0) ** np.arange(m)) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** x)
        c, E_new = sol[:deg + 1], sol[deg + 1]
        err = sum(c[k] * grid ** k for k in range(deg + 1)) / 2.0 ** grid - 1.0
        s = np.sign(err)
        s[s == 0] = 1
        cuts = np.flatnonzero(np.diff(s)) + 1
        runs = np.split(np.arange(len(grid)), cuts)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) > m:  # keep the window of m consecutive extrema with the largest minimum
            best, pick = -1.0, None
            for i in range(len(ext) - m + 1):
                w = min(abs(err[j]) for j in ext[i:i + m])
                if w > best:
                    best, pick = w, ext[i:i + m]
            ext = pick
        if len(ext) < m:
            break
        x = grid[np.array(ext)]
        if E is not None and abs(abs(E_new) - abs(E)) < 1e-16:
            E = E_new
            break
        E = E_new
    return c, abs(E)


def fp32_horner_error(c32):
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    p = np.full_like(f, c32[-1])
    for ck in c32[-2::-1]:
        p = (p * f + np.float32(ck)).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0)))


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, E = remez_exp2(deg)
    c32 = [np.float32(v) for v in c]
    print(f"degree {deg}: minimax relative error {E:.3e}; fp32 Horner error {fp32_horner_error(c32):.3e}")
    for k, v in enumerate(c32):
        print(f"  c{k} = {float(v):.9e}f  // 0x{np.float32(v).view(np.uint32):08x}")


if __name__ == "__main__":
    main()
