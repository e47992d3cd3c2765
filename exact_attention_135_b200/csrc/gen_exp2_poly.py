"""Derive the polynomial used by the kernels' FMA-pipe exp2 (run by hand; the
printed constants are pasted into sm100.cuh).

Method: Cody-Waite style range reduction x = n + f with n = round(x) and
f in [-1/2, 1/2], then 2^x = 2^n * p(f) where p is the degree-`n` polynomial
minimising the maximum RELATIVE error |p(f) - 2^f| / 2^f on [-1/2, 1/2].
The minimax polynomial is found with the Remez exchange algorithm (solve for
an equioscillating error on n+2 reference points, move the points to the
extrema of the new error curve, repeat), then the coefficients are rounded to
fp32 and the error of the rounded polynomial, evaluated in fp32 Horner form,
is reported.

    python exact_attention_135_b200/csrc/gen_exp2_poly.py [degree]
"""

import sys

import numpy as np


def remez_rel(degree: int, a: float = -0.5, b: float = 0.5, iters: int = 30):
    g = lambda x: np.exp2(x)
    m = degree + 2
    # Chebyshev extrema as the first reference set
    k = np.arange(m)
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * k[::-1] / (m - 1))
    coef = None
    for _ in range(iters):
        # p(x_i) - g(x_i) = (-1)^i E g(x_i)  ->  unknowns c_0..c_n, E
        A = np.zeros((m, m))
        for i in range(m):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * g(x[i])
        sol = np.linalg.solve(A, g(x))
        coef = sol[:degree + 1]
        # locate the extrema of the relative error between sign changes
        grid = np.linspace(a, b, 200001)
        err = (np.polyval(coef[::-1], grid) - g(grid)) / g(grid)
        idx = [0]
        for j in range(1, len(grid) - 1):
            if (err[j] - err[j - 1]) * (err[j + 1] - err[j]) <= 0:
                idx.append(j)
        idx.append(len(grid) - 1)
        cand = grid[idx]
        cerr = err[idx]
        # keep alternating extrema with the largest magnitudes
        pts = [0]
        for j in range(1, len(cand)):
            if np.sign(cerr[j]) == np.sign(cerr[pts[-1]]):
                if abs(cerr[j]) > abs(cerr[pts[-1]]):
                    pts[-1] = j
            else:
                pts.append(j)
        while len(pts) > m:
            # drop the smaller end
            if abs(cerr[pts[0]]) < abs(cerr[pts[-1]]):
                pts.pop(0)
            else:
                pts.pop()
        if len(pts) < m:
            break
        x = cand[pts]
    return coef


def fp32_horner_error(coef32, a=-0.5, b=0.5):
    f = np.linspace(a, b, 2000001).astype(np.float32)
    p = np.full_like(f, coef32[-1])
    for c in coef32[-2::-1]:
        p = (p * f + c).astype(np.float32)
    ref = np.exp2(f.astype(np.float64))
    return float(np.max(np.abs(p.astype(np.float64) - ref) / ref))


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    coef = remez_rel(deg)
    c32 = np.array(coef, dtype=np.float32)
    print(f"// degree {deg} minimax (relative) fit of 2^f on [-1/2, 1/2]; "
          f"max rel error in fp32 Horner: {fp32_horner_error(c32):.3e}")
    for i, c in enumerate(c32):
        print(f"constexpr float kExp2C{i} = {float(c):.9e}f;")


if __name__ == "__main__":
    main()
