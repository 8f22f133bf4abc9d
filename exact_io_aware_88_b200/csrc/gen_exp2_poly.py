"""Generates the polynomial used by the kernels' software exp2 (ptx.cuh, exp2_poly).

Method: Cody-Waite style range reduction x = n + f with n = round(x) and f in [-1/2, 1/2],
so 2^x = 2^n * 2^f; 2^f is approximated by the degree-3 polynomial p that minimises the
maximum RELATIVE error max |p(f) / 2^f - 1| on [-1/2, 1/2] (minimax, found with the Remez
exchange algorithm below); 2^n is applied by adding n to the exponent field.

The coefficients are rounded to fp32 and the fp32 error of Horner evaluation is checked on a
dense grid.  Run:  python gen_exp2_poly.py   (prints the C constants and the error bound).
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, lo=LO, hi=HI, iters=30):
    # Initial reference: Chebyshev extrema.
    k = np.arange(deg + 2)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (deg + 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # Solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  (relative equioscillation).
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(A, 2.0 ** x)
        c, E = sol[:deg + 1], sol[deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # New reference: extrema of the error between sign changes.
        s = np.sign(err)
        idx = np.where(np.diff(s) != 0)[0]
        bounds = np.concatenate([[0], idx + 1, [len(grid)]])
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        if len(ext) != deg + 2:
            break
        x = grid[ext]
    return c, abs(E)


def fp32_horner_error(c):
    c32 = np.array(c, dtype=np.float32)
    f = np.linspace(LO, HI, 2000001).astype(np.float32)
    p = c32[3]
    for k in (2, 1, 0):
        p = (p * f + c32[k]).astype(np.float32)
    return np.max(np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0))


if __name__ == "__main__":
    c, E = remez()
    print(f"// minimax relative error (exact coefficients): {E:.3e}")
    print(f"// fp32 Horner relative error on [-1/2, 1/2]:    {fp32_horner_error(c):.3e}")
    for k, v in enumerate(c):
        print(f"constexpr float kExp2C{k} = {float(np.float32(v)):.9g}f;")
