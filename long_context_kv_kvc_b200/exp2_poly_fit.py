"""Fits the polynomial used by the scoring kernel's software exp2.

2^y = 2^n * 2^f with n = round(y) and f = y - n in [-1/2, 1/2] (Cody-Waite range
reduction).  2^f is approximated by a degree-5 polynomial whose relative error is
equioscillating (Remez exchange algorithm, E. Ya. Remez, 1934), fitted here in double
precision and rounded to binary32.  Prints the coefficients and the measured maximum
relative error of the rounded polynomial evaluated in binary32 Horner form.

    python -m long_context_kv_kvc_b200.exp2_poly_fit
"""
import numpy as np

DEG = 5
LO, HI = -0.5, 0.5


def remez_relative(deg=DEG, lo=LO, hi=HI, iters=30):
    f = lambda x: np.exp2(x)
    # start from Chebyshev extrema
    k = np.arange(deg + 2)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (deg + 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E f(x_i) = f(x_i)   (relative error E)
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(xi)
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        idx = [0]
        sign_change = np.nonzero(np.diff(np.sign(err)))[0]
        bounds = [0] + list(sign_change + 1) + [len(grid)]
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:]) if b1 > b0]
        if len(ext) != deg + 2:
            break
        x = grid[ext]
        del idx
    return c, np.abs(err).max()


def horner32(c32, x32):
    acc = np.float32(c32[-1])
    for ck in c32[-2::-1]:
        acc = np.float32(np.float32(acc * x32) + ck)  # the kernel uses fused FMA; this is a bound
    return acc


if __name__ == "__main__":
    c, e = remez_relative()
    c32 = c.astype(np.float32)
    x = np.linspace(LO, HI, 100001).astype(np.float32)
    approx = np.array([horner32(c32, xi) for xi in x[::10]], dtype=np.float64)
    rel = np.abs(approx - np.exp2(x[::10].astype(np.float64))) / np.exp2(x[::10].astype(np.float64))
    print("double-precision minimax relative error: %.3e" % e)
    print("binary32 coefficients, max relative error on [-1/2, 1/2]: %.3e" % rel.max())
    for i, ci in enumerate(c32):
        print(f"c{i} = {float(ci)!r}f  ({ci.view(np.uint32):#010x})")
