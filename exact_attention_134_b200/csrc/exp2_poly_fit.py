"""Fits the polynomial the kernels use to evaluate 2^f on the FMA pipe.

Method: Cody–Waite range reduction (W. J. Cody and W. Waite, "Software Manual
for the Elementary Functions", 1980): 2^x = 2^j * 2^f with j = round(x) and
f = x - j in [-1/2, 1/2]; 2^j is applied by adding j to the exponent field.
2^f is approximated by a degree-3 polynomial whose coefficients minimise the
maximum RELATIVE error on [-1/2, 1/2], found here with the Remez exchange
algorithm (E. Ya. Remez, 1934) on a dense grid. The coefficients are rounded
to float32 and the final error is re-measured with float32 Horner evaluation.

    python exact_attention_134_b200/csrc/exp2_poly_fit.py
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez_relative(deg, iters=40):
    x = np.cos(np.linspace(np.pi, 0, deg + 2)) * (HI - LO) / 2 + (HI + LO) / 2
    grid = np.linspace(LO, HI, 200001)
    f = lambda t: np.exp2(t)  # noqa: E731
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i) for coefficients and E
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(xi)
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: alternating extrema of the error
        idx = [0]
        for k in range(1, len(grid) - 1):
            if (err[k] - err[k - 1]) * (err[k + 1] - err[k]) <= 0:
                idx.append(k)
        idx.append(len(grid) - 1)
        ext = grid[idx]
        e = err[idx]
        # keep deg+2 alternating points with the largest |error|
        pts = []
        for xi, ei in zip(ext, e):
            if pts and np.sign(ei) == np.sign(pts[-1][1]):
                if abs(ei) > abs(pts[-1][1]):
                    pts[-1] = (xi, ei)
            else:
                pts.append((xi, ei))
        while len(pts) > deg + 2:
            if abs(pts[0][1]) < abs(pts[-1][1]):
                pts.pop(0)
            else:
                pts.pop()
        if len(pts) == deg + 2:
            x = np.array([p[0] for p in pts])
    return c, np.max(np.abs(err))


def main():
    c, err = remez_relative(DEG)
    c32 = c.astype(np.float32)
    t = np.linspace(LO, HI, 400001).astype(np.float32)
    p = np.float32(c32[DEG])
    for k in range(DEG - 1, -1, -1):
        p = (p * t + c32[k]).astype(np.float32)
    err32 = np.max(np.abs(p.astype(np.float64) / np.exp2(t.astype(np.float64)) - 1))
    print("coefficients c0..c3 (float32):", [float(v) for v in c32])
    print("hex:", [hex(np.float32(v).view(np.uint32)) for v in c32])
    print(f"max relative error: remez {err:.3e}, float32 Horner {err32:.3e}")


if __name__ == "__main__":
    main()
