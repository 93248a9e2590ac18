"""Fit the polynomial used by the kernel's software exp2.

2^x is split as 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2];
2^f is approximated by a polynomial p of low degree whose maximum relative
error |p(f) / 2^f - 1| on [-1/2, 1/2] is minimised (minimax).  The fit is
Lawson's iteratively reweighted least squares on a dense grid, in float64,
followed by a check of the error of the float32 Horner evaluation.

    python -m exact_softmax_attention_02_b200.csrc.fit_exp2 [degree]

prints the coefficients (c0 .. cn, lowest power first) as C literals.
"""

import sys

import numpy as np


def fit(degree: int, iters: int = 400, grid: int = 20001):
    f = np.linspace(-0.5, 0.5, grid)
    target = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / target[:, None]
    b = np.ones_like(f)
    w = np.full(grid, 1.0 / grid)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w /= w.sum()
    rel = np.abs(np.polyval(c[::-1], f) / target - 1).max()
    return c, rel


def float32_error(c, n: int = 1 << 20):
    f = np.linspace(-0.5, 0.5, n).astype(np.float32)
    c32 = c.astype(np.float32)
    acc = np.full_like(f, c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        acc = (acc * f + c32[k]).astype(np.float32)
    return np.abs(acc.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1).max()


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, rel = fit(deg)
    print(f"// degree {deg}: minimax relative error {rel:.3e} (float64), "
          f"{float32_error(c):.3e} (float32 Horner)")
    for k, ck in enumerate(c):
        print(f"constexpr float kExp2C{k} = {float(np.float32(ck)):.9g}f;")
