"""Fits the polynomial the prefill kernel uses to compute part of its exp2 on the FMA pipe.

Method (range reduction in the style of Cody and Waite, then a minimax fit):
  x = n + f with n = round-to-nearest(x) and f in [-1/2, 1/2];
  2^x = 2^n * p(f), where p is the degree-3 polynomial minimising the maximum
  relative error |p(f) / 2^f - 1| on [-1/2, 1/2], found with the Remez exchange
  algorithm below; 2^n is applied by adding n to the float's exponent field.

    python paged_attention_varlen_b200/csrc/exp2_poly_fit.py

prints the coefficients (c0 + c1 f + c2 f^2 + c3 f^3) as float32 literals and
the maximum relative error of the float32 evaluation in the kernel's order.
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    # relative-error minimax: find c, E with (p(x_i) - 2^x_i) / 2^x_i = (-1)^i E at deg+2 points
    k = np.arange(deg + 2)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (deg + 1 - k) / (deg + 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1) / 2.0 ** xi
            A[i, deg + 1] = (-1) ** i
        sol = np.linalg.solve(A, np.ones(deg + 2))
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference points: the extrema of err between its sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        ext = sorted(idx, key=lambda i: -abs(err[i]))
        pts = []
        for i in sorted(ext[: 4 * (deg + 2)]):
            if not pts or np.sign(err[i]) != np.sign(err[pts[-1]]):
                pts.append(i)
            elif abs(err[i]) > abs(err[pts[-1]]):
                pts[-1] = i
        if len(pts) < deg + 2:
            break
        # keep the deg+2 alternating points with the largest errors
        while len(pts) > deg + 2:
            if abs(err[pts[0]]) < abs(err[pts[-1]]):
                pts.pop(0)
            else:
                pts.pop()
        x = grid[pts]
    return c


def eval_f32(c, x):
    """The kernel's evaluation order in float32: rounding shifter, Horner, exponent add."""
    x = np.maximum(np.float32(x), np.float32(-127.0))
    shifter = np.float32(12582912.0)  # 1.5 * 2^23: adding it rounds to an integer in the low mantissa bits
    t = (x + shifter).astype(np.float32)
    n = (t - shifter).astype(np.float32)
    f = (x - n).astype(np.float32)
    c = c.astype(np.float32)
    p = c[3]
    p = (p * f + c[2]).astype(np.float32)
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


if __name__ == "__main__":
    c = remez()
    print("coefficients:", ", ".join(f"{np.float32(v).item():.9e}f" for v in c))
    xs = np.linspace(-60.0, 8.0, 2_000_001).astype(np.float32)
    rel = np.abs(eval_f32(c, xs).astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1.0)
    print(f"max relative error of the float32 evaluation on [-60, 8]: {rel.max():.3e}")
