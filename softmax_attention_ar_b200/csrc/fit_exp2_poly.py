"""Fit the degree-3 polynomial behind exp2_poly() in arl2_device.cuh.

    python softmax_attention_ar_b200/csrc/fit_exp2_poly.py

Remez exchange for the polynomial p(f) ~ 2^f on [-1/2, 1/2] whose relative error
(p(f) - 2^f) / 2^f equioscillates. It prints the float32 coefficients c0..c3 and the
maximum relative error of the float32 polynomial evaluated the way the kernel does
(Horner with fused multiply-adds).
"""
import numpy as np


def remez(deg: int = 3, a: float = -0.5, b: float = 0.5, iters: int = 40):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(a, b, 400001)
    for _ in range(iters):
        y = 2.0 ** x
        A = np.zeros((n, n))
        for i in range(n):
            A[i, : deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * y[i]
        c = np.linalg.solve(A, y)[: deg + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        ext = [0] + [i for i in range(1, len(grid) - 1) if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0]
        ext.append(len(grid) - 1)
        pts = []
        for i in ext:
            if pts and np.sign(err[i]) == np.sign(err[pts[-1]]):
                if abs(err[i]) > abs(err[pts[-1]]):
                    pts[-1] = i
            else:
                pts.append(i)
        while len(pts) > n:
            pts.pop(0 if abs(err[pts[0]]) < abs(err[pts[-1]]) else -1)
        if len(pts) == n:
            x = grid[pts]
    return c


def eval_f32(c, x):
    """The kernel's evaluation: round-to-nearest split, Horner with single-rounding FMAs, exponent add."""
    c = np.asarray(c, dtype=np.float32)
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0))).astype(np.float32)

    def fma(p, q, r):  # fp32 operands: the fp64 product is exact, one rounding of the sum to fp32
        return (p.astype(np.float64) * q + r).astype(np.float32)

    p = fma(fma(fma(np.full_like(f, c[3]), f, c[2]), f, c[1]), f, c[0])
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


if __name__ == "__main__":
    c = remez(3).astype(np.float32)
    xs = np.linspace(-125, 64, 2_000_001, dtype=np.float32)
    rel = np.abs(eval_f32(c, xs).astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1)
    print("c0..c3 =", [float(v) for v in c])
    print(f"max relative error over [-125, 64]: {rel.max():.3e}")
