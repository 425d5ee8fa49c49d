"""Fit the cubic that the prefill kernel uses for 2^f on [-1/2, 1/2].

    python differential_attention_v2_b200/csrc/fit_exp2_poly.py

Remez exchange for the polynomial of degree 3 with the smallest maximum RELATIVE error
|p(f) - 2^f| / 2^f on [-1/2, 1/2]. Prints the coefficients c0..c3 (rounded to fp32) and the
error of fp32 Horner evaluation; the kernel's kExpC0..kExpC3 are these values.
"""
import numpy as np


def remez(deg, a=-0.5, b=0.5, iters=40, grid=200001):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    t = np.linspace(a, b, grid)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * np.exp2(x[i])
        c = np.linalg.solve(A, np.exp2(x))[:deg + 1]
        err = (np.polyval(c[::-1], t) - np.exp2(t)) / np.exp2(t)
        blocks = np.split(np.arange(grid), np.where(np.diff(np.sign(err)) != 0)[0] + 1)
        ext = [blk[np.argmax(np.abs(err[blk]))] for blk in blocks]
        if len(ext) > n:
            ext = sorted(sorted(ext, key=lambda i: -abs(err[i]))[:n])
        if len(ext) == n:
            x = t[ext]
    return c, float(np.max(np.abs(err)))


def horner_f32(c, f):
    p = np.float32(c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + np.float32(c[k])).astype(np.float32)
    return p


if __name__ == "__main__":
    c, e = remez(3)
    c32 = c.astype(np.float32)
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    e32 = np.max(np.abs(horner_f32(c32, f).astype(np.float64) - np.exp2(f.astype(np.float64)))
                 / np.exp2(f.astype(np.float64)))
    print("coefficients c0..c3:", ", ".join(f"{v:.8f}f" for v in c32))
    print(f"minimax relative error {e:.3e}; fp32 Horner {e32:.3e}")
