"""Fits the polynomial behind the kernels' FMA-pipe exp2.

Method (Cody and Waite range reduction with a minimax polynomial): write
x = n + f with n = round(x) and f in [-1/2, 1/2]; then 2^x = 2^n * 2^f, where
2^n is built directly in the exponent bits and 2^f comes from a degree-5
polynomial P(f) whose relative error is minimised (Remez exchange on the
relative error 2^-f P(f) - 1, starting from Chebyshev nodes).

Prints the coefficients c0..c5 (P(f) = c0 + c1 f + ... + c5 f^5), rounded to
fp32, and the worst relative error of the rounded polynomial evaluated in
fp32 Horner form over a dense grid. Run it to regenerate the constants in
losa_device.cuh:

    python block_sparse_attention_losa_b200/csrc/fit_exp2_poly.py
"""
import numpy as np

DEG = 5
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    # Equioscillation nodes: deg + 2 points.
    k = np.arange(deg + 2)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k / (deg + 1))[::-1]
    for _ in range(iters):
        # Solve P(x_i) - 2^x_i = (-1)^i E * 2^x_i  (relative error E).
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        # New extrema of the relative error.
        g = np.linspace(LO, HI, 200001)
        err = np.polyval(c[::-1], g) / 2.0 ** g - 1.0
        idx = [0]
        for i in range(1, len(g) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(g) - 1)
        idx = np.array(idx)
        if len(idx) >= deg + 2:
            # keep the deg+2 extrema with alternating signs and largest size
            pick = np.argsort(-np.abs(err[idx]))[:deg + 2]
            x = np.sort(g[idx[pick]])
    return c


def fp32_horner(c32, f):
    acc = np.float32(c32[-1])
    for ck in c32[-2::-1]:
        acc = np.float32(acc * f + ck)
    return acc


def main():
    c = remez()
    c32 = c.astype(np.float32)
    f = np.linspace(LO, HI, 400001).astype(np.float32)
    approx = fp32_horner(c32, f).astype(np.float64)
    rel = np.abs(approx / 2.0 ** f.astype(np.float64) - 1.0)
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v)!r}f  # {v.view(np.uint32):#010x}")
    print(f"max relative error (fp32 Horner on [-1/2, 1/2]): {rel.max():.3e}")


if __name__ == "__main__":
    main()
