"""Coefficients of the degree-3 polynomial p(f) ~ 2^f on [-1/2, 1/2] used by the
softmax of hybrid_attn_kernel to evaluate part of its exp2 calls on the FMA pipe.

Method: Cody-Waite range reduction (x = j + f, j = round(x), 2^x = 2^j * 2^f with 2^j
applied to the exponent bits) and a minimax polynomial for 2^f in RELATIVE error,
found with the Remez exchange algorithm on a dense grid (float64). Run:

    python hybrid_sparse_linear_hf_b200/csrc/exp2_poly_fit.py

It prints the coefficients (c0..c3, lowest order first) rounded to fp32 and the
maximum relative error of the fp32-rounded polynomial, which is far below the bf16
rounding (2^-9) applied to P afterwards.
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    # initial reference: Chebyshev extrema
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    f = lambda t: np.exp2(t)  # noqa: E731
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E f(x_i) = f(x_i)  (relative error equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: one extremum of the error per sign run
        sgn = np.sign(err)
        idx = []
        start = 0
        for i in range(1, len(grid) + 1):
            if i == len(grid) or sgn[i] != sgn[start]:
                seg = np.arange(start, i)
                idx.append(seg[np.argmax(np.abs(err[seg]))])
                start = i
        idx = np.array(idx)
        if len(idx) > n:  # keep the n largest alternating extrema
            while len(idx) > n:
                drop = 0 if abs(err[idx[0]]) < abs(err[idx[-1]]) else len(idx) - 1
                idx = np.delete(idx, drop)
        if len(idx) == n:
            x = grid[idx]
    return c


def main():
    c = remez()
    c32 = c.astype(np.float32).astype(np.float64)
    grid = np.linspace(LO, HI, 1000001)
    rel = np.abs(np.polyval(c32[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
    for i, v in enumerate(c.astype(np.float32)):
        print(f"c{i} = {float(v)!r}f  ({v.view(np.uint32):#010x})")
    print(f"max relative error (fp32 coefficients, exact arithmetic): {rel.max():.3e}")


if __name__ == "__main__":
    main()
