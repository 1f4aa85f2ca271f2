"""Derive the exp2 polynomials used by the softmax kernels (run once, offline).

Method: the Remez exchange algorithm for the weighted minimax approximation
of 2^f on [-1/2, 1/2] with weight 2^-f, i.e. minimising the maximum relative
error |p(f) 2^-f - 1|. Combined with round-to-nearest range reduction
x = n + f (n integer, |f| <= 1/2) and an exponent-field add of n, this gives
2^x for the FMA pipe (Cody and Waite's additive range reduction).

    python -m calibrated_block_sparse_b200.csrc.gen_exp2_poly

prints the coefficients (lowest degree first) and the achieved error in
double precision. The kernels evaluate the polynomial in fp32 (Horner).
"""
import numpy as np


def remez(degree, lo=-0.5, hi=0.5, iters=60):
    f = lambda x: np.exp2(x)
    w = lambda x: np.exp2(-x)  # relative error weight
    n = degree + 2
    # Chebyshev extrema as the initial reference
    ref = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    coef, err = None, None
    for _ in range(iters):
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :degree + 1] = x ** np.arange(degree + 1)
            A[i, degree + 1] = (-1) ** i / w(x)
        sol = np.linalg.solve(A, f(ref))
        coef, E = sol[:degree + 1], sol[degree + 1]
        e = (np.polyval(coef[::-1], grid) - f(grid)) * w(grid)
        # new reference: one extremum per sign-alternating run of the error
        sign = np.sign(e)
        idx, start = [], 0
        for i in range(1, len(grid) + 1):
            if i == len(grid) or sign[i] != sign[start]:
                seg = np.arange(start, i)
                idx.append(seg[np.argmax(np.abs(e[seg]))])
                start = i
        idx = np.array(idx)
        while len(idx) > n:  # drop the smallest end extremum
            drop = 0 if abs(e[idx[0]]) < abs(e[idx[-1]]) else -1
            idx = np.delete(idx, drop)
        if len(idx) < n:
            break
        ref = grid[idx]
        err = np.max(np.abs(e))
        if abs(err - abs(E)) < 1e-15 * max(1.0, err):
            break
    return coef, err


if __name__ == "__main__":
    for deg in (3, 4, 5):
        c, e = remez(deg)
        c32 = c.astype(np.float32)
        x = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
        p = np.zeros_like(x)
        for k in range(deg, -1, -1):
            p = (p * x + c32[k]).astype(np.float32)
        e32 = np.max(np.abs(p.astype(np.float64) * np.exp2(-x.astype(np.float64)) - 1))
        print(f"degree {deg}: max rel error {e:.3e} (double), {e32:.3e} (fp32 Horner)")
        print("  coefficients:", ", ".join(f"{float(v):.9e}f" for v in c32))
