"""Fits the polynomial p(f) ~ 2^f on [-1/2, 1/2] used by the attention kernel's FMA-pipe exp2.

Method: minimax in relative error by the Remez exchange algorithm (degree 5, 6 coefficients),
started from Chebyshev nodes.  Run to print the coefficients as binary32 literals and the
relative error of the binary32 Horner evaluation with fused multiply-adds:

    python precision_quantized_attention_b200/csrc/fit_exp2_poly.py
"""
import numpy as np

DEG = 5
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve sum_j c_j x_i^j - 2^x_i = (-1)^i E 2^x_i  (relative error equioscillation)
        A = np.zeros((n, n))
        A[:, :deg + 1] = x[:, None] ** np.arange(deg + 1)[None, :]
        A[:, deg + 1] = -((-1.0) ** k) * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # new reference: extrema of the error between sign changes
        idx = np.flatnonzero(np.diff(np.sign(err)) != 0)
        edges = np.concatenate([[0], idx + 1, [grid.size]])
        ext = [a + np.argmax(np.abs(err[a:b])) for a, b in zip(edges[:-1], edges[1:]) if b > a]
        if len(ext) != n:
            break
        x = grid[np.array(ext)]
    return c


def horner_f32(c32, f):
    """binary32 Horner with fused multiply-add (product exact in float64, one rounding)."""
    acc = np.full_like(f, c32[-1], dtype=np.float32)
    for ck in c32[-2::-1]:
        acc = (acc.astype(np.float64) * f.astype(np.float64) + np.float64(ck)).astype(np.float32)
    return acc


def main():
    c = remez()
    c32 = c.astype(np.float32)
    f = np.linspace(LO, HI, 1000001).astype(np.float32)
    rel = np.abs(horner_f32(c32, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1)
    for i, ck in enumerate(c32):
        print(f"c{i} = {float(ck).hex()}  ({float(ck):.9e})")
    print(f"max relative error of the binary32 evaluation on [-1/2, 1/2]: {rel.max():.3e}")


if __name__ == "__main__":
    main()
