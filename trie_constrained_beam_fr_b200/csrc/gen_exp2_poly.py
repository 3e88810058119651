"""Coefficients of the polynomial exp2 used on the FMA pipe in fr_step.cu.

2^y = 2^n * 2^f with n = round(y) and f = y - n in [-1/2, 1/2] (Cody & Waite
range reduction: "Software Manual for the Elementary Functions", 1980).  2^f
is approximated by a degree-5 polynomial whose *relative* error is
equioscillating (minimax), found here with the Remez exchange algorithm in
double precision.  The coefficients are rounded to float32, then the rounded
polynomial's error is measured on a dense grid.

    python trie_constrained_beam_fr_b200/csrc/gen_exp2_poly.py
prints the coefficients (c0..c5) and the max relative error.
"""
import numpy as np

DEG = 5
LO, HI = -0.5, 0.5


def remez_relative(deg: int, iters: int = 40):
    # Chebyshev-like initial reference of deg + 2 points
    k = np.arange(deg + 2)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (deg + 1))
    f = np.exp2
    for _ in range(iters):
        # solve sum_j c_j x_i^j + (-1)^i E f(x_i) = f(x_i)  (relative error E)
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, : deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(xi)
        sol = np.linalg.solve(A, f(x))
        c = sol[: deg + 1]
        # new reference: extrema of the relative error on a fine grid
        g = np.linspace(LO, HI, 200001)
        err = (np.polyval(c[::-1], g) - f(g)) / f(g)
        # split the grid into deg + 2 sign-alternating segments, take the extremum of each
        sgn = np.sign(err)
        idx = [0]
        for i in range(1, g.size):
            if sgn[i] != sgn[idx[-1]] and sgn[i] != 0:
                idx.append(i)
        seg_bounds = idx + [g.size]
        ext = []
        for a, b in zip(seg_bounds[:-1], seg_bounds[1:]):
            j = a + int(np.argmax(np.abs(err[a:b])))
            ext.append(j)
        if len(ext) != deg + 2:
            break
        x = g[ext]
    return c


def main():
    c = remez_relative(DEG)
    c32 = c.astype(np.float32)
    g = np.linspace(LO, HI, 2000001)
    # Horner in float32 with fused multiply-add semantics approximated in double
    p = np.full_like(g, np.float64(c32[DEG]))
    for j in range(DEG - 1, -1, -1):
        p = p * g + np.float64(c32[j])
    rel = np.abs(p - np.exp2(g)) / np.exp2(g)
    for j, v in enumerate(c32):
        print("c%d = %.9e  (0x%08x)" % (j, v, np.float32(v).view(np.uint32)))
    print("max relative error of the float32-rounded polynomial: %.3e (2^%.2f)" % (rel.max(), np.log2(rel.max())))


if __name__ == "__main__":
    main()
