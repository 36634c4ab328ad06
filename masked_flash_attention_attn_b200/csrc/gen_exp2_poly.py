"""Fit the polynomial that the forward kernel uses for part of its exp2 evaluations.

Method (textbook; no vendor code involved):
  * Cody-Waite style range reduction, W. J. Cody and W. Waite, "Software Manual for the
    Elementary Functions" (1980): x = n + f with n = round(x) and f in [-1/2, 1/2], so that
    2^x = 2^n * 2^f, and 2^n is applied by adding n to the exponent field.
  * 2^f on [-1/2, 1/2] is approximated by the polynomial of degree DEG that minimises the
    maximum RELATIVE error, found with the Remez exchange algorithm (E. Remez, 1934):
    solve for the coefficients that equioscillate on DEG+2 reference points, move the
    references to the extrema of the error, repeat until the extrema level out.

Run:  python masked_flash_attention_attn_b200/csrc/gen_exp2_poly.py
It prints the coefficients as C float literals and the achieved max relative error; the
values are pasted into attn_fwd.cu (EXP2_POLY_C*).
"""
import numpy as np

DEG = 3


def remez(deg=DEG, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)
    k = np.arange(deg + 2)
    ref = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (deg + 1 - k) / (deg + 1))  # Chebyshev points
    grid = np.linspace(lo, hi, 200001)
    coef = None
    for _ in range(iters):
        # p(x_i) - f(x_i) = (-1)^i E f(x_i)   (relative error equioscillation), unknowns c_0..c_deg, E
        A = np.zeros((deg + 2, deg + 2))
        for i, x in enumerate(ref):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x)
        sol = np.linalg.solve(A, f(ref))
        coef = sol[:deg + 1]
        err = (np.polyval(coef[::-1], grid) - f(grid)) / f(grid)
        # new reference: alternating extrema of the error
        s = np.sign(err)
        idx = [0]
        for j in range(1, len(grid)):
            if s[j] != s[idx[-1]]:
                idx.append(j)
            elif abs(err[j]) > abs(err[idx[-1]]):
                idx[-1] = j
        idx = np.array(idx)
        while len(idx) > deg + 2:   # drop the smallest end extremum
            if abs(err[idx[0]]) < abs(err[idx[-1]]):
                idx = idx[1:]
            else:
                idx = idx[:-1]
        if len(idx) == deg + 2:
            ref = grid[idx]
    err = (np.polyval(coef[::-1], grid) - f(grid)) / f(grid)
    return coef, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez()
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 100001)
    e32 = np.abs((np.polyval(c32[::-1].astype(np.float64), g) - np.exp2(g)) / np.exp2(g)).max()
    for i, v in enumerate(c32):
        print(f"#define EXP2_POLY_C{i} {float(v).hex()}f  // {float(v):.9g}")
    print(f"// max relative error on [-1/2, 1/2]: {e:.3e} (fp64 coefficients), {e32:.3e} (fp32 coefficients)")
