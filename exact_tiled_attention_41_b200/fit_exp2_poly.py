"""Fit the polynomial used for the FMA-pipe half of exp2 in the softmax kernels.

    python -m exact_tiled_attention_41_b200.fit_exp2_poly

2^x is split as 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2]; 2^f is
approximated by a degree-5 polynomial p(f) whose maximum *relative* error on
[-1/2, 1/2] is minimised with the Remez exchange algorithm (equioscillation of
the weighted error p(f)/2^f - 1 at 7 points).  The script prints the
coefficients (highest degree first, as used by Horner's rule in sm100.cuh) and
the worst relative error of the fp32 Horner evaluation against float64 2^x.
exp2_fma2 in csrc/sm100.cuh uses exactly the printed float32 values (a CPU test
re-runs the fit and compares them with the header).
"""

import numpy as np

DEG = 5
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    # initial reference: Chebyshev extrema mapped to [LO, HI]
    k = np.arange(n)
    xs = (LO + HI) / 2 + (HI - LO) / 2 * np.cos(np.pi * k / (n - 1))[::-1]
    for _ in range(iters):
        f = np.exp2(xs)
        # solve sum_i c_i x^i - (-1)^j E f(x_j) = f(x_j)   (relative-error weighting)
        A = np.zeros((n, n))
        for j, x in enumerate(xs):
            A[j, :deg + 1] = x ** np.arange(deg + 1)
            A[j, deg + 1] = (-1) ** j * f[j]
        sol = np.linalg.solve(A, f)
        c = sol[:deg + 1]
        grid = np.linspace(LO, HI, 200001)
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        # new reference: extrema of the error between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        cand = grid[idx]
        cerr = err[idx]
        # keep n alternating extrema with the largest magnitudes
        sel = []
        for x, e in zip(cand, cerr):
            if sel and np.sign(e) == np.sign(sel[-1][1]):
                if abs(e) > abs(sel[-1][1]):
                    sel[-1] = (x, e)
            else:
                sel.append((x, e))
        while len(sel) > n:
            # drop the smaller end
            sel = sel[1:] if abs(sel[0][1]) < abs(sel[-1][1]) else sel[:-1]
        if len(sel) == n:
            xs = np.array([s[0] for s in sel])
    return c


def fp32_horner_error(c):
    c32 = np.asarray(c[::-1], dtype=np.float32)      # highest degree first
    x = np.linspace(-125.0, 8.0, 4_000_001).astype(np.float32)
    j = np.rint(x).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = np.full_like(f, c32[0])
    for a in c32[1:]:
        p = (p * f + a).astype(np.float32)             # separate rounding; FMA is at least as accurate
    y = np.ldexp(p.astype(np.float64), j.astype(np.int64))
    ref = np.exp2(x.astype(np.float64))
    return np.max(np.abs(y / ref - 1.0))


def coefficients_f32(deg=DEG):
    """The fitted coefficients rounded to float32, highest degree first."""
    return [np.float32(a) for a in remez(deg)[::-1]]


if __name__ == "__main__":
    c = remez()
    for i, a in enumerate(c[::-1]):
        print(f"c{DEG - i} = {np.float32(a)!r}  ({a:.17g})")
    print("max relative error (fp32 Horner) over [-125, 8]:", fp32_horner_error(c))
