"""Fit the polynomial used for part of the exponentials in prefill.cu.

2^x is split Cody-Waite style: n = round-to-nearest(x), f = x - n in
[-1/2, 1/2], 2^x = 2^n * p(f), with p a degree-3 polynomial that minimises
the maximum RELATIVE error of p(f) against 2^f on [-1/2, 1/2].  The fit is a
Remez exchange on the weighted error (p(f) - 2^f) / 2^f, started from a
Chebyshev-node least-squares fit.  The probabilities that use it are rounded
to bf16 (relative spacing 2^-8) right after, so a relative error near 1e-4 is
far below what reaches the P V product.

Run: python fit_exp2_poly.py   (prints the coefficients pasted into prefill.cu)
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def rel_err(c, f):
    return np.polynomial.polynomial.polyval(f, c) / np.exp2(f) - 1.0


def remez(deg=DEG, iters=30):
    n = deg + 2
    # start: least squares on Chebyshev nodes, weighted by 1/2^f
    k = np.arange(4 * n)
    nodes = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (k + 0.5) / len(k))
    A = np.vander(nodes, deg + 1, increasing=True) / np.exp2(nodes)[:, None]
    c = np.linalg.lstsq(A, np.ones_like(nodes), rcond=None)[0]
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        e = rel_err(c, grid)
        # alternation points: extrema of the error, one per sign run
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (e[i] - e[i - 1]) * (e[i + 1] - e[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = np.array(idx)
        # keep the n largest alternating extrema
        runs, cur = [], [idx[0]]
        for i in idx[1:]:
            if np.sign(e[i]) == np.sign(e[cur[-1]]):
                cur.append(i)
            else:
                runs.append(cur)
                cur = [i]
        runs.append(cur)
        pts = [r[np.argmax(np.abs(e[r]))] for r in runs]
        while len(pts) > n:
            # drop the smaller end
            if abs(e[pts[0]]) < abs(e[pts[-1]]):
                pts = pts[1:]
            else:
                pts = pts[:-1]
        if len(pts) < n:
            break
        x = grid[pts]
        # solve p(x_i) / 2^x_i - 1 = (-1)^i E
        M = np.zeros((n, n))
        M[:, :deg + 1] = np.vander(x, deg + 1, increasing=True) / np.exp2(x)[:, None]
        M[:, deg + 1] = (-1.0) ** np.arange(n)
        sol = np.linalg.solve(M, np.ones(n))
        c = sol[:deg + 1]
    return c, np.abs(rel_err(c, grid)).max()


if __name__ == "__main__":
    c, err = remez()
    for i, v in enumerate(c):
        print(f"c{i} = {np.float32(v)!r}  ({v:.17g})")
    # the same evaluation in fp32, Horner form, as the kernel does it
    f = np.linspace(LO, HI, 1000001).astype(np.float32)
    cf = c.astype(np.float32)
    p = ((cf[3] * f + cf[2]) * f + cf[1]) * f + cf[0]
    print("max relative error (fp64 fit):", err)
    print("max relative error (fp32 Horner):", np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1).max())
