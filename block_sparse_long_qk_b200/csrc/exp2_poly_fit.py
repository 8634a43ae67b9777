"""Fits the cubic that approximates 2^f on [0, 1) in the attention softmax (attn.cu).

Method: Cody-Waite style range reduction x = n + f (n = floor(x), f in [0, 1)), then a
polynomial p(f) ~ 2^f, and the result assembled as p(f) * 2^n by adding n to the exponent
field. The cubic is fitted here by a Remez exchange on the relative error, with the end
conditions p(0) = 1 and p(1) = 2 so that the approximation is continuous across integers.

    python block_sparse_long_qk_b200/csrc/exp2_poly_fit.py

prints the coefficients (float32) and the achieved maximum relative error; the constants in
attn.cu were produced by this script.
"""
import numpy as np


def fit(iters=30, grid=200001):
    f = np.linspace(0.0, 1.0, grid)
    t = np.exp2(f)
    # Unknowns c1, c2 (c0 = 1, c3 = 1 - c1 - c2 from p(1) = 2) and the levelled error E.
    # p(f) - 2^f = (1 + c1 f + c2 f^2 + (1 - c1 - c2) f^3) - 2^f
    #            = c1 (f - f^3) + c2 (f^2 - f^3) + (1 + f^3 - 2^f)
    # Relative error e(f) = (p - 2^f) / 2^f equioscillates at 3 interior points.
    x = np.array([0.2, 0.5, 0.8])
    c = np.zeros(2)
    for _ in range(iters):
        A = np.zeros((3, 3))
        b = np.zeros(3)
        for i, xi in enumerate(x):
            w = np.exp2(xi)
            A[i, 0] = (xi - xi ** 3) / w
            A[i, 1] = (xi ** 2 - xi ** 3) / w
            A[i, 2] = (-1.0) ** i
            b[i] = -(1.0 + xi ** 3 - w) / w
        sol = np.linalg.solve(A, b)
        c = sol[:2]
        e = (c[0] * (f - f ** 3) + c[1] * (f ** 2 - f ** 3) + 1 + f ** 3 - t) / t
        # new reference: extrema of e on the three sign intervals between its zeros
        inner = e[1:-1]
        s = np.sign(inner)
        cuts = np.nonzero(np.diff(s) != 0)[0] + 1
        segs = np.split(np.arange(1, grid - 1), cuts)
        ext = [seg[np.argmax(np.abs(e[seg]))] for seg in segs if len(seg)]
        ext = sorted(ext, key=lambda i: -abs(e[i]))[:3]
        x = np.sort(f[ext])
    c1, c2 = c
    coef = np.array([1.0, c1, c2, 1.0 - c1 - c2])
    cf = coef.astype(np.float32)
    p = ((cf[3] * f.astype(np.float32) + cf[2]) * f.astype(np.float32) + cf[1]) * \
        f.astype(np.float32) + cf[0]
    rel = np.abs(p.astype(np.float64) - t) / t
    return cf, float(rel.max())


if __name__ == "__main__":
    cf, err = fit()
    for i, v in enumerate(cf):
        print(f"c{i} = {float(v)!r:>24}  ({v.view(np.uint32):#010x})")
    print(f"max relative error on [0, 1): {err:.3e}")
