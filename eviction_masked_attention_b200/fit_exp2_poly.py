"""Derive the cubic used for 2^f, f in [-1/2, 1/2], in the attention kernels.

The kernels evaluate part of their exponentials on the FMA pipe instead of the
special-function unit: 2^x = 2^n * 2^f with n = round(x) (found by adding
1.5 * 2^23, which needs no conversion instruction), and 2^f ~ c0 + f*(c1 +
f*(c2 + f*c3)). The coefficients minimise the maximum relative error on
[-1/2, 1/2] (a Remez exchange on the relative error, started from a least-
squares fit at Chebyshev nodes). The result only has to beat the bf16 rounding
that P gets before the MMA (2^-9): the cubic's maximum relative error is 7.5e-5,
in exact arithmetic and in the kernels' fp32 evaluation alike, for x > -126
(1.5e-4 at the clamp: arguments below -126 are evaluated at -126, result ~1e-38;
with an exponent below -126 a cubic value under 1 would carry into the sign bit).

Run: python -m eviction_masked_attention_b200.fit_exp2_poly
"""
import numpy as np


LO, HI = -0.5, 0.5


def fit(deg: int = 3, iters: int = 30):
    # initial least-squares fit of the relative error at Chebyshev nodes
    n = 64
    x = 0.5 * (LO + HI) - 0.5 * (HI - LO) * np.cos(np.pi * (np.arange(n) + 0.5) / n)
    y = np.exp2(x)
    A = np.vander(x, deg + 1, increasing=True) / y[:, None]
    c = np.linalg.lstsq(A, np.ones(n), rcond=None)[0]
    # Remez exchange on e(x) = p(x)/2^x - 1 with deg + 2 reference points
    ref = 0.5 * (LO + HI) - 0.5 * (HI - LO) * np.cos(np.pi * np.arange(deg + 2) / (deg + 1))
    grid = np.linspace(LO, HI, 20001)
    for _ in range(iters):
        yr = np.exp2(ref)
        M = np.zeros((deg + 2, deg + 2))
        M[:, : deg + 1] = np.vander(ref, deg + 1, increasing=True) / yr[:, None]
        M[:, deg + 1] = (-1.0) ** np.arange(deg + 2)
        sol = np.linalg.solve(M, np.ones(deg + 2))
        c = sol[: deg + 1]
        err = np.polynomial.polynomial.polyval(grid, c) / np.exp2(grid) - 1.0
        # new reference: extrema of the error between sign changes
        s = np.sign(err)
        idx = np.concatenate([[0], np.nonzero(np.diff(s))[0] + 1, [len(grid)]])
        ext = [a + np.argmax(np.abs(err[a:b])) for a, b in zip(idx[:-1], idx[1:]) if b > a]
        if len(ext) >= deg + 2:
            ext = sorted(ext, key=lambda i: -abs(err[i]))[: deg + 2]
            ref = np.sort(grid[ext])
    return c, float(np.abs(err).max())


MAGIC = np.float32(12582912.0)  # 1.5 * 2^23: x + MAGIC rounds x to an integer


def eval_fp32(c, x):
    """The kernels' fp32 evaluation: t = x + MAGIC (round to nearest), f = x - (t - MAGIC),
    p = cubic(f), result bits = bits(p) + bits(t) * 2^23 (mod 2^32)."""
    cf = c.astype(np.float32)
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    t = (x + MAGIC).astype(np.float32)
    f = (x - (t - MAGIC)).astype(np.float32)
    p = (((cf[3] * f + cf[2]) * f + cf[1]) * f + cf[0]).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def fp32_error(c):
    """Max relative error of the kernel's fp32 evaluation over x in [-126, 8]."""
    x = np.linspace(-126.0, 8.0, 2_000_001).astype(np.float32)
    got = eval_fp32(c, x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    return float(np.max(np.abs(got / want - 1.0)))


if __name__ == "__main__":
    c, e = fit()
    print("coefficients c0..c3:", ", ".join(f"{v:.9e}" for v in c))
    print(f"max relative error (exact arithmetic) {e:.3e}, fp32 evaluation {fp32_error(c):.3e}")
