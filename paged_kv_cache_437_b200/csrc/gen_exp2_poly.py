"""Coefficients of the degree-4 polynomial for 2^f, f in [-1/2, 1/2], used by
exp2_poly in mq_attention.cuh: a least-squares fit of the relative error on
2000 Chebyshev nodes, reweighted toward the largest errors (a few rounds of
iteratively reweighted least squares, approaching the minimax fit), printed
as fp32 constants with the fit's maximum relative error.

    python paged_kv_cache_437_b200/csrc/gen_exp2_poly.py
"""
import numpy as np


def fit(degree: int = 4, nodes: int = 2000, rounds: int = 50):
    k = np.arange(nodes)
    x = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)
    y = np.exp2(x)
    v = np.vander(x, degree + 1, increasing=True)
    w = 1.0 / y
    c = np.linalg.lstsq(v * w[:, None], y * w, rcond=None)[0]
    for _ in range(rounds):
        r = (v @ c - y) / y
        w2 = w * (1.0 + 20.0 * np.abs(r) / np.abs(r).max())
        c = np.linalg.lstsq(v * w2[:, None], y * w2, rcond=None)[0]
    c32 = c.astype(np.float32)
    xs = np.linspace(-0.5, 0.5, 200001)
    err = np.abs(np.polyval(c32[::-1].astype(np.float64), xs) / np.exp2(xs) - 1.0).max()
    return c32, err


if __name__ == "__main__":
    c, err = fit()
    print("coefficients c0..c4:", ", ".join(f"{v:.8f}f" for v in c))
    print(f"max relative error on [-1/2, 1/2]: {err:.3e}")
