"""Derivation of the exp2 polynomial used by the attention softmax (kExp2C0..3 in sm100.cuh).

A degree-3 polynomial p(f) ~ 2^f on f in [-1/2, 1/2], fitted for minimal maximum *relative*
error with Lawson's algorithm (iteratively reweighted least squares converging to the minimax
fit) on Chebyshev nodes.  The softmax rounds every probability to bf16 right after (relative
step 2^-8, rounding error <= 2^-9 = 1.95e-3), so a relative error near 1e-4 is invisible.

    python block_causal_streaming_b200/csrc/exp2_poly.py
"""
import numpy as np


def fit(degree: int = 3, nodes: int = 2000, iters: int = 200):
    f = 0.5 * np.cos(np.pi * (np.arange(nodes) + 0.5) / nodes)
    y = 2.0 ** f
    w = np.ones(nodes)
    for _ in range(iters):
        a = np.vander(f, degree + 1, increasing=True) / y[:, None]
        c, *_ = np.linalg.lstsq(a * np.sqrt(w)[:, None], np.sqrt(w), rcond=None)
        err = np.abs(np.polyval(c[::-1], f) / y - 1.0)
        w = w * (err + 1e-300)
        w /= w.sum()
    return c


def max_rel_error_fp32(c) -> float:
    c32 = np.asarray(c, dtype=np.float32)
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.zeros_like(f)
    for ci in c32[::-1]:
        p = (p * f + ci).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0)))


if __name__ == "__main__":
    c = fit()
    for i, ci in enumerate(np.asarray(c, dtype=np.float32)):
        print(f"kExp2C{i} = {float(ci):.17g}f")
    print(f"max relative error (fp32 Horner): {max_rel_error_fp32(c):.3e}")
