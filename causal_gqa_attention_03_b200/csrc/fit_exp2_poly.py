"""Fit the cubic that approximates 2^f on [-1/2, 1/2] for the kernel's exp2.

Method: Lawson's iteratively reweighted least squares for the minimax
(equi-oscillating) relative error, starting from Chebyshev nodes, in fp64;
the coefficients are then rounded to fp32 and the fp32 evaluation (Horner
with fused multiply-adds) is checked on a dense grid.  2^x = 2^j * 2^f with
j = round(x) and f = x - j in [-1/2, 1/2] (Cody-Waite style range reduction).

Run:  python causal_gqa_attention_03_b200/csrc/fit_exp2_poly.py
Prints the coefficients c0..c3 (2^f ~ c0 + c1 f + c2 f^2 + c3 f^3) and the
maximum relative error of the fp32 evaluation.
"""
import numpy as np


def fit(degree: int = 3, iters: int = 400):
    n = 4000
    f = 0.5 * np.cos(np.pi * (np.arange(n) + 0.5) / n)  # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]  # relative error
    w = np.ones(n) / n
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], np.ones(n) * sw, rcond=None)
        e = np.abs(A @ c - 1.0)
        w = w * (e + 1e-300)
        w /= w.sum()
    return c


def eval_fp32(c, f):
    c = c.astype(np.float32)
    f = f.astype(np.float32)
    p = c[3]
    for k in (2, 1, 0):  # Horner; fp32 with a final rounding per step
        p = (p.astype(np.float64) * f + c[k]).astype(np.float32)
    return p


if __name__ == "__main__":
    c = fit()
    g = np.linspace(-0.5, 0.5, 2_000_001)
    rel = np.abs(eval_fp32(c, g).astype(np.float64) / np.exp2(g) - 1.0)
    for k, v in enumerate(c.astype(np.float32)):
        print(f"c{k} = {float(v)!r}f  ({v.view(np.uint32):#010x})")
    print(f"max relative error (fp32 Horner) = {rel.max():.3e}")
