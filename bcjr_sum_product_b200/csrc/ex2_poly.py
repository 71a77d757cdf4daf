"""Coefficients of the FMA-pipe base-2 exponential used by the split-ex2 soft
kernel (bcjr_l16.cuh, ex2_fma).

Method: Cody and Waite's additive range reduction, x = n + f with n = round(x)
and f in [-1/2, 1/2], then 2^x = 2^n * P(f) with P a degree-5 polynomial.  P is
fitted here by least squares on 4001 Chebyshev nodes of [-1/2, 1/2], weighted
for relative error (each residual divided by 2^f), which comes within a small
factor of the minimax polynomial.  Running this file prints the coefficients
(highest degree first, as the Horner scheme in the kernel uses them) and the
relative error of P evaluated in fp32 with fused multiply-adds.

    python bcjr_sum_product_b200/csrc/ex2_poly.py
"""
import numpy as np

DEGREE = 5


def fit(degree: int = DEGREE) -> np.ndarray:
    k = np.arange(4001)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / len(k))          # Chebyshev nodes of [-1/2, 1/2]
    y = np.exp2(f)
    A = np.vander(f, degree + 1) / y[:, None]              # columns f^d .. f^0, relative weights
    coef, *_ = np.linalg.lstsq(A, np.ones_like(f), rcond=None)
    return coef                                            # highest degree first


def horner_fp32(coef: np.ndarray, f: np.ndarray) -> np.ndarray:
    c = coef.astype(np.float32)
    f = f.astype(np.float32)
    p = np.full_like(f, c[0])
    for ci in c[1:]:
        # one fp32 fused multiply-add: the product and sum rounded once
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(ci)).astype(np.float32)
    return p


def max_rel_error(coef: np.ndarray, n: int = 200001) -> float:
    f = np.linspace(-0.5, 0.5, n)
    p = horner_fp32(coef, f).astype(np.float64)
    ref = np.exp2(f.astype(np.float32).astype(np.float64))
    return float(np.max(np.abs(p - ref) / ref))


if __name__ == "__main__":
    c = fit()
    print("coefficients (f^5 .. f^0):", ", ".join(f"{float(np.float32(x))!r}f" for x in c))
    print("max relative error in fp32:", max_rel_error(c))
