"""Fit the polynomials behind hs2::exp2_poly<3> / exp2_poly<5> (exp2_poly.cuh).

2^x is computed as 2^n * 2^f with n = rint(x) and f = x - n in [-1/2, 1/2];
2^f is approximated by a polynomial fitted here: a least-squares fit of the
*relative* error 2^-f * P(f) - 1 on Chebyshev nodes of [-1/2, 1/2] (this is
close to the minimax fit), with P(0) = 1 imposed so that exact powers of two
come out exact.  Coefficients are rounded to float32 and the rounded
polynomial's relative error is reported (evaluated in float64 and in float32
Horner form).

    python -m long_context_sparse_flash_b200.csrc.gen_exp2_poly   # prints the header block
"""
import numpy as np


def fit(degree: int, n_nodes: int = 4001):
    k = np.arange(n_nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / n_nodes)  # Chebyshev nodes on [-1/2, 1/2]
    target = np.exp2(f)
    # P(f) = 1 + sum_{i>=1} c_i f^i ; minimise sum ((P - 2^f) / 2^f)^2
    A = np.stack([f ** i for i in range(1, degree + 1)], axis=1) / target[:, None]
    rhs = 1.0 - 1.0 / target
    c, *_ = np.linalg.lstsq(A, rhs, rcond=None)
    coef = np.concatenate([[1.0], c]).astype(np.float32)
    return coef


def rel_err(coef, n=200001):
    f = np.linspace(-0.5, 0.5, n)
    p64 = np.polyval(coef[::-1].astype(np.float64), f)
    e64 = np.max(np.abs(p64 / np.exp2(f) - 1))
    f32 = f.astype(np.float32)
    acc = np.float32(coef[-1]) * np.ones_like(f32)
    for ci in coef[-2::-1]:
        acc = acc * f32 + np.float32(ci)
    e32 = np.max(np.abs(acc.astype(np.float64) / np.exp2(f32.astype(np.float64)) - 1))
    return e64, e32


def main():
    for deg in (3, 5):
        coef = fit(deg)
        e64, e32 = rel_err(coef)
        names = ", ".join(f"{float(c):.9e}" for c in coef)
        print(f"// degree {deg}: max relative error {e64:.3e} (float64 eval), {e32:.3e} (float32 Horner)")
        print(f"// coefficients of f^0 .. f^{deg}: {names}")


if __name__ == "__main__":
    main()
