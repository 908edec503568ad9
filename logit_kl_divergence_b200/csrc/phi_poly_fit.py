"""Derivation of the polynomials the row kernel uses for phi(y) = e^y - 1 - y.

The kernel needs phi(y) to about 1e-6 relative accuracy for |y| <= 2.5 (it
is the second-order part of the quant/base normaliser ratio, the same order
as the KL itself). It evaluates phi(y) = y^2 * P(y) in fp32 Horner form,
with the cheapest of three tiers whose range holds a whole chunk: degree 5
on [-1, 1], degree 6 on [-1.5, 1.5], degree 8 on [-2.5, 2.5]. Each P is
fitted here by weighted least squares (relative error) at 400 Chebyshev
nodes of its range against phi(y)/y^2 evaluated in 40-digit arithmetic; the
script prints the coefficients and the worst relative error of the fp32
evaluation on a dense grid (1.7e-6, 1.6e-6, 9.0e-7).

    python logit_kl_divergence_b200/csrc/phi_poly_fit.py

Not run at build time; the printed coefficients are written into kld_rows_kernel.cuh.
"""
import numpy as np
from mpmath import mp

TAU = 2.5
DEG = 8


def phi_over_y2(y):
    y = mp.mpf(y)
    if abs(y) < mp.mpf("1e-30"):
        return mp.mpf(1) / 2
    return (mp.e ** y - 1 - y) / y ** 2


def fit(tau=TAU, deg=DEG, nodes=400):
    mp.dps = 40
    k = np.arange(nodes)
    xs = tau * np.cos(np.pi * (k + 0.5) / nodes)
    ys = np.array([float(phi_over_y2(x)) for x in xs])
    V = np.vander(xs, deg + 1, increasing=True)
    c, *_ = np.linalg.lstsq(V / ys[:, None], np.ones(nodes), rcond=None)
    return c


def fp32_rel_error(c, tau=TAU):
    mp.dps = 40
    xt = np.linspace(-tau, tau, 4001).astype(np.float32)
    cf = np.asarray(c, np.float32)
    p = np.full_like(xt, cf[-1])
    for ci in cf[-2::-1]:
        p = (p * xt + ci).astype(np.float32)
    phi32 = (xt * xt).astype(np.float32) * p
    ref = np.array([float(mp.e ** mp.mpf(float(x)) - 1 - mp.mpf(float(x))) for x in xt])
    keep = np.abs(xt) > 1e-6
    return float(np.max(np.abs(phi32[keep] - ref[keep]) / np.abs(ref[keep])))


TIERS = ((1.0, 5), (1.5, 6), (TAU, DEG))

if __name__ == "__main__":
    for tau, deg in TIERS:
        c = fit(tau, deg)
        print(f"[-{tau}, {tau}] degree {deg}:", ", ".join(f"{v:.10g}" for v in c))
        print("  max relative error of phi in fp32:", fp32_rel_error(c, tau))
