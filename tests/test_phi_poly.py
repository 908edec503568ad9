"""The polynomial constants of the row kernel's phi(y) = e^y - 1 - y tiers
are the ones the derivation script fits, and each tier holds its stated
error bound as the kernel evaluates it.

The kernel computes phi(lambda*x) = x^2 * Q(x) in fp32 Horner form with
Q_k = P_k * lambda^(k+2) rounded to fp32 (lambda = fl32(log2 e) * ln 2), the
P_k being the coefficients written into kld_rows_kernel.cuh from the printout of
csrc/phi_poly_fit.py. A transcription slip in any coefficient (a high-order
one only matters where |x| is large, which the benchmark data rarely reach)
fails the first test against the re-run fit, or the second against the
exact phi in 40-digit arithmetic. No GPU needed."""
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "logit_kl_divergence_b200", "csrc")
SRC = open(os.path.join(CSRC, "kld_rows_kernel.cuh")).read()


def _fit_module():
    spec = importlib.util.spec_from_file_location("phi_poly_fit", os.path.join(CSRC, "phi_poly_fit.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _array(name):
    m = re.search(r"constexpr double %s\[\d+\]\s*=\s*\{([^}]*)\}" % name, SRC)
    return [float(x) for x in m.group(1).replace("\n", " ").split(",")]


def _scalar(name):
    return float(re.search(r"\b%s\s*=\s*([0-9.eE+-]+)f?\b" % name, SRC).group(1))


def source_tiers():
    """(range, coefficients) of the three tiers as written in the kernel."""
    pc = [_scalar(f"kP{k}") for k in range(9)]
    return [(_scalar("kTauA"), _array("kPA")), (_scalar("kTauB"), _array("kPB")),
            (_scalar("kTau"), pc)]


# worst relative error of phi(lambda*x) per tier as evaluated in fp32 by the
# kernel (the kernel's comment states 1.7e-6 / 1.7e-6 / 9e-7)
BOUNDS = (1.75e-6, 1.7e-6, 9.0e-7)


def test_kernel_constants_are_the_fitted_ones():
    fit = _fit_module()
    tiers = source_tiers()
    assert [(t, len(c) - 1) for t, c in tiers] == [tuple(x) for x in fit.TIERS]
    for (tau, coeffs), (ftau, deg) in zip(tiers, fit.TIERS):
        ref = fit.fit(ftau, deg)
        rel = np.abs(np.asarray(coeffs) - ref) / np.abs(ref)
        # printed with 10 significant digits
        assert rel.max() <= 1e-9, (tau, rel)


def _fma32(a, b, c):
    # fp32 fused multiply-add: the product of two fp32 values is exact in
    # fp64, so one fp64 add and one rounding to fp32 (a double rounding that
    # can differ from a true FMA by one fp32 ulp, far inside the bounds)
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


@pytest.mark.parametrize("tier", [0, 1, 2])
def test_each_tier_holds_its_error_bound_in_fp32(tier):
    from mpmath import mp

    mp.dps = 40
    tau, coeffs = source_tiers()[tier]
    lam = float(np.float32(1.4426950408889634)) * 0.6931471805599453
    q = [np.float32(c * lam ** (k + 2)) for k, c in enumerate(coeffs)]
    worst = 0.0
    for x in np.linspace(-tau, tau, 8001).astype(np.float32):
        if abs(x) < 1e-6:
            continue
        acc = q[-1]
        for k in range(len(q) - 2, -1, -1):
            acc = _fma32(acc, x, q[k])
        phi = np.float32(np.float32(x * x) * acc)
        y = mp.mpf(float(x)) * mp.mpf(lam)
        ref = float(mp.expm1(y) - y)
        worst = max(worst, abs(float(phi) - ref) / abs(ref))
    assert worst <= BOUNDS[tier], (tier, worst)
    # and the bound is not slack enough to hide a wrong coefficient
    assert worst >= 0.3 * BOUNDS[tier]


def test_a_slipped_coefficient_is_caught():
    # the highest-order coefficient of tier C with one digit changed
    # (2.814820757e-07 -> 2.914820757e-07) breaks tier C's bound
    from mpmath import mp

    mp.dps = 40
    tau, coeffs = source_tiers()[2]
    bad = list(coeffs)
    bad[-1] *= 2.914820757 / 2.814820757
    lam = float(np.float32(1.4426950408889634)) * 0.6931471805599453
    q = [np.float32(c * lam ** (k + 2)) for k, c in enumerate(bad)]
    worst = 0.0
    for x in np.linspace(-tau, tau, 801).astype(np.float32):
        if abs(x) < 1e-6:
            continue
        acc = q[-1]
        for k in range(len(q) - 2, -1, -1):
            acc = _fma32(acc, x, q[k])
        phi = float(np.float32(np.float32(x * x) * acc))
        y = mp.mpf(float(x)) * mp.mpf(lam)
        worst = max(worst, abs(phi - float(mp.expm1(y) - y)) / abs(float(mp.expm1(y) - y)))
    assert worst > BOUNDS[2]
