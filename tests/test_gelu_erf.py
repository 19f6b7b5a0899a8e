"""The tensor-core MLP kernel evaluates erf by the rational approximation of
Abramowitz & Stegun, Handbook of Mathematical Functions, formula 7.1.26
(constants p, a1..a5 as published; |error| <= 1.5e-7).  This checks the
published bound for the constants the kernel uses, over the whole range the
MLP sees, and that GELU' built from the same exponential matches the exact
derivative.  The kernel itself is checked end to end by the MLP parity tests."""
import math

import numpy as np

P = 0.3275911
A = (0.254829592, -0.284496736, 1.421413741, -1.453152027, 1.061405429)


def erf_as(x):
    z = np.abs(x)
    t = 1.0 / (1.0 + P * z)
    poly = t * (A[0] + t * (A[1] + t * (A[2] + t * (A[3] + t * A[4]))))
    return np.sign(x) * (1.0 - poly * np.exp(-z * z)), np.exp(-z * z)


def test_erf_bound():
    x = np.linspace(-8.0, 8.0, 400001)
    approx, _ = erf_as(x)
    exact = np.array([math.erf(v) for v in x])
    assert np.max(np.abs(approx - exact)) <= 1.5e-7


def test_gelu_and_derivative():
    x = np.linspace(-10.0, 10.0, 20001)
    erf_v, ez = erf_as(x / math.sqrt(2.0))
    phi_cap = 0.5 * (1.0 + erf_v)
    gelu = x * phi_cap
    dgelu = phi_cap + x * ez / math.sqrt(2.0 * math.pi)   # exp(-(x/sqrt2)^2) = exp(-x^2/2)
    exact_phi = np.array([0.5 * (1.0 + math.erf(v / math.sqrt(2.0))) for v in x])
    exact = x * exact_phi
    exact_d = exact_phi + x * np.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)
    assert np.max(np.abs(gelu - exact)) <= 1.5e-6     # |x| <= 10 times the erf bound
    assert np.max(np.abs(dgelu - exact_d)) <= 1e-6
