"""Pins of the oracle's Lloyd-Max codebook.

* The solver reproduces Max's (1960) Gaussian tables (tests/golden/max1960_gaussian.txt).
* The Beta-law closed forms (cdf, first moment) agree with direct numerical
  integration of the density; the density integrates to 1 and has variance 1/d.
* The solution satisfies the Lloyd-Max conditions (centroid = conditional
  mean by independent quadrature; threshold = midpoint; odd symmetry).
* L = 2 closed form: c = +-E|T| = +-Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2)).
* Large-d limit: sqrt(d) c approaches the Gaussian solution at rate O(1/d).
* "TurboQuant explainer" (m.163.com), "合起来": the distortion stays within
  about 2.7x of the 4^-b lower bound and the gap is smaller at low bit width.
"""
import math
import os

import numpy as np
import pytest
from scipy import integrate, special

from oracle.codebook import BetaLaw, GaussLaw, lloyd_max, distortion, stored_codebook

GOLD = os.path.join(os.path.dirname(__file__), "golden", "max1960_gaussian.txt")


def _max_table():
    rows, tol = {}, {}
    for line in open(GOLD):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("tol_"):
            k, v = line.split()
            tol[k] = float(v)
            continue
        L, c, t, mse = [s.strip() for s in line.split("|")]
        rows[int(L)] = ([float(x) for x in c.split()], [float(x) for x in t.split()], float(mse))
    return rows, tol


def test_gaussian_solver_matches_max_1960():
    rows, tol = _max_table()
    for L, (cpos, tpos, mse) in rows.items():
        c, t = lloyd_max(GaussLaw(), L)
        np.testing.assert_allclose(c[L // 2:], cpos, atol=tol["tol_c"])
        np.testing.assert_allclose(t[L // 2 - 1:], tpos, atol=tol["tol_c"])
        assert abs(distortion(GaussLaw(), c, t) - mse) <= tol["tol_mse_rel"] * mse


@pytest.mark.parametrize("d", [16, 128, 256])
def test_beta_closed_forms_vs_quadrature(d):
    law = BetaLaw(d)
    tot, _ = integrate.quad(law.pdf, -1, 1, epsabs=1e-14, epsrel=1e-13, limit=200)
    assert abs(tot - 1) < 1e-12
    var, _ = integrate.quad(lambda s: s * s * law.pdf(s), -1, 1, epsabs=1e-15, epsrel=1e-13, limit=200)
    assert abs(var - 1.0 / d) < 1e-12
    for t in [-0.5, -0.1, 0.0, 0.03, 0.2, 0.4]:
        F, _ = integrate.quad(law.pdf, -1, t, epsabs=1e-15, epsrel=1e-13, limit=200)
        assert abs(F - law.cdf(t)) < 1e-12
        G, _ = integrate.quad(lambda s: s * law.pdf(s), -1, t, epsabs=1e-16, epsrel=1e-13, limit=200)
        assert abs(G - law.moment1(t)) < 1e-13


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_lloyd_max_conditions(d, bits):
    law = BetaLaw(d)
    L = 1 << bits
    c, t = lloyd_max(law, L)
    assert np.all(np.diff(c) > 0)
    np.testing.assert_allclose(c, -c[::-1], atol=0, rtol=0)
    np.testing.assert_allclose(t, 0.5 * (c[:-1] + c[1:]), atol=1e-18, rtol=0)
    edges = np.concatenate([[-1.0], t, [1.0]])
    for l in range(L):
        a, b = edges[l], edges[l + 1]
        m0, _ = integrate.quad(law.pdf, a, b, epsabs=1e-16, epsrel=1e-14, limit=400)
        m1, _ = integrate.quad(lambda s: s * law.pdf(s), a, b, epsabs=1e-18, epsrel=1e-14, limit=400)
        assert abs(m1 / m0 - c[l]) <= 1e-12 * max(1.0, abs(c[l]) * math.sqrt(d))


@pytest.mark.parametrize("d", [64, 128, 256, 1024])
def test_two_level_closed_form(d):
    c, t = lloyd_max(BetaLaw(d), 2)
    e_abs = math.exp(special.gammaln(d / 2) - 0.5 * math.log(math.pi) - special.gammaln((d + 1) / 2))
    assert abs(c[1] - e_abs) < 1e-14
    assert t[0] == 0.0


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_gaussian_limit(bits):
    L = 1 << bits
    cg, _ = lloyd_max(GaussLaw(), L)
    errs = []
    for d in (256, 1024, 4096):
        c, _ = lloyd_max(BetaLaw(d), L)
        errs.append(np.max(np.abs(np.sqrt(d) * c - cg)))
    # O(1/d): each 4x larger d shrinks the gap about 4x
    assert errs[0] < 0.05
    assert errs[1] < errs[0] / 3.0 and errs[2] < errs[1] / 3.0


@pytest.mark.parametrize("d", [128, 256])
def test_distortion_within_paper_factor(d):
    law = BetaLaw(d)
    ratios = []
    for bits in (1, 2, 3, 4):
        c, t = lloyd_max(law, 1 << bits)
        D = d * distortion(law, c, t)            # E||x_hat - Q(x_hat)||^2 for a unit vector
        ratios.append(D / 4.0 ** (-bits))
    assert max(ratios) <= 2.72                    # ~2.7x of the 4^-b bound
    assert all(a < b for a, b in zip(ratios, ratios[1:]))   # smaller gap at low bit width
    # the high-resolution limit of the Gaussian is sqrt(3) pi / 2 = 2.72
    assert ratios[-1] < math.sqrt(3) * math.pi / 2


def test_stored_rounding():
    c32, t32 = stored_codebook(128, 3)
    assert c32.dtype == np.float32 and t32.dtype == np.float32
    c64, _ = lloyd_max(BetaLaw(128), 8)
    np.testing.assert_array_equal(c32, c64.astype(np.float32))
    mid = (c32[:-1].astype(np.float64) + c32[1:].astype(np.float64)) / 2
    np.testing.assert_array_equal(t32, mid.astype(np.float32))
    assert t32[3] == 0.0
