"""Lloyd-Max scalar codebook for the rotated-coordinate law (TEST INFRASTRUCTURE).

"TurboQuant explainer" (m.163.com), "第一步：PolarQuant": after the random
rotation every coordinate follows a known, highly concentrated Beta law and the
coordinates are nearly i.i.d., so the vector problem splits into independent
one-dimensional Max-Lloyd problems, solved once and stored as a codebook that
is looked up online.

Reading: one coordinate of a uniformly random unit vector in R^d has density

    f_d(t) = C_d (1 - t^2)^((d-3)/2)  on (-1, 1),
    C_d = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)),

i.e. (t + 1)/2 ~ Beta((d-1)/2, (d-1)/2).  d is the padded (power-of-two)
dimension the rotation acts on.

The solver is the textbook Lloyd iteration: thresholds are midpoints of
neighbouring centroids, centroids are conditional means of their cells.  The
cell probability is the regularised incomplete beta function and the cell's
first moment has the closed form  int t f_d(t) dt = -C_d (1-t^2)^((d-1)/2)/(d-1).
The same iteration run on the standard normal law reproduces Max's (1960)
tables; tests/golden/max1960_gaussian.txt pins it.

Stored form (the library stores the same): centroids rounded to fp32 (round to
nearest even); thresholds are the fp32 rounding of the exact midpoint of two
neighbouring fp32 centroids.
"""
import math

import numpy as np
from scipy import special


class BetaLaw:
    """Marginal of one coordinate of a uniform unit vector in R^d."""

    def __init__(self, d):
        self.d = int(d)
        self.a = (self.d - 1) / 2.0
        self.logC = (special.gammaln(self.d / 2.0) - 0.5 * math.log(math.pi)
                     - special.gammaln((self.d - 1) / 2.0))

    def pdf(self, t):
        t = np.asarray(t, dtype=np.float64)
        return np.exp(self.logC) * np.power(np.clip(1 - t * t, 0, None), (self.d - 3) / 2.0)

    def cdf(self, t):
        return special.betainc(self.a, self.a, (1.0 + np.asarray(t, dtype=np.float64)) / 2.0)

    def moment1(self, t):
        """int_{-1}^{t} s f(s) ds."""
        t = np.asarray(t, dtype=np.float64)
        return -np.exp(self.logC) * np.power(np.clip(1 - t * t, 0, None), self.a) / (self.d - 1)

    def ppf(self, p):
        return 2.0 * special.betaincinv(self.a, self.a, p) - 1.0

    lo, hi = -1.0, 1.0
    second_moment_value = property(lambda self: 1.0 / self.d)


class GaussLaw:
    """Standard normal law (used only to pin the solver against Max's tables)."""
    lo, hi = -np.inf, np.inf
    second_moment_value = 1.0

    def pdf(self, t):
        return np.exp(-0.5 * np.asarray(t, dtype=np.float64) ** 2) / math.sqrt(2 * math.pi)

    def cdf(self, t):
        return special.ndtr(t)

    def moment1(self, t):
        return -self.pdf(t)

    def ppf(self, p):
        return special.ndtri(p)


def _cell_mass(law, a, b):
    """P(a < T <= b), computed on the side of 0 that avoids cancellation (law symmetric)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    right = a >= 0
    left_mass = law.cdf(b) - law.cdf(a)
    right_mass = law.cdf(-a) - law.cdf(-b)
    return np.where(right, right_mass, left_mass)


def lloyd_max(law, levels, tol=1e-14, max_iter=400000):
    """Solve the Lloyd-Max conditions for `levels` cells; returns (centroids, thresholds) in fp64.

    The iteration starts from the (l + 1/2)/levels quantiles and stops when no
    centroid moves by more than `tol` standard deviations of the law, or, once
    steps are below 1e-11 standard deviations, when they stop shrinking for
    5000 iterations (the special functions' rounding floor at large d).
    Symmetry c_l = -c_{L-1-l} is imposed after every step (the law is
    symmetric, so the fixed point is symmetric).
    """
    L = int(levels)
    std = np.sqrt(law.second_moment_value)
    c = law.ppf((np.arange(L) + 0.5) / L)
    best, best_it = np.inf, 0
    for it in range(max_iter):
        t = 0.5 * (c[:-1] + c[1:])
        edges = np.concatenate([[law.lo], t, [law.hi]])
        mass = _cell_mass(law, edges[:-1], edges[1:])
        mom = law.moment1(edges[1:]) - law.moment1(edges[:-1])
        c_new = mom / mass
        c_new = 0.5 * (c_new - c_new[::-1])
        step = np.max(np.abs(c_new - c)) / std
        c = c_new
        if step < tol:
            break
        if step < best:
            best, best_it = step, it
        elif best < 1e-11 and it - best_it > 5000:
            break
    else:
        raise RuntimeError("Lloyd-Max did not converge")
    return c, 0.5 * (c[:-1] + c[1:])


def distortion(law, centroids, thresholds):
    """Mean squared error E[(T - Q(T))^2] of a scalar quantizer under `law` (fp64)."""
    c = np.asarray(centroids, dtype=np.float64)
    edges = np.concatenate([[law.lo], np.asarray(thresholds, dtype=np.float64), [law.hi]])
    mass = _cell_mass(law, edges[:-1], edges[1:])
    mom = law.moment1(edges[1:]) - law.moment1(edges[:-1])
    return law.second_moment_value - 2.0 * np.sum(c * mom) + np.sum(c * c * mass)


def stored_codebook(d_pad, mse_bits):
    """The stored codebook for dimension d_pad and 2**mse_bits levels.

    Returns (centroids fp32 [L], thresholds fp32 [L-1]).
    """
    c64, _ = lloyd_max(BetaLaw(d_pad), 1 << int(mse_bits))
    c32 = c64.astype(np.float32)
    mid = 0.5 * (c32[:-1].astype(np.float64) + c32[1:].astype(np.float64))
    return c32, mid.astype(np.float32)
