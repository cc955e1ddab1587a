"""High-precision pin of the stored codebook digits: the Lloyd-Max fixed point
of the rotated-coordinate law at d_pad = 128 and 256, solved here by Newton's method
in 30-digit arithmetic with the cell integrals taken by mpmath's own
quadrature of the density (not the oracle's closed forms), must agree with the
oracle's fp64 centroids to 1e-11 of the law's standard deviation (the
oracle's documented stopping floor), and its fp32 rounding must be the stored
codebook, digit for digit."""
import mpmath as mp
import numpy as np
import pytest

from oracle.codebook import BetaLaw, lloyd_max, stored_codebook


def _mp_fixed_point(d, L, start):
    mp.mp.dps = 30
    a = mp.mpf(d - 3) / 2
    f = lambda t: (1 - t * t) ** a  # unnormalised density on (-1, 1)
    half = L // 2

    def residual(*c_pos):  # unknowns: the positive centroids; symmetry gives the rest
        c = [-x for x in reversed(c_pos)] + list(c_pos)
        edges = [mp.mpf(-1)] + [(c[j] + c[j + 1]) / 2 for j in range(L - 1)] + [mp.mpf(1)]
        out = []
        for j in range(half, L):
            m0 = mp.quad(f, [edges[j], edges[j + 1]])
            m1 = mp.quad(lambda t: t * f(t), [edges[j], edges[j + 1]])
            out.append(c[j] - m1 / m0)
        return out

    sol = mp.findroot(residual, [mp.mpf(x) for x in start[half:]], tol=mp.mpf(10) ** -26)
    return np.array([float(x) for x in (sol if hasattr(sol, "__len__") else [sol])])


@pytest.mark.parametrize("d,kb", [(128, 1), (128, 2), (128, 3), (128, 4), (256, 2), (256, 3)])
def test_codebook_digits(d, kb):
    L = 1 << kb
    c, _ = lloyd_max(BetaLaw(d), L)
    ref = _mp_fixed_point(d, L, c)
    full = np.concatenate([-ref[::-1], ref])
    assert np.max(np.abs(c - full)) < 1e-11 / np.sqrt(d)
    c32, _ = stored_codebook(d, kb)
    assert np.array_equal(c32, full.astype(np.float32))
