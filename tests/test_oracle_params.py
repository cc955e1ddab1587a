"""Pins of the oracle's random parameters (sign flips D, QJL matrix S).

The generator itself is pinned by Philox known-answer vectors
(test_oracle_philox.py); here the Box-Muller step and the stored rounding are
checked against the normal law and IEEE half rounding.
"""
import numpy as np
from scipy import stats

from oracle.params import sign_flips, gaussian_normals_f64, qjl_matrix
from oracle.philox import stream_words


def test_sign_flips_definition():
    w = stream_words(42, 0, 256)
    D = sign_flips(42, 256)
    np.testing.assert_array_equal(D == -1, (w & 1) == 1)
    assert set(np.unique(D)) == {-1, 1}


def test_box_muller_is_standard_normal():
    z = gaussian_normals_f64(7, 256, 256).ravel()
    ks = stats.kstest(z, "norm")
    assert ks.pvalue > 1e-3
    assert abs(z.mean()) < 4 / np.sqrt(z.size)
    assert abs(z.var() - 1) < 4 * np.sqrt(2 / z.size)
    # the two halves of every pair are uncorrelated
    r = np.corrcoef(z[0::2], z[1::2])[0, 1]
    assert abs(r) < 4 / np.sqrt(z.size / 2)


def test_box_muller_first_pair_by_hand():
    w = stream_words(123, 1, 2).astype(np.float64)
    ua, ub = (w + 0.5) / 2 ** 32
    rad = np.sqrt(-2 * np.log(ua))
    z = gaussian_normals_f64(123, 1, 2)[0]
    assert z[0] == rad * np.cos(2 * np.pi * ub)
    assert z[1] == rad * np.sin(2 * np.pi * ub)


def test_stored_s_is_half_rounding():
    z = gaussian_normals_f64(42, 128, 128)
    S = qjl_matrix(42, 128, 128)
    assert S.dtype == np.float16
    # round-to-nearest: no representable half is closer than the stored one
    err = np.abs(S.astype(np.float64) - z)
    up = np.abs(np.nextafter(S, np.float16(np.inf)).astype(np.float64) - z)
    dn = np.abs(np.nextafter(S, np.float16(-np.inf)).astype(np.float64) - z)
    assert np.all(err <= up) and np.all(err <= dn)
