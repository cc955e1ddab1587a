"""Pins of the oracle's product-code reconstruction (dequant_prod), the map
Q^-1 of "TurboQuant explainer" (m.163.com), "第二步：QJL".

* Linearity: the logit estimate is an inner product with the reconstruction,
  so <q, x_hat> equals logits_from_codes (itself pinned by unbiasedness over S
  in test_oracle_estimate.py) for every query — a transposed S, a missing
  gamma, a wrong sign convention or a wrong rotation direction fails it.
* With gamma = 0 it reduces to the MSE reconstruction; a zero vector
  reconstructs to zero.
* Unbiased over S: the mean of x_hat over independent Gaussian S (fp64,
  unrounded) is the MSE reconstruction plus the rotated-back residual, i.e. the
  input x, within 4 standard errors per coordinate.
"""
import numpy as np
import pytest

from oracle import codec, estimate
from oracle.codebook import stored_codebook
from oracle.params import sign_flips, qjl_matrix, gaussian_normals_f64


@pytest.mark.parametrize("d,d_pad,bits,m", [(128, 128, 3, 128), (128, 128, 4, 64), (200, 256, 2, 256), (64, 64, 4, 64)])
def test_inner_product_with_reconstruction_is_the_estimate(d, d_pad, bits, m):
    rng = np.random.default_rng(d + bits + m)
    c, t = stored_codebook(d_pad, bits - 1)
    D = sign_flips(7, d_pad)
    S = qjl_matrix(7, m, d_pad)
    x = rng.standard_normal((40, d)) * rng.uniform(0.5, 3.0, (40, 1))
    enc = codec.encode(x, D, c, t, S)
    xh = estimate.dequant_prod(enc["idx"], enc["signs"], enc["norm_f16"], enc["rnorm_f16"], c, D, S, m, d)
    q = rng.standard_normal((7, d))
    q_rot, u = estimate.prep_queries(q, D, S)
    lg = estimate.logits_from_codes(q_rot, u, enc["idx"], enc["signs"], enc["norm_f16"], enc["rnorm_f16"], c, m)
    assert np.allclose(q @ xh.T, lg, rtol=1e-11, atol=1e-11 * np.abs(lg).max())


def test_zero_residual_norm_is_the_mse_reconstruction_and_zero_is_zero():
    d = 128
    c, t = stored_codebook(d, 2)
    D = sign_flips(3, d)
    S = qjl_matrix(3, 128, d)
    x = np.random.default_rng(1).standard_normal((5, d))
    x[2] = 0.0
    enc = codec.encode(x, D, c, t, S)
    zero = np.zeros_like(enc["rnorm_f16"])
    xh = estimate.dequant_prod(enc["idx"], enc["signs"], enc["norm_f16"], zero, c, D, S, 128, d)
    assert np.allclose(xh, estimate.dequant_mse(enc["idx"], enc["norm_f16"], c, D, d), rtol=0, atol=1e-14)
    full = estimate.dequant_prod(enc["idx"], enc["signs"], enc["norm_f16"], enc["rnorm_f16"], c, D, S, 128, d)
    assert np.all(full[2] == 0.0)


def test_unbiased_over_S():
    d, m, N = 32, 32, 4000
    c, t = stored_codebook(d, 1)
    D = sign_flips(5, d)
    x = np.random.default_rng(9).standard_normal((1, d)) * 2.0
    acc = np.zeros((N, d))
    for s in range(N):
        S = gaussian_normals_f64(1000 + s, m, d)
        enc = codec.encode(x, D, c, t, S)
        # exact norms (no fp16 rounding) so that the expectation is x itself
        acc[s] = estimate.dequant_prod(enc["idx"], enc["signs"], enc["norm"], enc["gamma"], c, D, S, m, d)[0]
    mean, se = acc.mean(axis=0), acc.std(axis=0, ddof=1) / np.sqrt(N)
    assert np.all(np.abs(mean - x[0]) <= 4.0 * se + 1e-12)
