"""Pins of the oracle's estimators.

* "TurboQuant explainer" (m.163.com), "第二步：QJL": E[<y, Q^-1(Q(x))>] = <y, x>.
  Over independent Gaussian S (fp64, unrounded) the mean estimate equals
  <q, x> within 4 standard errors, and the sample variance matches the exact
  variance n^2 ((pi/2) gamma^2 ||q_rot||^2 - <q_rot, r>^2) / m.
* Same section: a 1-bit MSE quantizer alone shrinks inner products by 2/pi;
  the product code (1 MSE bit + QJL) removes the shrinkage.
* With gamma = 0 the estimate is exactly <q, k_mse> for the dequantised key
  (exercises the rotated query and the centroid term without randomness).
* Decode attention: weights sum to one; equal logits give the mean of the
  dequantised values; the rotated-domain accumulation (one inverse rotation of
  sum_j p_j n_j c[idx_j]) equals dequantise-then-attend to 1e-12.
* Top-k equals a full stable sort; ties go to the lower id.
"""
import numpy as np
import pytest

from oracle import codec, estimate
from oracle.codebook import stored_codebook
from oracle.params import sign_flips, qjl_matrix, gaussian_normals_f64


def _estimate_with(x, q, D, S, c, t, m):
    enc = codec.encode(x, D, c, t, S)
    q_rot, u = estimate.prep_queries(q, D, S)
    lg = estimate.logits_from_codes(q_rot, u, enc["idx"], enc["signs"], enc["norm"], enc["gamma"], c, m)
    return lg, enc, q_rot


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_unbiased_over_S(bits):
    d, m, N = 128, 128, 3000
    c, t = stored_codebook(d, bits - 1)
    rng = np.random.default_rng(bits)
    x = rng.standard_normal((1, d)) * 3.0
    q = rng.standard_normal((1, d))
    D = sign_flips(11, d)
    vals = []
    for s in range(N):
        S = gaussian_normals_f64(1000 + s, m, d)
        lg, enc, q_rot = _estimate_with(x, q, D, S, c, t, m)
        vals.append(lg[0, 0])
    vals = np.array(vals)
    truth = float(q[0] @ x[0])
    n, g = enc["norm"][0], enc["gamma"][0]
    r = enc["r"][0]
    var = n * n * ((np.pi / 2) * g * g * (q_rot[0] @ q_rot[0]) - (q_rot[0] @ r) ** 2) / m
    assert abs(vals.mean() - truth) < 4 * np.sqrt(var / N)
    assert abs(vals.var() / var - 1) < 4 * np.sqrt(2.0 / N)


def test_unbiased_over_D_and_S():
    d, m, N = 128, 128, 2000
    c, t = stored_codebook(d, 2)
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, d))
    q = x + 0.5 * rng.standard_normal((1, d))
    vals = []
    for s in range(N):
        D = sign_flips(2000 + s, d)
        S = gaussian_normals_f64(9000 + s, m, d)
        lg, _, _ = _estimate_with(x, q, D, S, c, t, m)
        vals.append(lg[0, 0])
    vals = np.array(vals)
    assert abs(vals.mean() - float(q[0] @ x[0])) < 4 * vals.std() / np.sqrt(N)


def test_two_over_pi_shrinkage_and_its_removal():
    d, N = 512, 300
    c1, t1 = stored_codebook(d, 1)
    rng = np.random.default_rng(8)
    x = rng.standard_normal((1, d))
    q = x + 0.3 * rng.standard_normal((1, d))
    truth = float(q[0] @ x[0])
    mse_vals, prod_vals = [], []
    for s in range(N):
        D = sign_flips(500 + s, d)
        enc = codec.encode(x, D, c1, t1)
        q_rot, _ = estimate.prep_queries(q, D, None)
        mse_vals.append(estimate.logits_from_codes(q_rot, None, enc["idx"], None, enc["norm"], None, c1, 0)[0, 0])
        S = gaussian_normals_f64(7000 + s, d, d)
        lg, _, _ = _estimate_with(x, q, D, S, c1, t1, d)
        prod_vals.append(lg[0, 0])
    mse_vals, prod_vals = np.array(mse_vals), np.array(prod_vals)
    ratio = mse_vals.mean() / truth
    se = mse_vals.std() / np.sqrt(N) / abs(truth)
    assert abs(ratio - 2 / np.pi) < 4 * se + 2e-3      # 2/pi shrinkage (O(1/d) correction allowed)
    assert abs(prod_vals.mean() - truth) < 4 * prod_vals.std() / np.sqrt(N)


def test_centroid_term_is_inner_product_with_dequantised_key():
    # with gamma = 0 the estimate is exactly <q, k_mse>, k_mse = n D H c[idx] / sqrt(d)
    d = 128
    c, _ = stored_codebook(d, 3)
    D = sign_flips(1, d)
    S = qjl_matrix(1, d, d)
    rng = np.random.default_rng(4)
    idx = rng.integers(0, 8, size=(5, d)).astype(np.uint8)
    signs = rng.integers(0, 2, size=(5, d)).astype(np.uint8)
    n = np.array([2.0, 0.5, 7.0, 1.0, 3.25])
    k_mse = estimate.dequant_mse(idx, n, c, D, d)
    q = rng.standard_normal((4, d))
    q_rot, u = estimate.prep_queries(q, D, S)
    lg = estimate.logits_from_codes(q_rot, u, idx, signs, n, np.zeros(5), c, d)
    np.testing.assert_allclose(lg, q @ k_mse.T, rtol=1e-12, atol=1e-12)


def test_decode_routes_agree():
    d, T = 128, 300
    kc, kt = stored_codebook(d, 2)
    vc, vt = stored_codebook(d, 3)
    kD, vD = sign_flips(42, d), sign_flips(43, d)
    S = qjl_matrix(42, d, d)
    rng = np.random.default_rng(6)
    K = rng.standard_normal((T, d)) * 2
    V = rng.standard_normal((T, d))
    ke = codec.encode(K, kD, kc, kt, S)
    ve = codec.encode(V, vD, vc, vt)
    q = rng.standard_normal((1, 1, d))
    out = estimate.decode_attention(q, kD, S, ke["idx"], ke["signs"], ke["norm_f16"], ke["rnorm_f16"], kc, d,
                                    vD, ve["idx"], ve["norm_f16"], vc, d, [T], 1, 1, T)
    # rotated-domain route
    q_rot, u = estimate.prep_queries(q[0], kD, S)
    lg = estimate.logits_from_codes(q_rot, u, ke["idx"], ke["signs"], ke["norm_f16"], ke["rnorm_f16"], kc, d)[0]
    s = lg / np.sqrt(d)
    p = np.exp(s - s.max())
    p /= p.sum()
    assert abs(p.sum() - 1) < 1e-14
    acc = (p * ve["norm_f16"].astype(np.float64)) @ vc.astype(np.float64)[ve["idx"]]
    o2 = codec.unrotate(acc[None, :], vD)[0]
    np.testing.assert_allclose(out[0, 0], o2, rtol=1e-12, atol=1e-12)
    # equal logits -> plain mean of dequantised values
    vhat = estimate.dequant_mse(ve["idx"], ve["norm_f16"], vc, vD, d)
    np.testing.assert_allclose(estimate.softmax_attend(np.zeros(T), vhat, 1.0), vhat.mean(axis=0), atol=1e-12)


def test_topk_ties_and_sort():
    s = np.array([[1.0, 3.0, 3.0, 2.0, 3.0, -1.0]])
    ids, sc = estimate.topk(s, 4)
    assert list(ids[0]) == [1, 2, 4, 3]
    rng = np.random.default_rng(0)
    s = rng.standard_normal((5, 1000))
    ids, sc = estimate.topk(s, 10)
    for r in range(5):
        assert list(ids[r]) == list(np.argsort(-s[r], kind="stable")[:10])
    assert estimate.recall_at_k(ids, ids) == 1.0
