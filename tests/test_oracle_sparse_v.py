"""Pins for the oracle's Sparse V rule (zhidx turboquant_plus article,
"Sparse V": the value work of tokens with negligible attention weight is
skipped).  Reading: a token whose softmax weight p_j is below v_eps adds no
value and its weight stays in the normalisation."""
import numpy as np

from oracle import estimate


def test_closed_form_three_tokens():
    # logits ln p with p = (0.5, 0.3, 0.2): softmax returns p exactly (up to rounding)
    p = np.array([0.5, 0.3, 0.2])
    lg = np.log(p)
    v = np.eye(3)
    assert np.allclose(estimate.softmax_attend(lg, v, 1.0), p, atol=1e-15)
    # token 3 (0.2 < 0.25) dropped, the others keep their full-softmax weights (no renormalisation)
    assert np.allclose(estimate.softmax_attend(lg, v, 1.0, v_eps=0.25), [0.5, 0.3, 0.0], atol=1e-15)
    assert np.allclose(estimate.softmax_attend(lg, v, 1.0, v_eps=0.35), [0.5, 0.0, 0.0], atol=1e-15)
    # a weight equal to v_eps is kept (strict "below")
    assert np.allclose(estimate.softmax_attend(np.log([0.5, 0.5]), np.eye(2), 1.0, v_eps=0.5), [0.5, 0.5])


def test_everything_below_threshold_gives_zero():
    rng = np.random.default_rng(3)
    lg = rng.normal(size=50)
    v = rng.normal(size=(50, 8))
    p = estimate.softmax_weights(lg, 0.7)
    assert np.all(estimate.softmax_attend(lg, v, 0.7, v_eps=p.max() * 1.0001) == 0.0)


def test_zero_threshold_is_the_full_sum():
    rng = np.random.default_rng(4)
    lg = rng.normal(size=200)
    v = rng.normal(size=(200, 16))
    assert np.array_equal(estimate.softmax_attend(lg, v, 0.3, v_eps=0.0), estimate.softmax_attend(lg, v, 0.3))


def test_change_within_bound():
    rng = np.random.default_rng(5)
    for eps in (1e-4, 1e-3, 1e-2):
        lg = 3.0 * rng.normal(size=1000)          # peaked attention: many tiny weights
        v = rng.normal(size=(1000, 32))
        full = estimate.softmax_attend(lg, v, 1.0)
        sp = estimate.softmax_attend(lg, v, 1.0, v_eps=eps)
        p = estimate.softmax_weights(lg, 1.0)
        bound = eps * np.sum(np.linalg.norm(v[p < eps], axis=1))
        exact = np.linalg.norm(np.sum(p[p < eps, None] * v[p < eps], axis=0))
        assert np.isclose(np.linalg.norm(full - sp), exact, rtol=1e-9, atol=1e-15)
        assert exact <= bound
        assert np.sum(p < eps) > 0
