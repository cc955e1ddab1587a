"""Pins of the oracle's rotation, encoder and canonical layout.

* Hadamard: H H^T = d I exactly (integers), H e_0 = all ones, and an
  independently written fast butterfly equals the dense matrix.
* The rotation preserves norms (orthogonality) to 1e-12.
* Brute force at d_pad = 4 and 8: the per-coordinate threshold rule equals the
  argmin over *all* L^d_pad index vectors of ||y - c[idx]|| (separability).
* Monte Carlo: for uniformly random unit vectors the mean squared residual
  equals d_pad times the one-dimensional Lloyd-Max distortion (quadrature),
  within 4 standard errors.
* Rotated coordinates of a fixed vector over random sign flips follow the Beta
  law of the explainer's "第一步：PolarQuant" section (KS statistic reported,
  loose gate) and are nearly uncorrelated.
* Layout: bytes per vector (zhidx turboquant_plus article: turbo4 = 4.25
  bit/value, about 3.8x smaller than fp16), exact bit positions of a hand-built
  example, pack/unpack round trip, zero-filled tail.
* Boundary conventions: a value exactly on a threshold goes to the lower cell;
  the zero vector keeps n = 0.
"""
import itertools

import numpy as np
import pytest
from scipy import stats

from oracle import codec
from oracle.codebook import BetaLaw, lloyd_max, distortion, stored_codebook
from oracle.params import sign_flips, qjl_matrix


def fwht_reference(v):
    """In-place iterative fast Walsh-Hadamard transform (unnormalised), natural order."""
    v = np.array(v, dtype=np.float64)
    n = v.shape[-1]
    h = 1
    while h < n:
        for i in range(0, n, 2 * h):
            a = v[..., i:i + h].copy()
            b = v[..., i + h:i + 2 * h].copy()
            v[..., i:i + h] = a + b
            v[..., i + h:i + 2 * h] = a - b
        h *= 2
    return v


@pytest.mark.parametrize("d", [4, 8, 32, 128, 256])
def test_hadamard_exact(d):
    H = codec.hadamard(d)
    np.testing.assert_array_equal(H @ H.T, d * np.eye(d))
    np.testing.assert_array_equal(H[:, 0], np.ones(d))
    x = np.random.default_rng(d).standard_normal((5, d))
    np.testing.assert_allclose(x @ H.T, fwht_reference(x), rtol=0, atol=1e-12)


@pytest.mark.parametrize("d", [128, 256])
def test_rotation_orthogonal(d):
    D = sign_flips(42, d)
    x = np.random.default_rng(1).standard_normal((50, d))
    y = codec.rotate(x, D)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    np.testing.assert_allclose(codec.unrotate(y, D), x, atol=1e-12)


@pytest.mark.parametrize("d_pad,bits", [(4, 1), (4, 2), (4, 3), (8, 1), (8, 2)])
def test_brute_force_nearest_code(d_pad, bits):
    L = 1 << bits
    c, t = stored_codebook(d_pad, bits)
    cands = np.array(list(itertools.product(range(L), repeat=d_pad)), dtype=np.uint8)
    C = c.astype(np.float64)[cands]                       # [L^d, d]
    D = sign_flips(3, d_pad)
    x = np.random.default_rng(7).standard_normal((40, d_pad))
    enc = codec.encode(x, D, c, t)
    for v in range(x.shape[0]):
        dist = np.sum((enc["y"][v][None, :] - C) ** 2, axis=1)
        best = cands[np.argmin(dist)]
        np.testing.assert_array_equal(enc["idx"][v], best)
        np.testing.assert_allclose(enc["gamma"][v] ** 2, dist.min(), rtol=1e-12)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_monte_carlo_distortion(bits):
    d = 128
    c, t = stored_codebook(d, bits)
    D = sign_flips(5, d)
    x = np.random.default_rng(bits).standard_normal((20000, d))
    enc = codec.encode(x, D, c, t)
    g2 = enc["gamma"] ** 2
    law = BetaLaw(d)
    expect = d * distortion(law, c, t)
    se = g2.std() / np.sqrt(g2.size)
    assert abs(g2.mean() - expect) < 4 * se


def test_rotated_law_and_decorrelation():
    d = 128
    x = np.random.default_rng(0).standard_normal(d)
    x /= np.linalg.norm(x)
    ys = np.stack([codec.rotate(x[None, :], sign_flips(s, d))[0] for s in range(400)])
    law = BetaLaw(d)
    ks = stats.kstest(ys[:, 5], law.cdf)
    assert ks.pvalue > 1e-3
    corr = np.corrcoef(ys[:, :8].T)
    off = corr[~np.eye(8, dtype=bool)]
    assert np.max(np.abs(off)) < 0.25


def test_layout_bytes_and_bit_accounting():
    # product code, b = 4 (3-bit indices + 128 signs), d = 128: 64 code bytes + 2 fp16 norms
    per_vec = codec.code_bytes(128, 3, 128, 32) / 32 + 4
    assert per_vec == 68
    assert per_vec * 8 / 128 == 4.25                  # turbo4: 4.25 bit/value
    assert abs(16 / 4.25 - 3.8) < 0.05               # ~3.8x smaller than fp16
    assert codec.code_bytes(128, 2, 128, 1) == 32 * 48       # b = 3: 48 B/vector, 52 with norms
    assert codec.code_bytes(128, 1, 128, 33) == 64 * 32      # two tiles
    assert codec.code_bytes(128, 3, 0, 32) == 32 * 48        # MSE-only b = 3: 48 (+2) B


def test_layout_bit_positions():
    d_pad, kb, m, n = 128, 2, 64, 35
    idx = np.zeros((n, d_pad), dtype=np.uint8)
    signs = np.zeros((n, m), dtype=np.uint8)
    idx[33, 37] = 3        # vector 33 (tile 1, slot 1), coordinate 37: bit 5 of word 1, both planes
    signs[2, 40] = 1       # vector 2 (tile 0, slot 2), sign 40: bit 8 of word 1
    buf = codec.pack(idx, signs, kb, m)
    tile_bytes = 32 * (kb * d_pad // 8 + m // 8)
    assert buf.size == 2 * tile_bytes
    words = buf.view(np.uint32)
    for p in range(kb):
        w = (tile_bytes + p * 32 * 16 + 1 * 16) // 4 + 1
        assert words[w] == 1 << 5
    w = (kb * 32 * 16 + 2 * 8) // 4 + 1
    assert words[w] == 1 << 8
    assert np.count_nonzero(buf) == 3
    i2, s2 = codec.unpack(buf, n, d_pad, kb, m)
    np.testing.assert_array_equal(i2, idx)
    np.testing.assert_array_equal(s2, signs)


def test_pack_roundtrip_random():
    rng = np.random.default_rng(3)
    for (d_pad, kb, m, n) in [(128, 3, 128, 77), (256, 1, 256, 32), (128, 4, 0, 5)]:
        idx = rng.integers(0, 1 << kb, size=(n, d_pad)).astype(np.uint8)
        signs = rng.integers(0, 2, size=(n, m)).astype(np.uint8) if m else None
        buf = codec.pack(idx, signs, kb, m)
        assert buf.size == codec.code_bytes(d_pad, kb, m, n)
        i2, s2 = codec.unpack(buf, n, d_pad, kb, m)
        np.testing.assert_array_equal(i2, idx)
        if m:
            np.testing.assert_array_equal(s2, signs)
        # tail slots of the last tile are zero
        i3, _ = codec.unpack(buf, ((n + 31) // 32) * 32, d_pad, kb, m)
        assert not np.any(i3[n:])


def test_threshold_tie_and_zero_vector():
    c, t = stored_codebook(128, 2)
    D = np.ones(128, dtype=np.int8)
    enc = codec.encode(np.zeros((1, 128)), D, c, t)
    assert enc["norm"][0] == 0 and enc["norm_f16"][0] == 0
    # y = 0 exactly on the middle threshold 0 -> lower cell (index L/2 - 1)
    assert np.all(enc["idx"][0] == 1)
    # a value placed exactly on threshold t[2] goes to cell 2
    y = np.zeros(128)
    y[0] = t[2]
    y[1] = np.nextafter(t[2], 1.0)
    y /= np.linalg.norm(y)
    # rotate back to an input whose rotation is exactly y (up to fp64 rounding)
    x = codec.unrotate(y[None, :], D)
    enc = codec.encode(x, D, c, t)
    assert enc["idx"][0, 0] in (2, 3)


def test_signs_follow_projection():
    d = 128
    c, t = stored_codebook(d, 3)
    D = sign_flips(42, d)
    S = qjl_matrix(42, d, d)
    x = np.random.default_rng(9).standard_normal((64, d))
    enc = codec.encode(x, D, c, t, S)
    z = enc["r"] @ S.astype(np.float64).T
    np.testing.assert_array_equal(enc["signs"], (z >= 0).astype(np.uint8))
    # the estimator's QJL term needs E[sign] structure: about half the bits set
    assert 0.4 < enc["signs"].mean() < 0.6


def test_sliced_layout_hand_example():
    # 33 vectors of d_pad 8 at kb = 2: vector 1 has index 3 at coordinate 5 (both planes), vector 32
    # (tile 1, t = 0) has index 2 at coordinate 0 (plane 1 only); everything else 0
    idx = np.zeros((33, 8), dtype=np.uint8)
    idx[1, 5] = 3
    idx[32, 0] = 2
    buf = codec.pack_sliced(idx, 2)
    w = buf.view("<u4").reshape(2, 2, 8)          # [tile][plane][coordinate]
    want = np.zeros((2, 2, 8), dtype=np.uint32)
    want[0, 0, 5] = 1 << 1
    want[0, 1, 5] = 1 << 1
    want[1, 1, 0] = 1
    assert np.array_equal(w, want)
    assert buf.size == codec.code_bytes(8, 2, 0, 33)
    assert np.array_equal(codec.unpack_sliced(buf, 33, 8, 2), idx)


def test_sliced_layout_is_the_transposed_tile():
    # each tile's plane in the sliced layout is the 32 x d_pad bit matrix of the canonical plane, transposed
    r = np.random.default_rng(3)
    n, d_pad, kb = 77, 128, 3
    idx = r.integers(0, 1 << kb, size=(n, d_pad)).astype(np.uint8)
    s = codec.pack_sliced(idx, kb)
    assert np.array_equal(codec.unpack_sliced(s, n, d_pad, kb), idx)
    c = codec.pack(idx, None, kb, 0)
    assert s.size == c.size
    tb = 32 * kb * d_pad // 8
    for tile in range((n + 31) // 32):
        for p in range(kb):
            cp = np.unpackbits(c[tile * tb + p * 32 * d_pad // 8: tile * tb + (p + 1) * 32 * d_pad // 8]
                               .reshape(32, d_pad // 8), axis=1, bitorder="little")          # [t][j]
            sp = np.unpackbits(s[tile * tb + p * d_pad * 4: tile * tb + (p + 1) * d_pad * 4]
                               .reshape(d_pad, 4), axis=1, bitorder="little")                # [j][t]
            assert np.array_equal(cp.T, sp)
