"""Pins of the oracle's tolerance-band functions and of its multi-head index maps.

codec.boundary_flags and polar.boundary_flags decide which GPU/oracle
differences the parity tests excuse, so each rule is checked here on
hand-built points just inside (0.9x) and just outside (1.1x) the band:

* code decisions: |y - t_l| <= 1e-6 * max(|t_l|, 1/sqrt(d_pad)), including the
  threshold at 0, where only the floor 1/sqrt(d_pad) applies;
* sign decisions: |z_i| <= 1e-6 * ||S_i|| * gamma with ||S_i|| the norm of ROW i
  of S (a hand-made S whose row and column norms differ);
* fp16 norms: within 1e-6 (relative) of a half-precision rounding tie;
* polar angles: distance of the point to the boundary ray at most
  1e-6 * max(radius, 1/sqrt(d_pad)).

The index maps of estimate.logits_gqa (query head h reads KV head h // group)
and estimate.decode_attention (vector (b * Hkv + g) * max_tokens + t, the first
seq_lens[b] tokens only) are checked against dense attention over explicitly
dequantised keys and values (a route pinned in test_oracle_estimate.py).
"""
import math

import numpy as np
import pytest

from oracle import codec, estimate, polar
from oracle.codebook import stored_codebook
from oracle.params import sign_flips


def _flags_for(y, t, d_pad):
    enc = dict(y=np.asarray(y, dtype=np.float64).reshape(1, -1), norm=np.array([1.0]), gamma=np.array([0.5]))
    return codec.boundary_flags(enc, np.asarray(t, dtype=np.float32))["idx"][0]


@pytest.mark.parametrize("d_pad", [4, 128])
def test_code_band_scale_and_floor(d_pad):
    fl = 1.0 / math.sqrt(d_pad)
    # |t| = 0.375 is above the floor at d_pad 128 (0.088) and below it at d_pad 4 (0.5)
    t = np.array([-0.375, 0.0, 0.375], dtype=np.float32)
    for tl in t.astype(np.float64):
        scale = max(abs(tl), fl)
        inside = [tl + 0.9e-6 * scale, tl - 0.9e-6 * scale]
        outside = [tl + 1.1e-6 * scale, tl - 1.1e-6 * scale]
        y = np.zeros(d_pad)
        y[:2] = inside
        y[2:4] = outside
        f = _flags_for(y, t, d_pad)
        assert f[0] and f[1], (tl, d_pad)
        assert not f[2] and not f[3], (tl, d_pad)


def test_code_band_small_threshold_uses_floor():
    # |t| = 0.01 < 1/sqrt(4) = 0.5: the band is 1e-6 * 0.5, not 1e-6 * 0.01
    d_pad = 4
    t = np.array([-0.01, 0.01], dtype=np.float32)
    tl = float(t[1])
    y = np.array([tl + 0.9e-6 * 0.5, tl + 1.1e-6 * 0.5, tl + 0.45e-6 * 0.5, 0.3])
    f = _flags_for(y, t, d_pad)
    assert list(f) == [True, False, True, False]
    # a floor of 1/d_pad (0.25) instead of 1/sqrt(d_pad) would not flag 0.9e-6 * 0.5 = 4.5e-7
    assert 0.9e-6 * 0.5 > 1e-6 * 0.25


def test_sign_band_uses_row_norms():
    # row norms 5, 1, 2; column norms sqrt(10), sqrt(20), 0: a band built on the wrong axis
    # would leave z_0 = 0.9e-6 * 5 * gamma (> 1e-6 * sqrt(10) * gamma) unflagged
    S = np.array([[3.0, 4.0, 0.0], [1.0, 0.0, 0.0], [0.0, 2.0, 0.0]])
    gamma = 0.5
    rows = np.array([5.0, 1.0, 2.0])
    z_in = 0.9e-6 * rows * gamma * np.array([1, -1, 1])
    z_out = 1.1e-6 * rows * gamma * np.array([-1, 1, -1])
    enc = dict(y=np.zeros((2, 4)), norm=np.ones(2), gamma=np.array([gamma, gamma]), z=np.vstack([z_in, z_out]))
    f = codec.boundary_flags(enc, np.array([0.0], dtype=np.float32), S)["signs"]
    assert f[0].all()
    assert not f[1].any()
    assert 0.9e-6 * 5 > 1e-6 * math.sqrt(10)
    # gamma scales the band: the same z with gamma = 0.25 is outside
    enc["gamma"] = np.array([0.25, 0.25])
    assert not codec.boundary_flags(enc, np.array([0.0], dtype=np.float32), S)["signs"][0].any()


def test_fp16_tie_band():
    tie = 1.0 + 2.0 ** -11                                     # halfway between fp16 1.0 and 1 + 2^-10
    vals = np.array([tie, tie + 0.5e-6, tie + 2e-6, tie - 2e-6, 1.0, 1.0 + 2.0 ** -10, 3.0 * 2.0 ** -20])
    enc = dict(y=np.zeros((len(vals), 4)), norm=vals, gamma=vals)
    f = codec.boundary_flags(enc, np.array([0.0], dtype=np.float32))
    expect = [True, True, False, False, False, False, False]
    assert list(f["norm"]) == expect
    assert list(f["rnorm"]) == expect


def _polar_enc(y):
    th, ps, radii = polar.polar(np.asarray(y, dtype=np.float64).reshape(1, -1))
    return dict(y=np.asarray(y, dtype=np.float64).reshape(1, -1), radii=radii)


def test_polar_level1_ray_distance():
    d_pad, w = 16, 2                                           # b1 = 3: level-1 boundaries every pi/4
    tabs = polar.tables(d_pad, w)
    y = np.zeros(d_pad)
    # pair 0: radius 1 at pi/4 + 0.9e-6 rad (distance 0.9e-6 * 1) -> flagged
    a = math.pi / 4 + 0.9e-6
    y[0], y[1] = math.cos(a), math.sin(a)
    # pair 1: radius 1 at pi/2 - 1.1e-6 -> not flagged
    a = math.pi / 2 - 1.1e-6
    y[2], y[3] = math.cos(a), math.sin(a)
    # pair 2: radius 0.01 below the floor 1/sqrt(16) = 0.25: band 2.5e-7 in distance
    r, a = 0.01, math.pi + 2.0e-5                              # distance 2e-7 -> flagged
    y[4], y[5] = r * math.cos(a), r * math.sin(a)
    r, a = 0.01, 3 * math.pi / 2 - 3.0e-5                      # distance 3e-7 -> not flagged
    y[6], y[7] = r * math.cos(a), r * math.sin(a)
    # pair 3: well inside a cell
    y[8], y[9] = math.cos(0.3), math.sin(0.3)
    f1, _ = polar.boundary_flags(_polar_enc(y), w, d_pad, tabs)
    assert list(f1[0, :5]) == [True, False, True, False, False]


def test_polar_higher_level_ray_distance():
    d_pad, w = 8, 3                                            # b2 = 2: level-2 thresholds t0 < t1 = pi/4 < t2
    tabs = polar.tables(d_pad, w)
    c2, t2 = tabs[1][0]
    t = float(t2[0])
    def pair_for(radius):                                      # a level-1 pair with this radius (angle 0)
        return [radius, 0.0]
    R, dlt = 0.8, 0.9e-6
    ra, rb = R * math.cos(t + dlt), R * math.sin(t + dlt)      # distance R*sin(0.9e-6) <= 1e-6 * R -> flagged
    R2, dlt2 = 0.6, -1.1e-6
    rc, rd = R2 * math.cos(t + dlt2), R2 * math.sin(t + dlt2)  # distance 1.1e-6 * R2 -> not flagged
    y = np.array(pair_for(ra) + pair_for(rb) + pair_for(rc) + pair_for(rd))
    _, fl = polar.boundary_flags(_polar_enc(y), w, d_pad, tabs)
    assert list(fl[0][0]) == [True, False]


def test_logits_gqa_index_map():
    d, Hkv, group, n = 128, 2, 2, 7
    c, _ = stored_codebook(d, 3)
    D = sign_flips(5, d)
    rng = np.random.default_rng(11)
    idx = rng.integers(0, 8, size=(Hkv * n, d)).astype(np.uint8)
    signs = rng.integers(0, 2, size=(Hkv * n, d)).astype(np.uint8)
    norms = rng.uniform(0.5, 3.0, Hkv * n)
    q = rng.standard_normal((Hkv * group, d))
    S = rng.standard_normal((d, d))
    got = estimate.logits_gqa(q, D, S, idx, signs, norms, np.zeros(Hkv * n), c, d, Hkv, group, n)
    kmse = estimate.dequant_mse(idx, norms, c, D, d)          # gamma = 0: the logit is <q, k_mse>
    for h in range(Hkv * group):
        g = h // group
        np.testing.assert_allclose(got[h], q[h] @ kmse[g * n:(g + 1) * n].T, rtol=1e-12, atol=1e-12)
    # the heads really differ (a map h % Hkv would be caught)
    assert not np.allclose(got[1], q[1] @ kmse[n:2 * n].T)


def test_decode_attention_index_map_and_lengths():
    d, B, Hkv, Hq, T = 128, 2, 2, 4, 6
    group = Hq // Hkv
    kc, _ = stored_codebook(d, 2)
    vc, _ = stored_codebook(d, 3)
    kD, vD = sign_flips(7, d), sign_flips(8, d)
    rng = np.random.default_rng(12)
    N = B * Hkv * T
    k_idx = rng.integers(0, 4, size=(N, d)).astype(np.uint8)
    k_sg = rng.integers(0, 2, size=(N, d)).astype(np.uint8)
    k_n = rng.uniform(0.5, 2.0, N) * 8.0
    v_idx = rng.integers(0, 8, size=(N, d)).astype(np.uint8)
    v_n = rng.uniform(0.5, 2.0, N)
    q = rng.standard_normal((B, Hq, d))
    seq_lens = [T, 3]
    S = rng.standard_normal((d, d))
    got = estimate.decode_attention(q, kD, S, k_idx, k_sg, k_n, np.zeros(N), kc, d, vD, v_idx, v_n, vc, d,
                                    seq_lens, Hq, Hkv, T)
    kmse = estimate.dequant_mse(k_idx, k_n, kc, kD, d)
    vhat = estimate.dequant_mse(v_idx, v_n, vc, vD, d)
    for b in range(B):
        for h in range(Hq):
            g = h // group
            rows = slice((b * Hkv + g) * T, (b * Hkv + g) * T + seq_lens[b])
            s = q[b, h] @ kmse[rows].T / math.sqrt(d)
            p = np.exp(s - s.max())
            p /= p.sum()
            np.testing.assert_allclose(got[b, h], p @ vhat[rows], rtol=1e-11, atol=1e-12)
    # sequence 1 is shorter than max_tokens: the trailing tokens must not count
    rows = slice((1 * Hkv + 0) * T, (1 * Hkv + 0) * T + T)
    s = q[1, 0] @ kmse[rows].T / math.sqrt(d)
    p = np.exp(s - s.max())
    p /= p.sum()
    assert not np.allclose(got[1, 0], p @ vhat[rows])


def test_f16_tie_flags_direct():
    tie = 2.0 ** -3 * (1.0 + 3 * 2.0 ** -11)                   # halfway between two fp16 values near 0.125
    f = codec.f16_tie_flags(np.array([tie, tie * (1 + 0.8e-6), tie * (1 + 1.2e-6), 0.125]))
    assert list(f) == [True, True, False, False]
