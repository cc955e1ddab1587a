"""Pins of the polar-coordinate oracle (oracle/polar.py) against facts that do
not come from it: the transform's exact inverse, the level-2 angle law's
Lloyd-Max fixed point in closed form, Monte-Carlo angle laws of rotated
Gaussian vectors against the Beta law, nearest-centroid decisions by brute
force, the bit layout on a hand-made example, <q, x_hat> = logit, and the
stored angle tables against a 30-digit Newton solution (mpmath)."""
import math

import numpy as np
import pytest

from oracle import codec, params, polar


def _gauss(n, d, seed):
    return np.random.default_rng(seed).standard_normal((n, d))


def test_polar_round_trip():
    y = _gauss(64, 128, 1)
    th, ps, radii = polar.polar(y)
    assert np.allclose(radii[-1][:, 0], np.linalg.norm(y, axis=1), rtol=1e-14)
    assert np.max(np.abs(polar.unpolar(th, ps, radii[-1][:, 0]) - y)) < 1e-13
    assert np.all((th >= 0) & (th < 2 * math.pi))
    assert all(np.all((p >= 0) & (p <= math.pi / 2)) for p in ps)


def _level2_fixed_point(L):
    """Lloyd-Max on density sin(2 psi) over [0, pi/2] with the integrals in closed form:
    mass(a,b) = (cos 2a - cos 2b)/2, moment(a,b) = [-psi cos(2psi)/2 + sin(2psi)/4]_a^b."""
    c = (np.arange(L) + 0.5) * (math.pi / 2) / L
    F = lambda p: -p * np.cos(2 * p) / 2 + np.sin(2 * p) / 4
    for _ in range(20000):
        e = np.concatenate([[0.0], 0.5 * (c[:-1] + c[1:]), [math.pi / 2]])
        new = (F(e[1:]) - F(e[:-1])) / ((np.cos(2 * e[:-1]) - np.cos(2 * e[1:])) / 2)
        if np.max(np.abs(new - c)) < 1e-15:
            c = new
            break
        c = new
    return c


@pytest.mark.parametrize("L", [2, 4])
def test_level2_lloyd_closed_form(L):
    c, t = polar.lloyd_max_angle(2, L)
    ref = _level2_fixed_point(L)
    assert np.max(np.abs(c - ref)) < 1e-10
    if L == 2:  # centroid of [0, pi/4] under sin(2 psi): (1/4) / (1/2)
        assert abs(c[0] - 0.5) < 1e-12 and abs(t[0] - math.pi / 4) < 1e-12


def test_single_cell_is_pi_over_4():
    for lv in (2, 5, 7):
        c, t = polar.lloyd_max_angle(lv, 1)
        assert c.tolist() == [math.pi / 4] and t.size == 0


@pytest.mark.parametrize("w", [1, 2, 3])
def test_level1_uniform_table(w):
    b1, _ = polar.widths(w)
    c1, _ = polar.tables(128, w)
    L = 1 << b1
    assert np.array_equal(c1, ((np.arange(L) + 0.5) * (2 * math.pi / L)).astype(np.float32))


def test_angle_laws_match_monte_carlo():
    """Rotated Gaussian vectors (d_pad 128): level-1 angles uniform, level-l angles with
    sin^2 psi ~ Beta(2^(l-2), 2^(l-2)); Kolmogorov distance below 0.01."""
    D = params.sign_flips(42, 128)
    x = _gauss(4000, 128, 7)
    y = codec.rotate(x, D)
    th, ps, _ = polar.polar(y)
    s = np.sort(th.ravel())
    emp = np.arange(1, s.size + 1) / s.size
    assert np.max(np.abs(emp - s / (2 * math.pi))) < 0.01
    for lv, p in zip(range(2, 8), ps):
        s = np.sort(p.ravel())
        emp = np.arange(1, s.size + 1) / s.size
        ks = np.max(np.abs(emp - polar.AngleLaw(lv).cdf(s)))
        assert ks < 0.01 + 1.6 / math.sqrt(s.size), (lv, ks)
        # a wrong exponent (the law of level l - 1 or l + 1) is far off
        wrong = np.max(np.abs(emp - polar.AngleLaw(lv + 1).cdf(s)))
        assert wrong > 3 * ks


@pytest.mark.parametrize("w", [2, 3])
def test_decisions_are_nearest_centroids(w):
    D = params.sign_flips(42, 128)
    x = _gauss(300, 128, 3)
    tabs = polar.tables(128, w)
    enc = polar.encode(x, D, w, tabs)
    c1, per_level = tabs
    # level 1: nearest centroid on the circle
    c = c1.astype(np.float64)
    dist = np.abs(np.angle(np.exp(1j * (enc["theta"][:, :, None] - c[None, None, :]))))
    assert np.array_equal(np.argmin(dist, axis=2), enc["i1"])
    for psi, ix, (cc, _) in zip(enc["psis"], enc["ihi"], per_level):
        near = np.argmin(np.abs(psi[:, :, None] - cc.astype(np.float64)[None, None, :]), axis=2)
        # thresholds are fp32 midpoints of fp32 centroids: the two agree away from ties
        ok = (near == ix) | (np.abs(np.abs(psi - cc[near]) - np.abs(psi - cc[ix])) < 1e-6)
        assert np.all(ok)


def test_pack_layout_by_hand():
    """w = 2 (b1 = 3, b2 = 1), d_pad 8: 4 level-1 indices, then 2 + 1 one-bit indices."""
    i1 = np.array([[5, 3, 0, 7]])
    ihi = [np.array([[1, 0]]), np.array([[1]])]
    buf = polar.pack(i1, ihi, 2, 8)
    # bits: 101 110 000 111 | 1 0 | 1  -> LSB first
    bits = [1, 0, 1, 1, 1, 0, 0, 0, 0, 1, 1, 1, 1, 0, 1, 0]
    expect = [sum(bits[8 * k + j] << j for j in range(8)) for k in range(2)]
    assert buf.tolist() == [expect]
    a, b = polar.unpack(buf.ravel(), 1, 2, 8)
    assert np.array_equal(a, i1) and all(np.array_equal(u, v) for u, v in zip(b, ihi))


def test_exact_angles_reconstruct_and_logits_identity():
    D = params.sign_flips(42, 128)
    x = _gauss(50, 100, 5)
    q = _gauss(4, 100, 6)
    enc = polar.encode(x, D, 3)
    lg = polar.logits(q, D, enc["i1"], enc["ihi"], enc["norm_f16"], 3)
    xr = polar.dequantize(enc["i1"], enc["ihi"], enc["norm_f16"], D, 100, 3)
    assert np.max(np.abs(lg - q @ xr.T)) < 1e-10 * np.max(np.abs(lg))
    # unquantized angles give back the rotated unit vector
    yh = polar.unpolar(enc["theta"], enc["psis"], np.ones(50))
    assert np.max(np.abs(yh - enc["y"][:, :128])) < 1e-13


def test_distortion_falls_with_bits_and_zero_vector():
    D = params.sign_flips(42, 128)
    x = _gauss(400, 128, 9)
    x[0] = 0.0
    errs = []
    for w in (1, 2, 3):
        enc = polar.encode(x, D, w)
        xr = polar.dequantize(enc["i1"], enc["ihi"], enc["norm_f16"], D, 128, w)
        assert np.all(xr[0] == 0) and enc["norm"][0] == 0
        errs.append(np.mean(np.sum((xr[1:] - x[1:]) ** 2, 1) / np.sum(x[1:] ** 2, 1)))
    assert errs[0] > errs[1] > errs[2] and errs[2] < 0.05


def _mp_angle_fixed_point(level, L, start):
    """Lloyd-Max on (sin psi cos psi)^(k-1) over [0, pi/2] by Newton in 30 digits, mpmath quadrature."""
    import mpmath as mp
    mp.mp.dps = 30
    k = 1 << (level - 1)
    f = lambda t: (mp.sin(t) * mp.cos(t)) ** (k - 1)
    half = L // 2
    q = mp.pi / 4

    def residual(*up):  # centroids above pi/4; the law is symmetric about pi/4
        c = [2 * q - x for x in reversed(up)] + list(up)
        e = [mp.mpf(0)] + [(c[j] + c[j + 1]) / 2 for j in range(L - 1)] + [2 * q]
        return [c[j] - mp.quad(lambda t: t * f(t), [e[j], e[j + 1]]) / mp.quad(f, [e[j], e[j + 1]])
                for j in range(half, L)]

    sol = mp.findroot(residual, [mp.mpf(x) for x in start[half:]], tol=mp.mpf(10) ** -26)
    up = np.array([float(x) for x in (sol if hasattr(sol, "__len__") else [sol])])
    return np.concatenate([math.pi / 2 - up[::-1], up])


@pytest.mark.parametrize("level,L", [(2, 2), (2, 4), (4, 4), (7, 2), (7, 4)])
def test_angle_tables_match_high_precision(level, L):
    """The stored fp32 angle centroids are the fp32 rounding of a 30-digit Newton
    solution of the level's Lloyd-Max conditions (mpmath quadrature of the density)."""
    c, _ = polar.lloyd_max_angle(level, L)
    ref = _mp_angle_fixed_point(level, L, c)
    assert np.max(np.abs(c - ref)) < 1e-11
    assert np.array_equal(c.astype(np.float32), ref.astype(np.float32))


@pytest.mark.parametrize("w", [1, 2])
def test_prod_stage_unbiased_over_S_with_its_variance(w):
    """QJL on the polar residual: over Gaussian S the estimate averages to <q, x>
    with variance n^2 ((pi/2) gamma^2 ||q~||^2 - <q~, r>^2) / m."""
    from oracle.params import gaussian_normals_f64
    d, m, N = 128, 128, 3000
    rng = np.random.default_rng(20 + w)
    x = rng.standard_normal((1, d)) * 2.0
    q = rng.standard_normal((1, d))
    D = params.sign_flips(13, d)
    tabs = polar.tables(d, w)
    vals = []
    for s in range(N):
        S = gaussian_normals_f64(3000 + s, m, d)
        enc = polar.encode_prod(x, D, w, S, tabs)
        vals.append(polar.logits_prod(q, D, S, enc["yhat"], enc["signs"], enc["norm"], enc["gamma"], m)[0, 0])
    vals = np.array(vals)
    qt = codec.rotate(q, D)[0]
    n, g, r = enc["norm"][0], enc["gamma"][0], enc["r"][0]
    var = n * n * ((math.pi / 2) * g * g * (qt @ qt) - (qt @ r) ** 2) / m
    assert abs(vals.mean() - float(q[0] @ x[0])) < 4 * math.sqrt(var / N)
    assert abs(vals.var() / var - 1) < 4 * math.sqrt(2.0 / N)


def test_prod_stage_removes_the_stage1_shrinkage():
    """Over random rotations the polar stage-1 estimate alone shrinks <q, x> (its
    reconstruction is shorter on average than y along y); adding the QJL stage
    makes the estimate unbiased over (D, S)."""
    from oracle.params import gaussian_normals_f64
    d, m, N, w = 128, 128, 1500, 1
    rng = np.random.default_rng(31)
    x = rng.standard_normal((1, d))
    q = x + 0.3 * rng.standard_normal((1, d))
    tabs = polar.tables(d, w)
    s1, s2 = [], []
    for s in range(N):
        D = params.sign_flips(5000 + s, d)
        S = gaussian_normals_f64(7000 + s, m, d)
        enc = polar.encode_prod(x, D, w, S, tabs)
        s1.append(polar.logits(q, D, enc["i1"], enc["ihi"], enc["norm"], w, tabs)[0, 0])
        s2.append(polar.logits_prod(q, D, S, enc["yhat"], enc["signs"], enc["norm"], enc["gamma"], m)[0, 0])
    truth = float(q[0] @ x[0])
    s1, s2 = np.array(s1), np.array(s2)
    assert s1.mean() < truth - 8 * s1.std() / math.sqrt(N)              # biased low
    assert abs(s2.mean() - truth) < 4 * s2.std() / math.sqrt(N)           # unbiased
