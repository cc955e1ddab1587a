"""Polar-coordinate code of the rotated vector (TEST INFRASTRUCTURE).

"TurboQuant explainer" (m.163.com), "第一步：PolarQuant" and the same page's
"它到底怎么做到的？ / 第一步：PolarQuant —— 换个坐标系压缩": after a random
rotation the vector is rewritten in polar form, a radius and angles; in high
dimension the angles follow a known, highly concentrated Beta law, so they are
coded with fixed, precomputed tables and no normalisation constant is stored.

The pages give no formulas.  Readings taken here:

* Rotation: the same sign flips and Walsh-Hadamard rotation as the scalar code
  (codec.rotate) of the unit vector x/||x||; the radius kept is ||x|| (fp16),
  as in the scalar code.
* Polar form: recursive on pairs.  Level 1 pairs coordinates (2i, 2i+1):
  radius hypot(y_2i, y_2i+1) and full angle theta = atan2(y_2i+1, y_2i) in
  [0, 2 pi).  Level l >= 2 pairs the level-(l-1) radii (2i, 2i+1): radius
  hypot(r_2i, r_2i+1) and angle psi = atan2(r_2i+1, r_2i) in [0, pi/2].  The
  last level leaves one radius, ||y|| = 1.
* Angle laws for a uniformly random direction (the rotated vector's law):
  theta is uniform on [0, 2 pi); at level l >= 2 each radius covers
  k = 2^(l-1) coordinates, so sin^2 psi ~ Beta(k/2, k/2) - the "Beta law" of
  the page - with density 2 sin^(k-1) psi cos^(k-1) psi / B(k/2, k/2).
* Tables: Lloyd-Max per level.  For the uniform law on the circle the equal
  cells [2 pi j / L, 2 pi (j+1) / L) with centroids at their middles are a
  fixed point; for l >= 2 the Lloyd iteration on the density above.
* Bit budget: w bits per coordinate in all (the page's b-1 bits of stage 1);
  a level-1 angle (two coordinates) gets b1 = w + 1 bits, a higher-level angle
  b2 = w - 1 bits (w = 1: none; such an angle is decoded at the centroid of
  the whole range, pi/4).  Total b1 d/2 + b2 (d/2 - 1) <= w d bits.
* Decisions: theta -> floor(theta L1 / 2 pi); psi -> #{t : psi > t} (a value
  on a threshold goes to the lower cell, as in the scalar code).
* Record layout (per vector, w d_pad / 8 bytes, vectors consecutive): one
  little-endian bit stream, LSB first: the d_pad/2 level-1 indices (b1 bits
  each, pair order), then level 2 (d_pad/4 indices), ..., the last level
  (1 index), b2 bits each; unused bits zero.

All arithmetic is fp64; the tables are used as stored (fp32).
"""
import math

import numpy as np
from scipy import integrate, special

from . import codec


def widths(w):
    """(b1, b2): bits of a level-1 angle and of a higher-level angle for w bits per coordinate."""
    w = int(w)
    if not 1 <= w <= 3:
        raise ValueError("w must be 1..3")
    return w + 1, w - 1


def levels(d_pad):
    lv = int(d_pad).bit_length() - 1
    if 1 << lv != d_pad or lv < 2:
        raise ValueError("d_pad must be a power of two >= 4")
    return lv


class AngleLaw:
    """Law of psi = atan2(|u|, |v|) for two independent blocks of k = 2^(l-1) Gaussian coordinates."""

    def __init__(self, level):
        self.level = int(level)
        self.k = 1 << (self.level - 1)
        self.a = self.k / 2.0
        self.logC = math.log(2.0) - special.betaln(self.a, self.a)

    def pdf(self, psi):
        psi = np.asarray(psi, dtype=np.float64)
        s, c = np.sin(psi), np.cos(psi)
        with np.errstate(divide="ignore"):
            return np.exp(self.logC + (self.k - 1) * (np.log(s) + np.log(c)))

    def cdf(self, psi):
        return special.betainc(self.a, self.a, np.sin(np.asarray(psi, dtype=np.float64)) ** 2)

    def cell(self, lo, hi):
        """(mass, first moment) of the cell (lo, hi] by adaptive quadrature."""
        mass = self.cdf(hi) - self.cdf(lo)
        mom = integrate.quad(lambda t: t * float(self.pdf(t)), lo, hi, epsabs=0, epsrel=1e-13, limit=200)[0]
        return mass, mom


def lloyd_max_angle(level, n_cells, tol=1e-13, max_iter=10000):
    """Lloyd-Max centroids and thresholds (fp64) of the level-`level` angle law on [0, pi/2]."""
    law = AngleLaw(level)
    L = int(n_cells)
    if L == 1:
        return np.array([math.pi / 4]), np.zeros(0)
    # start from the quantiles of the law; the law is symmetric about pi/4, so is the fixed point
    q = (np.arange(L) + 0.5) / L
    c = np.arcsin(np.sqrt(special.betaincinv(law.a, law.a, q)))
    for _ in range(max_iter):
        t = 0.5 * (c[:-1] + c[1:])
        edges = np.concatenate([[0.0], t, [math.pi / 2]])
        new = np.empty(L)
        for j in range(L):
            mass, mom = law.cell(edges[j], edges[j + 1])
            new[j] = mom / mass
        new = 0.5 * (new + (math.pi / 2 - new[::-1]))  # symmetry about pi/4
        step = np.max(np.abs(new - c))
        c = new
        if step < tol:
            break
    else:
        raise RuntimeError("angle Lloyd-Max did not converge")
    return c, 0.5 * (c[:-1] + c[1:])


def tables(d_pad, w):
    """Stored tables (fp32): level-1 centroids [L1]; per level 2..LV centroids [L2] and thresholds [L2-1]."""
    b1, b2 = widths(w)
    L1, L2 = 1 << b1, 1 << b2
    c1 = ((np.arange(L1) + 0.5) * (2 * math.pi / L1)).astype(np.float32)
    per_level = []
    for lv in range(2, levels(d_pad) + 1):
        c, _ = lloyd_max_angle(lv, L2)
        c32 = c.astype(np.float32)
        t32 = (0.5 * (c32[:-1].astype(np.float64) + c32[1:].astype(np.float64))).astype(np.float32)
        per_level.append((c32, t32))
    return c1, per_level


def polar(y):
    """Recursive polar form of rows of y: (theta [n, d/2], psi list per level 2.., radii list per level 1..)."""
    y = np.asarray(y, dtype=np.float64)
    a, b = y[:, 0::2], y[:, 1::2]
    theta = np.mod(np.arctan2(b, a), 2 * math.pi)
    r = np.hypot(a, b)
    radii, psis = [r], []
    while r.shape[1] > 1:
        ra, rb = r[:, 0::2], r[:, 1::2]
        psis.append(np.arctan2(rb, ra))
        r = np.hypot(ra, rb)
        radii.append(r)
    return theta, psis, radii


def unpolar(theta, psis, top):
    """Inverse of `polar`: rows of y from the angles and the top radius [n]."""
    r = np.asarray(top, dtype=np.float64)[:, None]
    for psi in reversed(psis):
        out = np.empty((r.shape[0], 2 * r.shape[1]))
        out[:, 0::2] = r * np.cos(psi)
        out[:, 1::2] = r * np.sin(psi)
        r = out
    y = np.empty((r.shape[0], 2 * r.shape[1]))
    y[:, 0::2] = r * np.cos(theta)
    y[:, 1::2] = r * np.sin(theta)
    return y


def encode(x, D, w, tabs=None):
    """Encode rows of x (n x d): norm, rotated unit vector, level-1 and higher-level indices."""
    d_pad = D.shape[0]
    b1, b2 = widths(w)
    L1 = 1 << b1
    c1, per_level = tabs if tabs is not None else tables(d_pad, w)
    x = np.asarray(x).astype(np.float64)
    n = np.sqrt(np.sum(x * x, axis=1))
    safe = np.where(n > 0, n, 1.0)
    xh = np.where(n[:, None] > 0, x / safe[:, None], 0.0)
    y = codec.rotate(codec.pad(xh, d_pad), D)
    theta, psis, radii = polar(y)
    i1 = np.minimum(np.floor(theta * (L1 / (2 * math.pi))).astype(np.int64), L1 - 1)
    ihi = []
    for psi, (c, t) in zip(psis, per_level):
        ihi.append(np.sum(psi[:, :, None] > t.astype(np.float64)[None, None, :], axis=2).astype(np.int64))
    return dict(norm=n, norm_f16=n.astype(np.float16), y=y, theta=theta, psis=psis, radii=radii,
                i1=i1, ihi=ihi)


def decode_unit(i1, ihi, w, d_pad, tabs=None):
    """y_hat (unit radius) from the indices, with the stored tables."""
    c1, per_level = tabs if tabs is not None else tables(d_pad, w)
    th = c1.astype(np.float64)[i1]
    ps = [c.astype(np.float64)[ix] for ix, (c, _) in zip(ihi, per_level)]
    return unpolar(th, ps, np.ones(i1.shape[0]))


def dequantize(i1, ihi, norm_f16, D, d, w, tabs=None):
    """x_hat = n D H y_hat / sqrt(d_pad), first d coordinates."""
    yh = decode_unit(i1, ihi, w, D.shape[0], tabs)
    return (codec.unrotate(yh, D) * norm_f16.astype(np.float64)[:, None])[:, :d]


def logits(q, D, i1, ihi, norm_f16, w, tabs=None):
    """l[h, k] = n_k <q~_h, y_hat_k>, q~ = H D q / sqrt(d_pad) (= <q, x_hat_k>)."""
    d_pad = D.shape[0]
    qt = codec.rotate(codec.pad(q, d_pad), D)
    yh = decode_unit(i1, ihi, w, d_pad, tabs)
    return (qt @ yh.T) * norm_f16.astype(np.float64)[None, :]


def boundary_flags(enc, w, d_pad, tabs=None, rel=1e-6):
    """Decisions within `rel` of a boundary: the point's distance to the boundary ray is at
    most rel * max(its radius, 1/sqrt(d_pad)).  Returns (flag1 [n, d/2], flags per level)."""
    b1, _ = widths(w)
    L1 = 1 << b1
    c1, per_level = tabs if tabs is not None else tables(d_pad, w)
    floor_ = 1.0 / math.sqrt(d_pad)
    y = enc["y"]
    a, b = y[:, 0::2], y[:, 1::2]
    r1 = np.hypot(a, b)
    phi = np.arange(L1) * (2 * math.pi / L1)
    dist = np.abs(a[:, :, None] * np.sin(phi) - b[:, :, None] * np.cos(phi))
    f1 = np.any(dist <= rel * np.maximum(r1, floor_)[:, :, None], axis=2)
    fl = []
    for lv, (c, t) in enumerate(per_level):
        r = enc["radii"][lv]
        ra, rb = r[:, 0::2], r[:, 1::2]
        R = np.hypot(ra, rb)
        if t.size == 0:
            fl.append(np.zeros(ra.shape, dtype=bool))
            continue
        tt = t.astype(np.float64)
        dd = np.abs(ra[:, :, None] * np.sin(tt) - rb[:, :, None] * np.cos(tt))
        fl.append(np.any(dd <= rel * np.maximum(R, floor_)[:, :, None], axis=2))
    return f1, fl


def record_bytes(d_pad, w):
    """Bytes of one record: w * d_pad bits, rounded up to whole bytes (exact for d_pad >= 8)."""
    return (int(w) * int(d_pad) + 7) // 8


def pack(i1, ihi, w, d_pad):
    """Records (uint8 [n, w d_pad / 8]) from the indices."""
    b1, b2 = widths(w)
    n = i1.shape[0]
    nbits = record_bytes(d_pad, w) * 8
    bits = np.zeros((n, nbits), dtype=np.uint8)
    pos = 0
    for j in range(i1.shape[1]):
        for k in range(b1):
            bits[:, pos] = (i1[:, j] >> k) & 1
            pos += 1
    for ix in ihi:
        for j in range(ix.shape[1]):
            for k in range(b2):
                bits[:, pos] = (ix[:, j] >> k) & 1
                pos += 1
    return np.packbits(bits, axis=1, bitorder="little")


def unpack(buf, n, w, d_pad):
    """Inverse of `pack`: (i1 [n, d/2], list of per-level indices)."""
    b1, b2 = widths(w)
    rb = record_bytes(d_pad, w)
    raw = np.asarray(buf, dtype=np.uint8)[: n * rb].reshape(n, rb)
    bits = np.unpackbits(raw, axis=1, bitorder="little").astype(np.int64)
    pos = 0
    i1 = np.zeros((n, d_pad // 2), dtype=np.int64)
    for j in range(d_pad // 2):
        for k in range(b1):
            i1[:, j] |= bits[:, pos] << k
            pos += 1
    ihi = []
    cnt = d_pad // 4
    while cnt >= 1:
        ix = np.zeros((n, cnt), dtype=np.int64)
        for j in range(cnt):
            for k in range(b2):
                ix[:, j] |= bits[:, pos] << k
                pos += 1
        ihi.append(ix)
        cnt //= 2
    return i1, ihi


# ---- QJL stage on the polar residual --------------------------------------------
# "TurboQuant explainer" (m.163.com), "第二步：QJL" and "合起来": the residual of
# stage 1 is JL-projected and kept as sign bits, and the estimator
# E[<y, Q^-1(Q(x))>] = <y, x> is unbiased; b - 1 bits of stage 1 plus 1 bit.
# Here stage 1 is the polar code: r = y - y_hat with y_hat the unit-radius
# reconstruction from the stored tables.

def encode_prod(x, D, w, S, tabs=None):
    """Polar stage 1 plus the QJL stage: adds y_hat, r, gamma (fp64 and fp16), z = S r, signs [z >= 0]."""
    enc = encode(x, D, w, tabs)
    yh = decode_unit(enc["i1"], enc["ihi"], w, D.shape[0], tabs)
    r = enc["y"] - yh
    gamma = np.sqrt(np.sum(r * r, axis=1))
    z = r @ np.asarray(S, dtype=np.float64).T
    enc.update(yhat=yh, r=r, gamma=gamma, rnorm_f16=gamma.astype(np.float16), z=z, signs=(z >= 0).astype(np.uint8))
    return enc


def logits_prod(q, D, S, yhat, signs, norm, gamma, m):
    """l[h, k] = n_k (<q~_h, y_hat_k> + gamma_k sqrt(pi/2)/m <S q~_h, 2 s_k - 1>), q~ = H D q / sqrt(d_pad)."""
    d_pad = D.shape[0]
    qt = codec.rotate(codec.pad(q, d_pad), D)
    u = qt @ np.asarray(S, dtype=np.float64).T
    pm = 2.0 * np.asarray(signs, dtype=np.float64) - 1.0
    corr = (u @ pm.T) * (math.sqrt(math.pi / 2.0) / m) * np.asarray(gamma, dtype=np.float64)[None, :]
    return (qt @ np.asarray(yhat, dtype=np.float64).T + corr) * np.asarray(norm, dtype=np.float64)[None, :]
