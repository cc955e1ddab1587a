"""Encoder and canonical code layout (TEST INFRASTRUCTURE).

Steps, in the order of "TurboQuant explainer" (m.163.com), "TurboQuant 怎么做的":

1. per-vector norm n = ||x|| and unit vector x/n ("第一步：PolarQuant": the
   rotated law is fixed, so no per-block normalisation constants are stored;
   the per-vector norm is the only scale, stored in fp16 - the zhidx
   turboquant_plus article's turbo4 format is 4.25 bit/value, which is what a
   3-bit code, a 128-sign sketch and two fp16 norms per 128 values give);
2. rotation y = H D x_hat / sqrt(d_pad): random sign flips D, then the
   Sylvester Walsh-Hadamard matrix H (natural order, H_ij = (-1)^popcount(i&j));
3. scalar code idx_j = #{l : y_j > t_l} with the stored Lloyd-Max thresholds
   (b-1 bits in the product mode, b bits in the MSE-only mode);
4. residual r = y - c[idx] and its norm gamma ("第二步：QJL");
5. QJL sign bits s_i = [ (S r)_i >= 0 ] (product mode only).

Readings: zero-padding to d_pad before the rotation; sign(0) = +1; a
coordinate exactly on a threshold goes to the lower cell; a zero vector keeps
n = 0 and x_hat = 0; norms are rounded to fp16 with round-to-nearest-even.

All arithmetic is fp64 except the stored fp32 codebook and fp16 S, which are
used as stored.

Canonical layout (part of the library's contract; unpacked here
independently):  vectors are grouped in tiles of 32; inside a tile come the
k_b bit-planes (plane p holds bit p of every index), each 32 x d_pad/8 bytes,
vector t at byte offset t*d_pad/8, coordinate j at bit j%32 of little-endian
32-bit word j//32; then the sign words, 32 x m/8 bytes, sign i at bit i%32 of
word i//32.  The last tile is zero-filled.  Norms and residual norms are
separate fp16 arrays indexed by vector.

Token-sliced layout (MSE codes only; the value cache read by the decode scan):
the same tiles of 32 vectors and the same k_b planes, but plane p of a tile
is d_pad little-endian 32-bit words, one per coordinate j in order, whose bit
t is bit p of the index of vector t of the tile at coordinate j.  Same bytes
per tile as the canonical layout; the last tile is zero-filled.
"""
import functools

import numpy as np

TILE = 32


@functools.lru_cache(maxsize=None)
def _hadamard_cached(d_pad):
    i = np.arange(d_pad)
    x = i[:, None] & i[None, :]
    pc = np.zeros_like(x)
    while np.any(x):
        pc += x & 1
        x >>= 1
    H = np.where(pc % 2 == 1, -1.0, 1.0)
    H.setflags(write=False)
    return H


def hadamard(d_pad):
    """Sylvester Hadamard matrix, natural order, entries (-1)^popcount(i & j)."""
    return _hadamard_cached(int(d_pad))


def rotate(v, D):
    """y = H (D o v) / sqrt(d_pad) for each row of v (already padded), fp64."""
    d_pad = D.shape[0]
    H = hadamard(d_pad)
    return (v * D.astype(np.float64)) @ H.T / np.sqrt(d_pad)


def unrotate(y, D):
    """Inverse of `rotate`: D o (H y) / sqrt(d_pad)  (H H^T = d_pad I, D D = I)."""
    d_pad = D.shape[0]
    H = hadamard(d_pad)
    return (y @ H) / np.sqrt(d_pad) * D.astype(np.float64)


def pad(x, d_pad):
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros((x.shape[0], d_pad), dtype=np.float64)
    out[:, :x.shape[1]] = x
    return out


def encode(x, D, centroids, thresholds, S=None):
    """Encode rows of x (n_vec x d, any float dtype; values taken exactly in fp64).

    Returns a dict with fp64 intermediates (norm, y, r, gamma, z) and stored
    results (idx uint8, signs uint8 0/1, norm_f16, rnorm_f16).
    """
    d_pad = D.shape[0]
    x = np.asarray(x).astype(np.float64)
    n = np.sqrt(np.sum(x * x, axis=1))
    safe = np.where(n > 0, n, 1.0)
    xh = np.where(n[:, None] > 0, x / safe[:, None], 0.0)
    y = rotate(pad(xh, d_pad), D)
    t = np.asarray(thresholds, dtype=np.float64)
    c = np.asarray(centroids, dtype=np.float64)
    idx = np.sum(y[:, :, None] > t[None, None, :], axis=2).astype(np.uint8)
    r = y - c[idx]
    gamma = np.sqrt(np.sum(r * r, axis=1))
    out = dict(norm=n, y=y, idx=idx, r=r, gamma=gamma,
               norm_f16=n.astype(np.float16), rnorm_f16=gamma.astype(np.float16))
    if S is not None:
        z = r @ np.asarray(S, dtype=np.float64).T
        out["z"] = z
        out["signs"] = (z >= 0).astype(np.uint8)
    return out


def boundary_flags(enc, thresholds, S=None, rel=1e-6):
    """Decisions that lie within `rel` of a boundary (the parity tolerance band).

    * index j of a vector: |y_j - t_l| <= rel * max(|t_l|, 1/sqrt(d_pad)) for some l
      (the scale is floored at the coordinate standard deviation because every
      even-level codebook has a threshold at exactly 0);
    * sign i: |z_i| <= rel * ||S_i|| * gamma;
    * fp16 norm / residual norm: the value is within `rel` (relative) of a
      half-precision rounding tie, i.e. fp16(v(1-rel)) != fp16(v(1+rel)).
    """
    y = enc["y"]
    d_pad = y.shape[1]
    t = np.asarray(thresholds, dtype=np.float64)
    scale = np.maximum(np.abs(t), 1.0 / np.sqrt(d_pad))
    idx_flag = np.any(np.abs(y[:, :, None] - t[None, None, :]) <= rel * scale[None, None, :], axis=2)

    flags = dict(idx=idx_flag, norm=f16_tie_flags(enc["norm"], rel), rnorm=f16_tie_flags(enc["gamma"], rel))
    if S is not None:
        Sn = np.sqrt(np.sum(np.asarray(S, dtype=np.float64) ** 2, axis=1))
        flags["signs"] = np.abs(enc["z"]) <= rel * Sn[None, :] * enc["gamma"][:, None]
    return flags


def f16_tie_flags(v, rel=1e-6):
    """Values within `rel` (relative) of a half-precision rounding tie:
    fp16(v(1-rel)) != fp16(v(1+rel)), so either rounding of v is acceptable."""
    v = np.asarray(v, dtype=np.float64)
    return (v * (1 - rel)).astype(np.float16) != (v * (1 + rel)).astype(np.float16)


def code_bytes(d_pad, kb, m, n_vec):
    """Bytes of a code buffer for n_vec vectors (whole tiles)."""
    n_tiles = (int(n_vec) + TILE - 1) // TILE
    return n_tiles * TILE * (kb * d_pad // 8 + m // 8)


def _bits_to_bytes(bits):
    """Rows of 0/1 -> little-endian bit-packed bytes (bit j%8 of byte j//8)."""
    return np.packbits(bits.astype(np.uint8), axis=1, bitorder="little")


def _bytes_to_bits(b, nbits):
    return np.unpackbits(b, axis=1, bitorder="little", count=nbits)


def pack(idx, signs, kb, m):
    """Canonical code buffer (uint8) from indices [n, d_pad] and signs [n, m] (or None)."""
    n, d_pad = idx.shape
    n_tiles = (n + TILE - 1) // TILE
    pb = d_pad // 8
    sb = m // 8
    tile_bytes = TILE * (kb * pb + sb)
    buf = np.zeros(n_tiles * tile_bytes, dtype=np.uint8)
    v = np.arange(n)
    tile, slot = v // TILE, v % TILE
    for p in range(kb):
        plane = _bits_to_bytes((idx >> p) & 1)                 # [n, pb]
        base = tile * tile_bytes + p * TILE * pb + slot * pb
        buf[base[:, None] + np.arange(pb)[None, :]] = plane
    if m:
        sbytes = _bits_to_bytes(signs)
        base = tile * tile_bytes + kb * TILE * pb + slot * sb
        buf[base[:, None] + np.arange(sb)[None, :]] = sbytes
    return buf


def unpack(buf, n, d_pad, kb, m):
    """Inverse of `pack`: returns (idx uint8 [n, d_pad], signs uint8 [n, m] or None)."""
    buf = np.asarray(buf, dtype=np.uint8)
    pb = d_pad // 8
    sb = m // 8
    tile_bytes = TILE * (kb * pb + sb)
    v = np.arange(n)
    tile, slot = v // TILE, v % TILE
    idx = np.zeros((n, d_pad), dtype=np.uint8)
    for p in range(kb):
        base = tile * tile_bytes + p * TILE * pb + slot * pb
        idx |= (_bytes_to_bits(buf[base[:, None] + np.arange(pb)[None, :]], d_pad) << p).astype(np.uint8)
    signs = None
    if m:
        base = tile * tile_bytes + kb * TILE * pb + slot * sb
        signs = _bytes_to_bits(buf[base[:, None] + np.arange(sb)[None, :]], m)
    return idx, signs


def pack_sliced(idx, kb):
    """Token-sliced code buffer (uint8) from MSE indices [n, d_pad]."""
    idx = np.asarray(idx, dtype=np.uint8)
    n, d_pad = idx.shape
    n_tiles = (n + TILE - 1) // TILE
    words = np.zeros((n_tiles, kb, d_pad), dtype=np.uint32)
    for v in range(n):
        tile, t = divmod(v, TILE)
        for p in range(kb):
            bits = ((idx[v] >> p) & 1).astype(np.uint32)
            words[tile, p] |= bits << np.uint32(t)
    return words.reshape(-1).astype("<u4").view(np.uint8).copy()


def unpack_sliced(buf, n, d_pad, kb):
    """Inverse of `pack_sliced`: indices uint8 [n, d_pad]."""
    n_tiles = (n + TILE - 1) // TILE
    words = np.asarray(buf, dtype=np.uint8)[:n_tiles * kb * d_pad * 4].view("<u4").reshape(n_tiles, kb, d_pad)
    idx = np.zeros((n, d_pad), dtype=np.uint8)
    for v in range(n):
        tile, t = divmod(v, TILE)
        for p in range(kb):
            idx[v] |= (((words[tile, p] >> np.uint32(t)) & 1) << p).astype(np.uint8)
    return idx
