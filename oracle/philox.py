"""Philox4x32-10, written from its published definition (TEST INFRASTRUCTURE).

Reference: J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw, "Parallel
Random Numbers: As Easy as 1, 2, 3", SC'11.  One round maps a counter
(c0, c1, c2, c3) under key (k0, k1) to

    (hi(M1*c2) ^ c1 ^ k0,  lo(M1*c2),  hi(M0*c0) ^ c3 ^ k1,  lo(M0*c0))

with M0 = 0xD2511F53, M1 = 0xCD9E8D57; between rounds the key is bumped by the
Weyl constants (0x9E3779B9, 0xBB67AE85).  Ten rounds.

Pinned by the generator's published known-answer vectors
(tests/golden/philox4x32_10_kat.txt).

The pages name no generator; using one counter-based generator on both sides
is how the random rotation and the QJL matrix are reproduced exactly.
"""
import numpy as np

M0 = np.uint64(0xD2511F53)
M1 = np.uint64(0xCD9E8D57)
W0 = 0x9E3779B9
W1 = 0xBB67AE85
MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr, key):
    """Apply Philox4x32-10 to counters.

    ctr: uint array of shape (..., 4); key: pair of ints (k0, k1).
    Returns uint32 array of shape (..., 4).
    """
    c = np.asarray(ctr, dtype=np.uint64) & MASK32
    c0, c1, c2, c3 = c[..., 0], c[..., 1], c[..., 2], c[..., 3]
    k0, k1 = int(key[0]) & 0xFFFFFFFF, int(key[1]) & 0xFFFFFFFF
    for rnd in range(10):
        if rnd > 0:
            k0 = (k0 + W0) & 0xFFFFFFFF
            k1 = (k1 + W1) & 0xFFFFFFFF
        p0 = M0 * c0          # < 2^64, exact in uint64
        p1 = M1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & MASK32
        c0, c1, c2, c3 = (hi1 ^ c1 ^ np.uint64(k0), lo1,
                          hi0 ^ c3 ^ np.uint64(k1), lo0)
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def stream_words(seed, stream, n_words):
    """First n_words 32-bit outputs of stream `stream` under 64-bit `seed`.

    Block i uses counter (i, stream, 0, 0) and key (seed low 32, seed high 32);
    word w of the stream is output lane w % 4 of block w // 4.
    """
    seed = int(seed)
    key = (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    n_blocks = (n_words + 3) // 4
    ctr = np.zeros((n_blocks, 4), dtype=np.uint64)
    ctr[:, 0] = np.arange(n_blocks, dtype=np.uint64)
    ctr[:, 1] = stream
    return philox4x32_10(ctr, key).reshape(-1)[:n_words]
