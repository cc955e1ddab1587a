"""Pins of the oracle's Philox4x32-10 against the generator's published
known-answer vectors (tests/golden/philox4x32_10_kat.txt)."""
import os

import numpy as np
import pytest

from oracle.philox import philox4x32_10, stream_words

GOLD = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def _kat():
    rows = []
    for line in open(GOLD):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        v = [int(x, 16) for x in line.split()]
        rows.append((v[0:4], v[4:6], v[6:10]))
    return rows


@pytest.mark.parametrize("ctr,key,out", _kat())
def test_known_answers(ctr, key, out):
    got = philox4x32_10(np.array(ctr, dtype=np.uint64), key)
    assert [int(x) for x in got] == out


def test_stream_layout():
    # word w of stream s is lane w%4 of block w//4 with counter (w//4, s, 0, 0)
    seed = 0x0123456789ABCDEF
    w = stream_words(seed, 1, 10)
    blk2 = philox4x32_10(np.array([2, 1, 0, 0], dtype=np.uint64), (seed & 0xFFFFFFFF, seed >> 32))
    assert int(w[9]) == int(blk2[1])
    assert int(w[8]) == int(blk2[0])
