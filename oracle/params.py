"""Random parameters of the method: sign flips D and the QJL matrix S (TEST INFRASTRUCTURE).

"TurboQuant explainer" (m.163.com), "第一步：PolarQuant": a random rotation
is applied before quantization; zhidx turboquant_plus article: the rotation is
a Walsh-Hadamard rotation.  The plain reading used here: random sign flips D
(a diagonal of +-1) followed by the Sylvester Walsh-Hadamard matrix.
"第二步：QJL": a Johnson-Lindenstrauss projection of the residual; the plain
reading is a dense m x d_pad matrix of i.i.d. standard normals.

Readings where the pages are silent:
* Generator: Philox4x32-10 keyed by the 64-bit seed (low word, high word).
  Stream 0 gives D, stream 1 gives S.
* D_j = -1 when bit 0 of word j of stream 0 is set, else +1.
* S is row-major; entries 2p and 2p+1 are the Box-Muller pair made from
  words 2p and 2p+1 of stream 1: u = (w + 1/2) / 2^32,
  R = sqrt(-2 ln u_a), theta = 2 pi u_b, (R cos theta, R sin theta).
* S is stored rounded to IEEE half precision (round to nearest even).  Both
  sides use exactly these stored values; the tensor-core projection then has
  exact operands.
"""
import numpy as np

from .philox import stream_words


def sign_flips(seed, d_pad):
    """D as an int8 array of +-1, length d_pad."""
    w = stream_words(seed, 0, d_pad)
    return np.where((w & 1) != 0, -1, 1).astype(np.int8)


def gaussian_normals_f64(seed, m, d_pad):
    """The m x d_pad Box-Muller normals before rounding (fp64)."""
    n = m * d_pad
    n_even = n + (n & 1)
    w = stream_words(seed, 1, n_even).astype(np.float64)
    u = (w + 0.5) / 4294967296.0
    ua, ub = u[0::2], u[1::2]
    rad = np.sqrt(-2.0 * np.log(ua))
    th = 2.0 * np.pi * ub
    z = np.empty(n_even, dtype=np.float64)
    z[0::2] = rad * np.cos(th)
    z[1::2] = rad * np.sin(th)
    return z[:n].reshape(m, d_pad)


def qjl_matrix(seed, m, d_pad):
    """S as float16 (m x d_pad), the stored parameter."""
    return gaussian_normals_f64(seed, m, d_pad).astype(np.float16)
