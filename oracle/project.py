"""Oracle: the K/V projection that feeds the quantize-on-write path.

Test infrastructure only: imported by tests/, the smoke check and bench.py's
CPU baseline, never by the library.

The fused path ("turboquant_plus" article, "01 turboquant_plus：介绍与详解",
the prefill path of the runtime port) codes the output of an attention layer's
K (or V) projection without storing it.  What it codes is what an unfused
layer would store and then quantize: k = x W_h^T for head h, rounded to bf16
(the cache dtype).  Here the sum is taken in float64 - every bf16 x bf16
product is exact in float64 and the sums of a few thousand of them are exact
to far below a bf16 ulp - and rounded once, to nearest, ties to even.
"""
import numpy as np


def bf16_round(v):
    """Nearest bfloat16 value of v (float64 in, float64 out), ties to even.

    bfloat16 keeps 8 significant bits: v = m * 2^e with 0.5 <= |m| < 1 is
    rounded at 2^(e-8).  Values beyond the bf16 range are not expected here.
    """
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)
    q = np.rint(m * 256.0)  # numpy rounds half to even
    return np.ldexp(q, e - 8)


def project(x, w, n_heads, d=128):
    """Vectors of every head in the path's order: row h * n_tok + t is
    bf16(x[t] . w[h*d : (h+1)*d]^T).  x [n_tok, hidden], w [n_heads*d, hidden]."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    n_tok = x.shape[0]
    out = np.empty((n_heads * n_tok, d), dtype=np.float64)
    for h in range(n_heads):
        out[h * n_tok:(h + 1) * n_tok] = x @ w[h * d:(h + 1) * d].T
    return bf16_round(out)


def project_exact(x, w, n_heads, d=128):
    """The unrounded sums and the sums of |products| (for rounding-tie flags), same order."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    n_tok = x.shape[0]
    s = np.empty((n_heads * n_tok, d))
    a = np.empty((n_heads * n_tok, d))
    for h in range(n_heads):
        wh = w[h * d:(h + 1) * d]
        s[h * n_tok:(h + 1) * n_tok] = x @ wh.T
        a[h * n_tok:(h + 1) * n_tok] = np.abs(x) @ np.abs(wh).T
    return s, a


def bf16_tie_flags(s, a, rel=2e-5):
    """Sums whose bf16 rounding an fp32 accumulation may take either way: the
    exact sum lies within rel * sum|products| of a rounding midpoint."""
    s = np.asarray(s, dtype=np.float64)
    lo = bf16_round(s - rel * a)
    hi = bf16_round(s + rel * a)
    return lo != hi
