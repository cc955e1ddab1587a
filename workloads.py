"""Seeded synthetic inputs (keys, values, queries, search sets).

This module holds only input generators: it contains none of the codec's
arithmetic, and both the library's tests/benchmarks and the independent
oracle draw their inputs from it.

Data law for keys/values (the pages give none; this is the stated workload):
    x[t, c] = z[t, c] * sigma_c * (20 if c in O else 1) * rho_t
    z ~ N(0, 1);  sigma_c = exp(N(0, 0.5^2)) once per channel;
    O = 4 distinct outlier channels (seeded permutation);
    rho_t = exp(N(0, 0.3^2)) per token (or 1 when token_scale is False).
Queries are N(0, 1).  Each (sequence, head) has its own generator stream
derived from (seed, sequence, head).

Projection inputs (the fused projection + quantize path): a layer input
x[t, k] = z[t, k] * rho_t (z ~ N(0, 1), rho_t = exp(N(0, 0.3^2))) and a
weight w[o, k] = z'[o, k] * sigma_o * (20 if o is an outlier row) / sqrt(hidden)
with 4 outlier output rows per head, both rounded to bf16, so that the
projected vectors follow the key law above (per-channel lognormal scales,
4 outlier channels, per-token norm multiplier).

Search set: x ~ N(0, Q diag(i^-0.8) Q^T), i = 1..d, Q a seeded Haar-random
orthogonal matrix (QR of a Gaussian matrix with the sign of R's diagonal
folded into Q), rows normalised to unit length.  It stands in for the GloVe
d=200 word vectors the search comparison used, which are not available here.
"""
import numpy as np

SEED_KEYS = 0
SEED_VALUES = 1
SEED_QUERIES = 2
SEED_PARAMS = 42


def _rng(*keys):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in keys])))


def to_bf16(x):
    """Round float32 values to the nearest bfloat16 (ties to even); returned as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).reshape(x.shape)


def head_vectors(n_tokens, d, seed, seq=0, head=0, token_scale=True):
    """One (sequence, head) block of keys or values: float32 [n_tokens, d]."""
    r = _rng(seed, seq, head)
    sigma = np.exp(r.normal(0.0, 0.5, size=d))
    outl = r.permutation(d)[:4]
    sigma[outl] *= 20.0
    rho = np.exp(r.normal(0.0, 0.3, size=n_tokens)) if token_scale else np.ones(n_tokens)
    z = r.standard_normal(size=(n_tokens, d), dtype=np.float32)
    return (z * sigma[None, :].astype(np.float32) * rho[:, None].astype(np.float32)).astype(np.float32)


def kv_block(n_seq, n_heads, n_tokens, d, seed, token_scale=True, bf16=True, seqs=None):
    """Keys or values for n_seq sequences x n_heads heads: float32 [n_seq, n_heads, n_tokens, d]
    (values exactly representable in bf16 when bf16=True).  `seqs` restricts to a subset
    of sequence indices (the result then has len(seqs) rows)."""
    seqs = range(n_seq) if seqs is None else seqs
    out = np.empty((len(seqs), n_heads, n_tokens, d), dtype=np.float32)
    for i, s in enumerate(seqs):
        for h in range(n_heads):
            v = head_vectors(n_tokens, d, seed, s, h, token_scale)
            out[i, h] = to_bf16(v) if bf16 else v
    return out


def projection_inputs(n_tok, hidden, n_heads, seed, d=128):
    """(x [n_tok, hidden], w [n_heads * d, hidden]): bf16-valued float32 arrays."""
    r = _rng(seed, 21, 21)
    rho = np.exp(r.normal(0.0, 0.3, size=n_tok)).astype(np.float32)
    x = to_bf16(r.standard_normal(size=(n_tok, hidden), dtype=np.float32) * rho[:, None])
    sig = np.exp(r.normal(0.0, 0.5, size=n_heads * d))
    for h in range(n_heads):
        sig[h * d + r.permutation(d)[:4]] *= 20.0
    w = r.standard_normal(size=(n_heads * d, hidden), dtype=np.float32)
    w = to_bf16(w * (sig / np.sqrt(hidden)).astype(np.float32)[:, None])
    return x, w


def queries(n, d, seed=SEED_QUERIES):
    """float32 [n, d] standard normal queries."""
    return _rng(seed, 0, 0).standard_normal(size=(n, d), dtype=np.float32)


def haar_orthogonal(d, seed):
    r = _rng(seed, 7, 7)
    a = r.standard_normal(size=(d, d))
    q, rr = np.linalg.qr(a)
    return q * np.sign(np.diag(rr))[None, :]


def search_set(n, d, seed, basis_seed=SEED_PARAMS + 1, decay=0.8, chunk=1 << 17):
    """float32 [n, d] unit vectors drawn from N(0, Q diag(i^-decay) Q^T)."""
    Q = haar_orthogonal(d, basis_seed)
    lam_sqrt = np.arange(1, d + 1, dtype=np.float64) ** (-decay / 2.0)
    A = (Q * lam_sqrt[None, :]).astype(np.float64)
    r = _rng(seed, 11, 11)
    out = np.empty((n, d), dtype=np.float32)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        z = r.standard_normal(size=(e - s, d))
        x = z @ A.T
        x /= np.linalg.norm(x, axis=1, keepdims=True)
        out[s:e] = x
    return out
