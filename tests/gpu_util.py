"""Shared helpers for the GPU parity tests: oracle-side parameters, the
decision-aware comparison of codes, and the logit tolerance.

Oracle inputs never come from the CUDA path: the oracle builds its own
codebook, D and S (tests/test_abi.py checks they equal the library's), and
decode-side tests feed codes produced by the oracle to both sides.
"""
import numpy as np
import torch

import vector_quantization_randomized_b200 as tq
from oracle import codec, estimate
from oracle.codebook import stored_codebook
from oracle.params import sign_flips, qjl_matrix


class OracleParams:
    def __init__(self, d, bits, mode, m, seed, d_pad):
        self.d, self.bits, self.mode, self.m, self.seed, self.d_pad = d, bits, mode, m, seed, d_pad
        self.kb = bits - 1 if mode == tq.TQ_MODE_PROD else bits
        self.c, self.t = stored_codebook(d_pad, self.kb)
        self.D = sign_flips(seed, d_pad)
        self.S = qjl_matrix(seed, m, d_pad) if m else None


def make_pair(d, bits, mode=tq.TQ_MODE_PROD, m=None, seed=42, layout=tq.TQ_LAYOUT_PLANES):
    d_pad = 128 if d <= 128 else 256
    if mode == tq.TQ_MODE_PROD and m is None:
        m = d_pad
    m = m if mode == tq.TQ_MODE_PROD else 0
    return tq.Params(d, bits, mode, m, seed, d_pad, layout=layout), OracleParams(d, bits, mode, m, seed, d_pad)


def gpu_quantize(p, x_t):
    """Run tq_quantize on device tensor x_t [n, >=d]; returns host (codes u8, norms f16, rnorms f16|None)."""
    n = x_t.shape[0]
    codes = torch.full((max(p.code_bytes(n), 16),), 0xAB, dtype=torch.uint8, device="cuda")
    norms = torch.zeros(n, dtype=torch.int16, device="cuda")
    rn = torch.zeros(n, dtype=torch.int16, device="cuda") if p.mode == tq.TQ_MODE_PROD else None
    tq.tq_quantize(p, x_t, codes, norms, rn)
    torch.cuda.synchronize()
    return (codes.cpu().numpy()[:p.code_bytes(n)], norms.cpu().numpy().view(np.float16),
            None if rn is None else rn.cpu().numpy().view(np.float16))


def f16_neighbours(a, b):
    """True where two fp16 arrays differ by at most one unit in the last place."""
    ai = a.view(np.int16).astype(np.int32)
    bi = b.view(np.int16).astype(np.int32)
    return np.abs(ai - bi) <= 1


def compare_codes(op, x, codes, norms, rnorms):
    """Compare GPU codes with the oracle's encoding of the same inputs.

    Bit-exact except decisions inside the tolerance band (flags); a vector
    whose index decision was flagged *and* differs has a different residual,
    so its signs and residual norm are not comparable and are counted instead.
    Returns a dict of counts; raises AssertionError on any unflagged mismatch.
    """
    n = x.shape[0]
    enc = codec.encode(x, op.D, op.c, op.t, op.S)
    fl = codec.boundary_flags(enc, op.t, op.S)
    idx, signs = codec.unpack(codes, n, op.d_pad, op.kb, op.m)
    # tail of the last tile must be zero
    n_tail = (-n) % 32
    if n_tail:
        i_all, s_all = codec.unpack(codes, n + n_tail, op.d_pad, op.kb, op.m)
        assert not np.any(i_all[n:]), "tail indices not zeroed"
        if op.m:
            assert not np.any(s_all[n:]), "tail signs not zeroed"
    dif = idx != enc["idx"]
    assert not np.any(dif & ~fl["idx"]), f"unflagged index mismatches: {np.argwhere(dif & ~fl['idx'])[:10]}"
    vec_changed = np.any(dif, axis=1)
    ok_n = (norms == enc["norm_f16"]) | (fl["norm"] & f16_neighbours(norms, enc["norm_f16"]))
    assert np.all(ok_n), f"norm mismatches at {np.argwhere(~ok_n)[:10].ravel()}"
    out = dict(n=n, idx_flagged=int(fl["idx"].sum()), idx_mismatch=int(dif.sum()),
               vectors_changed=int(vec_changed.sum()))
    if op.m:
        sd = (signs != enc["signs"]) & ~vec_changed[:, None]
        assert not np.any(sd & ~fl["signs"]), f"unflagged sign mismatches: {np.argwhere(sd & ~fl['signs'])[:10]}"
        ok_r = (rnorms == enc["rnorm_f16"]) | (fl["rnorm"] & f16_neighbours(rnorms, enc["rnorm_f16"])) | vec_changed
        assert np.all(ok_r), f"residual norm mismatches at {np.argwhere(~ok_r)[:10].ravel()}"
        out.update(sign_flagged=int(fl["signs"].sum()), sign_mismatch=int(sd.sum()))
    return out


def compare_codes_sliced(op, x, codes, norms):
    """compare_codes for MSE codes in the token-sliced layout (unpacked by the oracle)."""
    n = x.shape[0]
    enc = codec.encode(x, op.D, op.c, op.t, None)
    fl = codec.boundary_flags(enc, op.t, None)
    n_tail = (-n) % 32
    idx_all = codec.unpack_sliced(codes, n + n_tail, op.d_pad, op.kb)
    assert not np.any(idx_all[n:]), "tail indices not zeroed"
    idx = idx_all[:n]
    dif = idx != enc["idx"]
    assert not np.any(dif & ~fl["idx"]), f"unflagged index mismatches: {np.argwhere(dif & ~fl['idx'])[:10]}"
    ok_n = (norms == enc["norm_f16"]) | (fl["norm"] & f16_neighbours(norms, enc["norm_f16"]))
    assert np.all(ok_n), f"norm mismatches at {np.argwhere(~ok_n)[:10].ravel()}"
    return dict(n=n, idx_flagged=int(fl["idx"].sum()), idx_mismatch=int(dif.sum()))


def oracle_codes(op, x):
    """Oracle encoding packed in the canonical layout: (codes u8, norms f16, rnorms f16|None, enc)."""
    enc = codec.encode(x, op.D, op.c, op.t, op.S)
    buf = codec.pack(enc["idx"], enc.get("signs"), op.kb, op.m)
    return buf, enc["norm_f16"], (enc["rnorm_f16"] if op.m else None), enc


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype) if t.dtype.itemsize == torch.empty((), dtype=dtype).element_size() else t.to(dtype)
    return t.cuda()


def logit_tolerance(ref, norm_f16, q):
    """|delta| <= 1e-4 |l| + 1e-5 n ||q||  (relative 1e-4; the absolute 1e-5 is
    taken in units of ||q|| ||k||, i.e. on the cosine, since raw logits carry the
    arbitrary scale n ||q||)."""
    qn = np.linalg.norm(np.asarray(q, dtype=np.float64), axis=1)
    return 1e-4 * np.abs(ref) + 1e-5 * qn[:, None] * norm_f16.astype(np.float64)[None, :]
