"""Python binding of the TurboQuant codec library (libtq.so, C ABI in include/tq.h).

Argument marshalling only: every step of quantization and estimation runs in
the library's CUDA kernels.  PyTorch supplies device memory and streams.
The functions keep the C names; tensors are passed by device pointer.

If libtq.so is missing this module raises at import: there is no fallback.
Build it with ``python vector_quantization_randomized_b200/build.py``.
"""
import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

TQ_OK, TQ_EINVAL, TQ_EUNSUPPORTED, TQ_ECUDA, TQ_ETIMEOUT = 0, -1, -2, -3, -4
TQ_MODE_PROD, TQ_MODE_MSE = 0, 1
TQ_F32, TQ_F16, TQ_BF16 = 0, 1, 2
TQ_LAYOUT_PLANES, TQ_LAYOUT_SLICED = 0, 1

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} not found: build it with `python vector_quantization_randomized_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)


class tq_params(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("d_pad", ctypes.c_int32), ("bits", ctypes.c_int32),
                ("mode", ctypes.c_int32), ("m", ctypes.c_int32), ("layout", ctypes.c_int32),
                ("centroids", ctypes.c_void_p), ("thresholds", ctypes.c_void_p),
                ("signs_D", ctypes.c_void_p), ("S", ctypes.c_void_p)]


class tq_polar_params(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("d_pad", ctypes.c_int32), ("w", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("tables", ctypes.c_void_p), ("signs_D", ctypes.c_void_p)]


_P = ctypes.POINTER(tq_params)
_PP = ctypes.POINTER(tq_polar_params)
_vp, _i32, _i64, _u64, _f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_float
_SIGS = {
    "tq_make_codebook": (_i32, [_i32, _i32, _vp, _vp]),
    "tq_make_params": (_i32, [_i32, _i32, _u64, _vp, _vp]),
    "tq_code_bytes": (_i64, [_i32, _i32, _i32, _i64]),
    "tq_quantize": (_i32, [_P, _vp, _i32, _i64, _i64, _vp, _vp, _vp, _vp]),
    "tq_project_quantize": (_i32, [_P, _vp, _i64, _i64, _i32, _vp, _i32, _i64, _vp, _vp, _vp, _vp, _i64, _vp]),
    "tq_dequantize": (_i32, [_P, _vp, _vp, _vp, _i64, _vp, _i64, _vp]),
    "tq_logits_workspace": (_i64, [_P, _i32]),
    "tq_logits": (_i32, [_P, _vp, _i32, _i32, _vp, _vp, _vp, _i64, _i32, _vp, _vp, _i64, _vp]),
    "tq_logits_ld": (_i32, [_P, _vp, _i32, _i32, _vp, _vp, _vp, _i64, _i32, _vp, _i64, _vp, _i64, _vp]),
    "tq_logits_noalloc_max_scratch": (_i64, []),
    "tq_logits_noalloc": (_i32, [_P, _vp, _i32, _i32, _vp, _vp, _vp, _i64, _i32, _vp, _vp]),
    "tq_decode_attn_workspace": (_i64, [_P, _i32, _i32, _i32, _i64]),
    "tq_decode_attn": (_i32, [_P, _P, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _f32, _vp,
                              _vp, _i64, _vp]),
    "tq_decode_attn_sparse": (_i32, [_P, _P, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _f32,
                                     _f32, _vp, _vp, _i64, _vp]),
    "tq_search_workspace": (_i64, [_P, _i32, _i64, _i32]),
    "tq_search_topk": (_i32, [_P, _vp, _i32, _vp, _vp, _vp, _i64, _i32, _vp, _vp, _vp, _i64, _vp]),
    "tq_decode_attn_partial_bytes": (_i64, [_P, _i32, _i32]),
    "tq_decode_attn_partial": (_i32, [_P, _P, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _f32, _vp,
                                      _vp, _i64, _vp]),
    "tq_decode_attn_merge": (_i32, [_P, _vp, _i32, _i32, _i32, _vp, _vp]),
    "tq_search_merge": (_i32, [_vp, _vp, _i32, _vp, _i32, _i32, _vp, _vp, _vp]),
    "tq_device_status": (_i32, [_i32]),
    "tq_diag_bounded_wait": (_i32, [_i64, _vp]),
    "tq_polar_table_floats": (_i64, [_i32, _i32]),
    "tq_polar_make_tables": (_i32, [_i32, _i32, _vp]),
    "tq_polar_code_bytes": (_i64, [_i32, _i32, _i64]),
    "tq_polar_quantize": (_i32, [_PP, _vp, _i32, _i64, _i64, _vp, _vp, _vp]),
    "tq_polar_dequantize": (_i32, [_PP, _vp, _vp, _i64, _vp, _i64, _vp]),
    "tq_polar_logits": (_i32, [_PP, _vp, _i32, _vp, _vp, _i64, _i32, _vp, _vp]),
    "tq_polar_qjl": (_i32, [_PP, _vp, _i32, _vp, _i32, _i64, _i64, _vp, _vp, _vp, _vp]),
    "tq_polar_logits_prod": (_i32, [_PP, _vp, _i32, _vp, _i32, _vp, _vp, _vp, _vp, _i64, _i32, _vp, _vp]),
    "tq_last_error": (ctypes.c_char_p, []),
    "tq_version": (_i32, []),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class TQError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{msg} (status {code})")
        self.code = code


def _check(rc):
    if rc != TQ_OK:
        raise TQError(rc, tq_last_error())
    return rc


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def tq_last_error():
    return _lib.tq_last_error().decode()


def tq_version():
    return _lib.tq_version()


def tq_device_status(clear=False):
    """Synchronize the device; TQ_OK, or TQ_ETIMEOUT if a bounded device wait gave up (message in tq_last_error)."""
    return _lib.tq_device_status(1 if clear else 0)


def tq_diag_bounded_wait(polls, stream=None):
    """Diagnostic: a kernel whose barrier wait runs out after `polls` polls (sets the diagnostic fault word)."""
    return _check(_lib.tq_diag_bounded_wait(polls, _stream(stream)))


def tq_make_codebook(d_pad, kb):
    """Host: Lloyd-Max codebook for the rotated-coordinate law -> (centroids, thresholds) fp32."""
    c = np.zeros(1 << kb, np.float32)
    t = np.zeros((1 << kb) - 1, np.float32)
    _check(_lib.tq_make_codebook(d_pad, kb, c.ctypes.data, t.ctypes.data))
    return c, t


def tq_make_params(d_pad, m, seed):
    """Host: sign flips D (int8) and QJL matrix S (fp16 bit patterns as uint16, m x d_pad)."""
    D = np.zeros(d_pad, np.int8)
    S = np.zeros((max(m, 1), d_pad), np.uint16)
    _check(_lib.tq_make_params(d_pad, m, seed, D.ctypes.data, S.ctypes.data if m else None))
    return D, (S if m else None)


def tq_code_bytes(d_pad, kb, m, n_vec):
    return _lib.tq_code_bytes(d_pad, kb, m, n_vec)


class Params:
    """A quantizer: host-made codebook/D/S copied to the device, plus the C struct."""

    def __init__(self, d, bits, mode=TQ_MODE_PROD, m=None, seed=42, d_pad=None, device="cuda", layout=0):
        import torch
        d_pad = d_pad or (128 if d <= 128 else 256)
        if mode == TQ_MODE_PROD and m is None:
            m = d_pad
        m = m if mode == TQ_MODE_PROD else 0
        self.d, self.d_pad, self.bits, self.mode, self.m, self.seed = d, d_pad, bits, mode, m, seed
        self.kb = bits - 1 if mode == TQ_MODE_PROD else bits
        c, t = tq_make_codebook(d_pad, self.kb)
        D, S = tq_make_params(d_pad, m, seed)
        self.host = dict(centroids=c, thresholds=t, D=D, S=S)
        self.centroids = torch.from_numpy(c).to(device)
        self.thresholds = torch.from_numpy(t).to(device)
        self.D = torch.from_numpy(D).to(device)
        self.S = torch.from_numpy(S.view(np.int16)).to(device) if m else None
        self.layout = layout
        self.struct = tq_params(d, d_pad, bits, mode, m, layout, _ptr(self.centroids), _ptr(self.thresholds),
                                _ptr(self.D), _ptr(self.S))

    @property
    def ref(self):
        return ctypes.byref(self.struct)

    def code_bytes(self, n_vec):
        return tq_code_bytes(self.d_pad, self.kb, self.m, n_vec)


def _dtype_code(x):
    import torch
    return {torch.float32: TQ_F32, torch.float16: TQ_F16, torch.bfloat16: TQ_BF16}[x.dtype]


def tq_quantize(p, x, codes, norms, rnorms=None, n_vec=None, ld=None, stream=None):
    """Encode rows of x (device tensor [n, ld] fp32/fp16/bf16) into codes/norms/rnorms."""
    n_vec = x.shape[0] if n_vec is None else n_vec
    ld = x.stride(0) if ld is None else ld
    return _check(_lib.tq_quantize(p.ref, _ptr(x), _dtype_code(x), n_vec, ld, _ptr(codes), _ptr(norms),
                                   _ptr(rnorms), _stream(stream)))


def tq_project_quantize(p, x, w, n_heads, codes, norms, rnorms=None, k_out=None, stream=None):
    """Fused K/V projection + encode: vectors bf16(x W_h^T) of every head h (x: device bf16
    [n_tok, hidden]; w: device bf16 [n_heads * 128, hidden]); vector h * n_tok + t is token t of
    head h.  k_out (optional, device bf16 [n_tok, >= n_heads * 128]) receives the projected rows."""
    return _check(_lib.tq_project_quantize(p.ref, _ptr(x), x.shape[0], x.stride(0), x.shape[1], _ptr(w), n_heads,
                                           w.stride(0), _ptr(codes), _ptr(norms), _ptr(rnorms), _ptr(k_out),
                                           k_out.stride(0) if k_out is not None else 0, _stream(stream)))


def tq_dequantize(p, codes, norms, rnorms, n_vec, out, ld=None, stream=None):
    """Reconstruction x_hat = Q^-1(codes) into out (device fp32 [n_vec, ld])."""
    ld = out.stride(0) if ld is None else ld
    return _check(_lib.tq_dequantize(p.ref, _ptr(codes), _ptr(norms), _ptr(rnorms), n_vec, _ptr(out), ld,
                                     _stream(stream)))


def tq_logits_workspace(p, n_q):
    return _lib.tq_logits_workspace(p.ref, n_q)


def tq_logits(p, q, group, codes, norms, rnorms, n_keys, n_kv_heads, logits, workspace, stream=None):
    return _check(_lib.tq_logits(p.ref, _ptr(q), q.shape[0], group, _ptr(codes), _ptr(norms), _ptr(rnorms),
                                 n_keys, n_kv_heads, _ptr(logits), _ptr(workspace), workspace.numel(),
                                 _stream(stream)))


def tq_logits_ld(p, q, group, codes, norms, rnorms, n_keys, n_kv_heads, logits, ld_logits, workspace, stream=None):
    """tq_logits writing query row h at logits + h*ld_logits (pass a column-offset view for a segment)."""
    return _check(_lib.tq_logits_ld(p.ref, _ptr(q), q.shape[0], group, _ptr(codes), _ptr(norms), _ptr(rnorms),
                                    n_keys, n_kv_heads, _ptr(logits), ld_logits, _ptr(workspace), workspace.numel(),
                                    _stream(stream)))


def tq_logits_noalloc_max_scratch():
    return _lib.tq_logits_noalloc_max_scratch()


def tq_logits_noalloc(p, q, group, codes, norms, rnorms, n_keys, n_kv_heads, logits, stream=None):
    """tq_logits with the library's static device scratch instead of a caller workspace."""
    return _check(_lib.tq_logits_noalloc(p.ref, _ptr(q), q.shape[0], group, _ptr(codes), _ptr(norms), _ptr(rnorms),
                                         n_keys, n_kv_heads, _ptr(logits), _stream(stream)))


def tq_decode_attn_workspace(kp, batch, n_q_heads, n_kv_heads, max_tokens):
    return _lib.tq_decode_attn_workspace(kp.ref, batch, n_q_heads, n_kv_heads, max_tokens)


def tq_decode_attn(kp, vp, q, n_kv_heads, kcodes, knorms, krnorms, vcodes, vnorms, seq_lens, max_tokens, out,
                   workspace, scale=0.0, stream=None):
    batch, n_q_heads = q.shape[0], q.shape[1]
    return _check(_lib.tq_decode_attn(kp.ref, vp.ref, _ptr(q), batch, n_q_heads, n_kv_heads, _ptr(kcodes),
                                      _ptr(knorms), _ptr(krnorms), _ptr(vcodes), _ptr(vnorms), _ptr(seq_lens),
                                      max_tokens, scale, _ptr(out), _ptr(workspace), workspace.numel(),
                                      _stream(stream)))


def tq_decode_attn_sparse(kp, vp, q, n_kv_heads, kcodes, knorms, krnorms, vcodes, vnorms, seq_lens, max_tokens,
                          out, workspace, v_eps, scale=0.0, stream=None):
    """tq_decode_attn with Sparse V: tokens whose attention weight is below v_eps add no value."""
    batch, n_q_heads = q.shape[0], q.shape[1]
    return _check(_lib.tq_decode_attn_sparse(kp.ref, vp.ref, _ptr(q), batch, n_q_heads, n_kv_heads, _ptr(kcodes),
                                             _ptr(knorms), _ptr(krnorms), _ptr(vcodes), _ptr(vnorms), _ptr(seq_lens),
                                             max_tokens, scale, v_eps, _ptr(out), _ptr(workspace),
                                             workspace.numel(), _stream(stream)))


def tq_search_workspace(p, n_q, n_db, k):
    return _lib.tq_search_workspace(p.ref, n_q, n_db, k)


def tq_search_topk(p, q, codes, norms, rnorms, n_db, k, ids, scores, workspace, stream=None):
    return _check(_lib.tq_search_topk(p.ref, _ptr(q), q.shape[0], _ptr(codes), _ptr(norms), _ptr(rnorms), n_db,
                                      k, _ptr(ids), _ptr(scores), _ptr(workspace), workspace.numel(),
                                      _stream(stream)))


# ---- sharded forms (one device per shard, see parallel.py) ---------------------
def tq_decode_attn_partial_bytes(vp, batch, n_q_heads):
    return _lib.tq_decode_attn_partial_bytes(vp.ref, batch, n_q_heads)


def tq_decode_attn_partial(kp, vp, q, n_kv_heads, kcodes, knorms, krnorms, vcodes, vnorms, seq_lens, max_tokens,
                           partial, workspace, scale=0.0, stream=None):
    """Decode attention over the tokens this caller holds, as an unnormalised partial
    (device fp32 [batch, n_q_heads, d_pad + 2]: o_rot, m, l) for tq_decode_attn_merge."""
    batch, n_q_heads = q.shape[0], q.shape[1]
    return _check(_lib.tq_decode_attn_partial(kp.ref, vp.ref, _ptr(q), batch, n_q_heads, n_kv_heads, _ptr(kcodes),
                                              _ptr(knorms), _ptr(krnorms), _ptr(vcodes), _ptr(vnorms),
                                              _ptr(seq_lens), max_tokens, scale, _ptr(partial), _ptr(workspace),
                                              workspace.numel(), _stream(stream)))


def tq_decode_attn_merge(vp, partials, out, stream=None):
    """Log-sum-exp merge of partials (device fp32 [n_parts, batch, n_q_heads, d_pad + 2]) into out [batch, n_q_heads, d]."""
    n_parts, batch, n_q_heads = partials.shape[0], partials.shape[1], partials.shape[2]
    return _check(_lib.tq_decode_attn_merge(vp.ref, _ptr(partials), n_parts, batch, n_q_heads, _ptr(out),
                                            _stream(stream)))


def tq_search_merge(ids, scores, id_offsets, k, out_ids, out_scores, stream=None):
    """Global top-k from per-shard lists ids/scores (device [n_parts, n_q, k]); id_offsets: the
    first global id of each shard (host sequence of n_parts ints)."""
    n_parts, n_q = ids.shape[0], ids.shape[1]
    offs = np.ascontiguousarray(np.asarray(id_offsets, dtype=np.int64))
    return _check(_lib.tq_search_merge(_ptr(ids), _ptr(scores), n_parts, offs.ctypes.data, n_q, k, _ptr(out_ids),
                                       _ptr(out_scores), _stream(stream)))


# ---- polar-coordinate stage 1 -------------------------------------------------
def tq_polar_make_tables(d_pad, w):
    """Host: the polar code's angle tables (fp32, layout of include/tq.h)."""
    n = _lib.tq_polar_table_floats(d_pad, w)
    if n < 0:
        raise TQError(TQ_EINVAL, "tq_polar_table_floats: bad arguments")
    t = np.zeros(n, np.float32)
    _check(_lib.tq_polar_make_tables(d_pad, w, t.ctypes.data))
    return t


def tq_polar_code_bytes(d_pad, w, n_vec):
    return _lib.tq_polar_code_bytes(d_pad, w, n_vec)


class PolarParams:
    """A polar-code quantizer: host-made tables and sign flips copied to the device, plus the C struct."""

    def __init__(self, d, w, seed=42, d_pad=None, device="cuda"):
        import torch
        d_pad = d_pad or (128 if d <= 128 else 256)
        self.d, self.d_pad, self.w, self.seed = d, d_pad, w, seed
        t = tq_polar_make_tables(d_pad, w)
        D, _ = tq_make_params(d_pad, 0, seed)
        self.host = dict(tables=t, D=D)
        self.tables = torch.from_numpy(t).to(device)
        self.D = torch.from_numpy(D).to(device)
        self.struct = tq_polar_params(d, d_pad, w, 0, _ptr(self.tables), _ptr(self.D))

    @property
    def ref(self):
        return ctypes.byref(self.struct)

    def code_bytes(self, n_vec):
        return tq_polar_code_bytes(self.d_pad, self.w, n_vec)


def tq_polar_quantize(p, x, codes, norms, n_vec=None, ld=None, stream=None):
    """Polar-code rows of x (device [n, ld] fp32/fp16/bf16) into codes / norms."""
    n_vec = x.shape[0] if n_vec is None else n_vec
    ld = x.stride(0) if ld is None else ld
    return _check(_lib.tq_polar_quantize(p.ref, _ptr(x), _dtype_code(x), n_vec, ld, _ptr(codes), _ptr(norms),
                                         _stream(stream)))


def tq_polar_dequantize(p, codes, norms, n_vec, out, ld=None, stream=None):
    ld = out.stride(0) if ld is None else ld
    return _check(_lib.tq_polar_dequantize(p.ref, _ptr(codes), _ptr(norms), n_vec, _ptr(out), ld, _stream(stream)))


def tq_polar_logits(p, q, group, codes, norms, n_keys, n_kv_heads, logits, stream=None):
    return _check(_lib.tq_polar_logits(p.ref, _ptr(q), group, _ptr(codes), _ptr(norms), n_keys, n_kv_heads,
                                       _ptr(logits), _stream(stream)))


def tq_polar_qjl(p, S, m, x, codes, signs, rnorms, n_vec=None, ld=None, stream=None):
    """QJL stage on the polar residual: sign bits of S r (device uint8 [n_vec * m / 8]) and gamma (fp16)."""
    n_vec = x.shape[0] if n_vec is None else n_vec
    ld = x.stride(0) if ld is None else ld
    return _check(_lib.tq_polar_qjl(p.ref, _ptr(S), m, _ptr(x), _dtype_code(x), n_vec, ld, _ptr(codes), _ptr(signs),
                                    _ptr(rnorms), _stream(stream)))


def tq_polar_logits_prod(p, S, m, q, group, codes, norms, signs, rnorms, n_keys, n_kv_heads, logits, stream=None):
    return _check(_lib.tq_polar_logits_prod(p.ref, _ptr(S), m, _ptr(q), group, _ptr(codes), _ptr(norms), _ptr(signs),
                                            _ptr(rnorms), n_keys, n_kv_heads, _ptr(logits), _stream(stream)))
