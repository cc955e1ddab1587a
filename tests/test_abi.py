"""CPU checks of the C ABI library: it loads, exports every function that
include/tq.h declares, its host-side functions agree with the oracle, and
argument validation rejects bad calls before anything reaches the GPU."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import vector_quantization_randomized_b200 as tq
from oracle.codebook import stored_codebook
from oracle.params import sign_flips, qjl_matrix
from oracle import codec

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tq.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 12
    out = subprocess.check_output(["nm", "-D", "--defined-only", tq.LIB_PATH]).decode()
    exported = set(re.findall(r" T (tq_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(tq.LIB_PATH)
    for n in names:
        assert getattr(lib, n) is not None


def test_version():
    assert tq.tq_version() >= 100


@pytest.mark.parametrize("d_pad", [16, 128, 256])
@pytest.mark.parametrize("kb", [1, 2, 3, 4])
def test_codebook_matches_independent_oracle_solver(d_pad, kb):
    c, t = tq.tq_make_codebook(d_pad, kb)
    co, to = stored_codebook(d_pad, kb)
    np.testing.assert_array_equal(c, co)
    np.testing.assert_array_equal(t, to)


@pytest.mark.parametrize("d_pad,m,seed", [(128, 128, 42), (256, 256, 7), (128, 64, 2 ** 40 + 3), (128, 0, 1)])
def test_params_match_oracle_generator(d_pad, m, seed):
    D, S = tq.tq_make_params(d_pad, m, seed)
    np.testing.assert_array_equal(D, sign_flips(seed, d_pad))
    if m:
        np.testing.assert_array_equal(S.view(np.float16), qjl_matrix(seed, m, d_pad))


def test_code_bytes():
    for (d_pad, kb, m, n) in [(128, 3, 128, 1), (128, 2, 128, 4097), (256, 1, 256, 10 ** 6), (128, 3, 0, 33)]:
        assert tq.tq_code_bytes(d_pad, kb, m, n) == codec.code_bytes(d_pad, kb, m, n)


def _fake_params(**kw):
    p = dict(d=128, d_pad=128, bits=4, mode=tq.TQ_MODE_PROD, m=128, layout=tq.TQ_LAYOUT_PLANES)
    p.update(kw)
    buf = np.zeros(64, np.float32)
    ptr = buf.ctypes.data
    st = tq.tq_params(p["d"], p["d_pad"], p["bits"], p["mode"], p["m"], p["layout"], ptr, ptr, ptr, ptr)
    return st, buf


@pytest.mark.parametrize("kw,code", [
    (dict(d_pad=64), tq.TQ_EUNSUPPORTED),
    (dict(d=0), tq.TQ_EINVAL),
    (dict(d=129), tq.TQ_EINVAL),
    (dict(bits=5), tq.TQ_EINVAL),
    (dict(bits=1), tq.TQ_EINVAL),
    (dict(m=48), tq.TQ_EINVAL),
    (dict(mode=7), tq.TQ_EINVAL),
    (dict(mode=tq.TQ_MODE_MSE, m=128), tq.TQ_EINVAL),
    (dict(layout=7), tq.TQ_EINVAL),                                     # unknown layout
    (dict(layout=tq.TQ_LAYOUT_SLICED), tq.TQ_EINVAL),                   # sliced holds MSE codes only
])
def test_validation_rejects_bad_params(kw, code):
    st, keep = _fake_params(**kw)
    lib = tq._lib
    rc = lib.tq_quantize(ctypes.byref(st), None, tq.TQ_BF16, 10, 128, None, None, None, None)
    assert rc == code
    assert tq.tq_last_error()


def test_validation_rejects_null_and_misaligned():
    st, keep = _fake_params()
    lib = tq._lib
    buf = np.zeros(1024, np.uint8)
    base = buf.ctypes.data
    base16 = (base + 15) // 16 * 16
    # NULL input
    assert lib.tq_quantize(ctypes.byref(st), None, tq.TQ_BF16, 10, 128, base16, base16, base16, None) == tq.TQ_EINVAL
    # misaligned x
    assert lib.tq_quantize(ctypes.byref(st), base16 + 2, tq.TQ_BF16, 10, 128, base16, base16, base16,
                           None) == tq.TQ_EINVAL
    # ld < d
    assert lib.tq_quantize(ctypes.byref(st), base16, tq.TQ_BF16, 10, 64, base16, base16, base16, None) == tq.TQ_EINVAL
    # bad dtype
    assert lib.tq_quantize(ctypes.byref(st), base16, 9, 10, 128, base16, base16, base16, None) == tq.TQ_EINVAL
    # n_vec == 0 is a no-op that touches nothing
    assert lib.tq_quantize(ctypes.byref(st), None, tq.TQ_BF16, 0, 128, None, None, None, None) == tq.TQ_OK
    # logits: n_q != heads*group
    assert lib.tq_logits(ctypes.byref(st), base16, 5, 4, base16, base16, base16, 100, 1, base16, base16, 1 << 20,
                         None) == tq.TQ_EINVAL
    # logits: workspace too small
    assert lib.tq_logits(ctypes.byref(st), base16, 4, 4, base16, base16, base16, 100, 1, base16, base16, 16,
                         None) == tq.TQ_EINVAL
    # logits: unsupported shape (d_pad 256 with 3 index bits takes MSE codes or m = 256)
    st2, keep2 = _fake_params(d=200, d_pad=256, m=128)
    assert lib.tq_logits(ctypes.byref(st2), base16, 4, 4, base16, base16, base16, 100, 1, base16, base16,
                         1 << 20, None) == tq.TQ_EUNSUPPORTED
    # decode: value params must be MSE mode
    assert lib.tq_decode_attn(ctypes.byref(st), ctypes.byref(st), base16, 1, 4, 1, base16, base16, base16, base16,
                              base16, base16, 64, 0.0, base16, base16, 1 << 20, None) == tq.TQ_EUNSUPPORTED
    assert lib.tq_code_bytes(-1, 1, 1, 1) == -1


def test_project_quantize_validation():
    """tq_project_quantize rejects bad shapes, NULL and misaligned buffers on the host, before
    any tensor map or launch; n_tok == 0 is a no-op."""
    st, keep = _fake_params()  # d = d_pad = 128, product mode, m = 128
    f = tq._lib.tq_project_quantize
    buf = np.zeros(4096, np.uint8)
    b = (buf.ctypes.data + 15) // 16 * 16
    ok = dict(x=b, n_tok=4, ld_x=64, hidden=64, w=b, n_heads=1, ld_w=64, codes=b, norms=b, rnorms=b, k_out=None,
              ld_k=0)

    def call(params=st, **kw):
        a = dict(ok, **kw)
        return f(ctypes.byref(params), a["x"], a["n_tok"], a["ld_x"], a["hidden"], a["w"], a["n_heads"], a["ld_w"],
                 a["codes"], a["norms"], a["rnorms"], a["k_out"], a["ld_k"], None)

    assert call(hidden=48, ld_x=48, ld_w=48) == tq.TQ_EINVAL          # hidden not a multiple of 32
    assert call(hidden=0) == tq.TQ_EINVAL
    assert call(n_heads=0) == tq.TQ_EINVAL
    assert call(n_tok=-1) == tq.TQ_EINVAL
    assert call(n_tok=0, x=None, w=None, codes=None, norms=None, rnorms=None) == tq.TQ_OK
    assert call(x=None) == tq.TQ_EINVAL
    assert call(rnorms=None) == tq.TQ_EINVAL                           # product mode needs residual norms
    assert call(x=b + 2) == tq.TQ_EINVAL                               # x not 16-byte aligned
    assert call(ld_x=32) == tq.TQ_EINVAL                               # ld_x < hidden
    assert call(ld_w=68) == tq.TQ_EINVAL                               # row stride not a multiple of 8
    assert call(k_out=b, ld_k=64) == tq.TQ_EINVAL                      # ld_k < 128 * n_heads
    assert call(codes=b + 8) == tq.TQ_EINVAL                           # codes not 16-byte aligned
    st2, keep2 = _fake_params(d=200, d_pad=256, m=256)
    assert call(params=st2) == tq.TQ_EUNSUPPORTED                      # d_pad 256
    st3, keep3 = _fake_params(m=64)
    assert call(params=st3) == tq.TQ_EUNSUPPORTED                      # product mode with m < 128
    assert tq.tq_last_error()


def test_sliced_decode_validation():
    """tq_decode_attn with token-sliced values (the tensor-memory decode) rejects the shapes it does not
    serve and bad buffers on the host; batch == 0 is a no-op; the sparse and partial forms refuse it."""
    kp, keep_k = _fake_params(bits=3)                                        # keys: product, m = 128
    vp, keep_v = _fake_params(bits=3, mode=tq.TQ_MODE_MSE, m=0, layout=tq.TQ_LAYOUT_SLICED)
    f = tq._lib.tq_decode_attn
    buf = np.zeros(4096, np.uint8)
    b = (buf.ctypes.data + 15) // 16 * 16
    ok = dict(kp=kp, q=b, batch=1, hq=4, hkv=1, kc=b, kn=b, krn=b, vc=b, vn=b, sl=b, T=64, out=b, ws=b,
              wsb=1 << 40)

    def call(**kw):
        a = dict(ok, **kw)
        return f(ctypes.byref(a["kp"]), ctypes.byref(vp), a["q"], a["batch"], a["hq"], a["hkv"], a["kc"], a["kn"],
                 a["krn"], a["vc"], a["vn"], a["sl"], a["T"], 0.0, a["out"], a["ws"], a["wsb"], None)

    assert call(hq=8) == tq.TQ_EUNSUPPORTED                  # 8 query heads per KV head
    assert call(T=48) == tq.TQ_EUNSUPPORTED                  # max_tokens not a multiple of 32
    k64, keep64 = _fake_params(bits=3, m=64)
    assert call(kp=k64) == tq.TQ_EUNSUPPORTED                # keys with m < 128
    k256, keep256 = _fake_params(d=200, d_pad=256, bits=3, m=256)
    assert call(kp=k256) == tq.TQ_EUNSUPPORTED               # d_pad 256
    assert call(batch=-1) == tq.TQ_EINVAL
    assert call(batch=0, q=None, kc=None, out=None, ws=None) == tq.TQ_OK
    assert call(q=None) == tq.TQ_EINVAL
    assert call(vn=b + 2) == tq.TQ_EINVAL                    # norms not 16-byte aligned
    assert call(wsb=16) == tq.TQ_EINVAL                      # workspace too small
    g = tq._lib.tq_decode_attn_sparse
    assert g(ctypes.byref(kp), ctypes.byref(vp), b, 1, 4, 1, b, b, b, b, b, b, 64, 0.0, 1e-3, b, b, 1 << 40,
             None) == tq.TQ_EUNSUPPORTED                     # Sparse V reads plane-layout values
    assert tq.tq_last_error()


def test_logits_d256_kb3_validation():
    """tq_logits at d_pad 256 with 3 index bits (the search scan writing every score): a ragged key
    count across several KV heads and a short workspace are refused on the host."""
    st, keep = _fake_params(d=200, d_pad=256, bits=4, m=256)
    f = tq._lib.tq_logits
    buf = np.zeros(4096, np.uint8)
    b = (buf.ctypes.data + 15) // 16 * 16
    need = tq._lib.tq_logits_workspace(ctypes.byref(st), 8)
    assert need > 0
    # q, n_q, group, codes, norms, rnorms, n_keys, n_kv_heads, logits, workspace, bytes, stream
    assert f(ctypes.byref(st), b, 8, 4, b, b, b, 100, 2, b, b, need, None) == tq.TQ_EUNSUPPORTED
    assert f(ctypes.byref(st), b, 8, 4, b, b, b, 128, 2, b, b, need - 1, None) == tq.TQ_EINVAL
    assert f(ctypes.byref(st), b, 8, 4, b, b, b, 0, 2, b, b, 0, None) == tq.TQ_OK   # no keys: nothing to do


def test_host_validation_of_the_other_entry_points():
    """Dequantize, logits with a row stride, search, the sharded merges and the partial decode refuse
    bad arguments on the host (and empty calls are no-ops), before anything reaches the GPU."""
    lib = tq._lib
    st, keep = _fake_params()                                              # d 128, product, b = 4, m = 128
    sm, keep_m = _fake_params(mode=tq.TQ_MODE_MSE, m=0, bits=3)           # MSE values
    sl, keep_s = _fake_params(mode=tq.TQ_MODE_MSE, m=0, bits=3, layout=tq.TQ_LAYOUT_SLICED)
    s256, keep2 = _fake_params(d=200, d_pad=256, bits=4, m=256)
    buf = np.zeros(4096, np.uint8)
    b = (buf.ctypes.data + 15) // 16 * 16
    R = ctypes.byref
    # tq_dequantize(p, codes, norms, rnorms, n_vec, out, ld, stream)
    assert lib.tq_dequantize(R(st), b, b, b, 0, None, 0, None) == tq.TQ_OK
    assert lib.tq_dequantize(R(st), b, b, b, -1, b, 128, None) == tq.TQ_EINVAL
    assert lib.tq_dequantize(R(st), b, b, None, 4, b, 128, None) == tq.TQ_EINVAL      # product mode, no rnorms
    assert lib.tq_dequantize(R(st), b, b, b, 4, b, 64, None) == tq.TQ_EINVAL          # ld < d
    assert lib.tq_dequantize(R(st), b + 4, b, b, 4, b, 128, None) == tq.TQ_EINVAL     # codes misaligned
    # tq_logits_ld(p, q, n_q, group, codes, norms, rnorms, n_keys, n_kv_heads, logits, ld, ws, ws_bytes, stream)
    assert lib.tq_logits_ld(R(st), b, 4, 4, b, b, b, 256, 1, b, 128, b, 1 << 30, None) == tq.TQ_EINVAL  # ld < n_keys
    assert lib.tq_logits_ld(R(sl), b, 4, 4, b, b, None, 256, 1, b, 256, b, 1 << 30, None) == tq.TQ_EUNSUPPORTED
    # tq_search_workspace / tq_search_topk(p, q, n_q, codes, norms, rnorms, n_db, k, ids, scores, ws, bytes, s)
    assert lib.tq_search_workspace(R(s256), 16, 1000, 0) == -1                      # k < 1
    need = lib.tq_search_workspace(R(s256), 16, 1000, 10)
    assert need > 0
    assert lib.tq_search_topk(R(s256), b, 0, None, None, None, 1000, 10, None, None, None, 0, None) == tq.TQ_OK
    assert lib.tq_search_topk(R(s256), b, 16, b, b, b, 5, 10, b, b, b, need, None) == tq.TQ_EINVAL   # n_db < k
    assert lib.tq_search_topk(R(s256), b, 16, b, b, b, 1000, 0, b, b, b, need, None) == tq.TQ_EUNSUPPORTED
    assert lib.tq_search_topk(R(s256), b, 16, b, b, b, 1000, 10, b, b, b, need - 1, None) == tq.TQ_EINVAL
    assert lib.tq_search_topk(R(s256), b, 16, b + 8, b, b, 1000, 10, b, b, b, need, None) == tq.TQ_EINVAL
    assert lib.tq_search_topk(R(sl), b, 16, b, b, None, 1000, 10, b, b, b, need, None) == tq.TQ_EUNSUPPORTED
    # tq_search_merge(ids, scores, n_parts, id_offsets, n_q, k, out_ids, out_scores, stream)
    assert lib.tq_search_merge(b, b, 0, b, 4, 10, b, b, None) == tq.TQ_EINVAL        # no parts
    assert lib.tq_search_merge(b, b, 2, b, 4, 0, b, b, None) == tq.TQ_EINVAL         # k < 1
    assert lib.tq_search_merge(b, b, 2, b, 0, 10, None, None, None) == tq.TQ_OK      # no queries
    assert lib.tq_search_merge(None, b, 2, b, 4, 10, b, b, None) == tq.TQ_EINVAL
    assert lib.tq_search_merge(b + 2, b, 2, b, 4, 10, b, b, None) == tq.TQ_EINVAL    # ids misaligned
    # tq_decode_attn_partial_bytes / tq_decode_attn_partial / tq_decode_attn_merge
    assert lib.tq_decode_attn_partial_bytes(R(sm), 2, 8) == 2 * 8 * (128 + 2) * 4
    assert lib.tq_decode_attn_partial_bytes(R(sm), -1, 8) == -1
    assert lib.tq_decode_attn_partial(R(st), R(sm), b, 1, 4, 1, b, b, b, b, b, b, 64, 0.0, None, b, 1 << 30,
                                      None) == tq.TQ_EINVAL                          # NULL partial
    assert lib.tq_decode_attn_merge(R(st), b, 2, 1, 4, b, None) == tq.TQ_EUNSUPPORTED  # needs the value params
    assert lib.tq_decode_attn_merge(R(sm), b, 0, 1, 4, b, None) == tq.TQ_EINVAL        # no parts
    assert lib.tq_decode_attn_merge(R(sm), b, 2, 0, 4, None, None) == tq.TQ_OK         # empty batch
    assert lib.tq_decode_attn_merge(R(sm), None, 2, 1, 4, b, None) == tq.TQ_EINVAL
    assert tq.tq_last_error()


def test_polar_qjl_validation():
    """The polar code's QJL stage (tq_polar_qjl) and its logits (tq_polar_logits_prod) refuse bad
    arguments on the host; an empty call is a no-op."""
    lib = tq._lib
    pp, keep = _fake_polar()
    buf = np.zeros(4096, np.uint8)
    b = (buf.ctypes.data + 15) // 16 * 16
    R = ctypes.byref
    # tq_polar_qjl(p, S, m, x, dtype, n_vec, ld, codes, signs, rnorms, stream)
    q = lambda **kw: lib.tq_polar_qjl(R(pp), kw.get("S", b), kw.get("m", 128), kw.get("x", b),
                                      kw.get("dtype", tq.TQ_BF16), kw.get("n_vec", 4), kw.get("ld", 128),
                                      b, b, b, None)
    assert q(m=48) == tq.TQ_EINVAL                                   # m not a multiple of 32
    assert q(m=256) == tq.TQ_EINVAL                                  # m > d_pad
    assert q(n_vec=-1) == tq.TQ_EINVAL
    assert q(n_vec=0, x=None, S=None) == tq.TQ_OK
    assert q(dtype=9) == tq.TQ_EINVAL
    assert q(S=None) == tq.TQ_EINVAL
    assert q(ld=64) == tq.TQ_EINVAL                                  # ld < d
    assert q(x=b + 2) == tq.TQ_EINVAL                                # x not 16-byte aligned
    # tq_polar_logits_prod(p, S, m, q, group, codes, norms, signs, rnorms, n_keys, n_kv_heads, logits, s)
    lp = lambda p=R(pp), m=128, signs=b: lib.tq_polar_logits_prod(p, b, m, b, 4, b, b, signs, b, 64, 1, b, None)
    assert lp(p=None) == tq.TQ_EINVAL
    assert lp(m=0) == tq.TQ_EINVAL
    assert lp(signs=None) == tq.TQ_EINVAL
    assert lp(signs=b + 2) == tq.TQ_EINVAL                           # signs not 4-byte aligned
    assert tq.tq_last_error()


@pytest.mark.parametrize("d_pad", [128, 256, 1024, 4096])
@pytest.mark.parametrize("w", [1, 2, 3])
def test_polar_tables_match_oracle(d_pad, w):
    """The library's angle tables (C++ Gauss-Legendre Lloyd iteration) equal the oracle's
    (betainc masses, adaptive-quadrature moments) value for value."""
    from oracle import polar
    t = tq.tq_polar_make_tables(d_pad, w)
    c1, per_level = polar.tables(d_pad, w)
    L1, L2 = len(c1), len(per_level[0][0])
    assert len(t) == tq._lib.tq_polar_table_floats(d_pad, w) == 3 * L1 + len(per_level) * (4 * L2 - 1)
    assert np.array_equal(t[:L1], c1)
    assert np.allclose(t[L1:3 * L1:2], np.cos(c1.astype(np.float64)), atol=1e-7)
    assert np.allclose(t[L1 + 1:3 * L1:2], np.sin(c1.astype(np.float64)), atol=1e-7)
    off = 3 * L1
    for c, th in per_level:
        assert np.array_equal(t[off:off + L2], c)
        assert np.array_equal(t[off + L2:off + 2 * L2 - 1], th)
        cs = t[off + 2 * L2 - 1:off + 4 * L2 - 1]
        assert np.allclose(cs[0::2], np.cos(c.astype(np.float64)), atol=1e-7)
        assert np.allclose(cs[1::2], np.sin(c.astype(np.float64)), atol=1e-7)
        off += 4 * L2 - 1


def test_polar_sizes_and_validation():
    assert tq.tq_polar_code_bytes(128, 2, 10) == 10 * 32
    # a record is w * d_pad / 8 whole bytes: d_pad 8 is the smallest (w = 1: one byte)
    assert tq.tq_polar_code_bytes(8, 1, 3) == 3
    assert tq.tq_polar_code_bytes(8, 3, 3) == 9
    for w in (1, 2, 3):
        assert tq.tq_polar_code_bytes(4, w, 1) == -1
    assert tq._lib.tq_polar_table_floats(100, 2) == -1
    assert tq._lib.tq_polar_table_floats(128, 4) == -1
    bad = tq.tq_polar_params(128, 128, 4, 0, None, None)
    assert tq._lib.tq_polar_quantize(ctypes.byref(bad), None, 2, 1, 128, None, None, None) == tq.TQ_EINVAL


def _fake_polar(**kw):
    p = dict(d=128, d_pad=128, w=2)
    p.update(kw)
    buf = np.zeros(256, np.float32)
    ptr = buf.ctypes.data
    return tq.tq_polar_params(p["d"], p["d_pad"], p["w"], 0, ptr, ptr), buf


@pytest.mark.parametrize("kw,code", [
    (dict(d_pad=64), tq.TQ_EUNSUPPORTED),
    (dict(d=0), tq.TQ_EINVAL),
    (dict(d=129), tq.TQ_EINVAL),
    (dict(w=0), tq.TQ_EINVAL),
    (dict(w=4), tq.TQ_EINVAL),
])
def test_polar_validation_rejects_bad_params(kw, code):
    st, keep = _fake_polar(**kw)
    lib = tq._lib
    p = ctypes.byref(st)
    assert lib.tq_polar_quantize(p, keep.ctypes.data, tq.TQ_BF16, 10, 128, keep.ctypes.data, keep.ctypes.data,
                                 None) == code
    assert lib.tq_polar_dequantize(p, keep.ctypes.data, keep.ctypes.data, 10, keep.ctypes.data, 128, None) == code
    assert lib.tq_polar_logits(p, keep.ctypes.data, 4, keep.ctypes.data, keep.ctypes.data, 10, 1,
                               keep.ctypes.data, None) == code
    assert tq.tq_last_error()


def test_polar_validation_rejects_null_misaligned_and_sizes():
    st, keep = _fake_polar()
    lib = tq._lib
    p = ctypes.byref(st)
    ok = keep.ctypes.data  # 16-byte aligned host buffer: never dereferenced before validation fails
    assert lib.tq_polar_quantize(p, None, tq.TQ_BF16, 10, 128, ok, ok, None) == tq.TQ_EINVAL
    assert lib.tq_polar_quantize(p, ok, 9, 10, 128, ok, ok, None) == tq.TQ_EINVAL
    assert lib.tq_polar_quantize(p, ok, tq.TQ_BF16, 10, 100, ok, ok, None) == tq.TQ_EINVAL  # ld < d
    assert lib.tq_polar_quantize(p, ok + 4, tq.TQ_BF16, 10, 128, ok, ok, None) == tq.TQ_EINVAL
    assert lib.tq_polar_quantize(p, ok, tq.TQ_BF16, -1, 128, ok, ok, None) == tq.TQ_EINVAL
    assert lib.tq_polar_quantize(p, None, tq.TQ_BF16, 0, 128, None, None, None) == tq.TQ_OK  # nothing to do
    assert lib.tq_polar_dequantize(p, ok + 8, ok, 10, ok, 128, None) == tq.TQ_EINVAL
    assert lib.tq_polar_logits(p, ok, 0, ok, ok, 10, 1, ok, None) == tq.TQ_EINVAL
    assert lib.tq_polar_logits(p, ok, 9, ok, ok, 10, 1, ok, None) == tq.TQ_EINVAL
    assert lib.tq_polar_logits(p, ok, 4, ok, ok, 0, 1, ok, None) == tq.TQ_OK
    null = tq.tq_polar_params(128, 128, 2, 0, None, None)
    assert lib.tq_polar_logits(ctypes.byref(null), ok, 4, ok, ok, 10, 1, ok, None) == tq.TQ_EINVAL


def test_polar_quantize_rejects_row_length_off_16_bytes():
    """d * element size must be a multiple of 16 bytes (the kernel loads groups of 4 elements)."""
    lib = tq._lib
    for d, dtype, code in ((6, tq.TQ_F32, tq.TQ_EINVAL), (100, tq.TQ_BF16, tq.TQ_EINVAL), (10, tq.TQ_F32, tq.TQ_EINVAL)):
        st, keep = _fake_polar(d=d)
        ok = keep.ctypes.data
        assert lib.tq_polar_quantize(ctypes.byref(st), ok, dtype, 10, 128, ok, ok, None) == code, (d, dtype)
