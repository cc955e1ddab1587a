"""GPU parity of the polar-coordinate stage 1 against oracle/polar.py.

* tq_polar_quantize: every angle index bit-exact except decisions flagged by
  the oracle (the point within 1e-6 of its radius - floored at 1/sqrt(d_pad) -
  of a cell boundary, counted), norms exact except fp16 rounding ties; bf16
  and fp16 keys at d = 128, fp32 at d = 200 (d_pad 256), ragged counts.
* tq_polar_dequantize on oracle-made records: |x_hat - x_hat_oracle| <=
  1e-5 n (fp32 tree of cos / sin products and rotation).
* tq_polar_logits on oracle-made records: |l - l_oracle| <= 1e-4 |l| +
  1e-5 n ||q||, every group size 1..8, several KV heads, key counts that are
  not multiples of the 128-key block.
* The bench's full launch (8 KV heads x 32768 keys, 32 query heads) at
  w = 2 and 3: sampled keys' indices and norms, and their logits.
"""
import numpy as np
import pytest
import torch

import vector_quantization_randomized_b200 as tq
import workloads as wl
from oracle import codec, polar
from oracle.params import sign_flips
from gpu_util import f16_neighbours, logit_tolerance

pytestmark = pytest.mark.gpu
dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _oracle(d, w):
    d_pad = 128 if d <= 128 else 256
    return sign_flips(42, d_pad), polar.tables(d_pad, w), d_pad


def _quantize_check(x_host, dtype, d, w):
    p = tq.PolarParams(d, w, seed=42)
    D, tabs, d_pad = _oracle(d, w)
    xt = torch.from_numpy(x_host).to(dtype)
    xin = xt.float().numpy().astype(np.float64)
    n = x_host.shape[0]
    codes = torch.full((p.code_bytes(n),), 0xAB, dtype=torch.uint8, device="cuda")
    norms = torch.zeros(n, dtype=torch.int16, device="cuda")
    tq.tq_polar_quantize(p, xt.cuda(), codes, norms)
    torch.cuda.synchronize()
    i1, ihi = polar.unpack(codes.cpu().numpy(), n, w, d_pad)
    enc = polar.encode(xin, D, w, tabs)
    f1, fl = polar.boundary_flags(enc, w, d_pad, tabs)
    bad = (i1 != enc["i1"]) & ~f1
    assert not np.any(bad), np.argwhere(bad)[:5]
    flagged, mismatched = int(f1.sum()), int((i1 != enc["i1"]).sum())
    for a, b, f in zip(ihi, enc["ihi"], fl):
        assert not np.any((a != b) & ~f)
        flagged += int(f.sum())
        mismatched += int((a != b).sum())
    nn = norms.cpu().numpy().view(np.float16)
    tie = codec.f16_tie_flags(enc["norm"])
    assert np.all((nn == enc["norm_f16"]) | (tie & f16_neighbours(nn, enc["norm_f16"])))
    assert mismatched <= flagged
    return mismatched, flagged


@pytest.mark.parametrize("w", [1, 2, 3])
def test_quantize_bf16_d128(w):
    x = wl.to_bf16(wl.head_vectors(3000, 128, seed=3))
    _quantize_check(x, torch.bfloat16, 128, w)


def test_quantize_fp16_ragged_and_zero():
    x = wl.head_vectors(77, 128, seed=4)
    x[5] = 0.0
    _quantize_check(x.astype(np.float16).astype(np.float32), torch.float16, 128, 2)


@pytest.mark.parametrize("w", [2, 3])
def test_quantize_fp32_d200(w):
    x = wl.search_set(1000, 200, seed=5).astype(np.float32)
    _quantize_check(x, torch.float32, 200, w)


def _oracle_records(x, d, w):
    D, tabs, d_pad = _oracle(d, w)
    enc = polar.encode(x, D, w, tabs)
    return polar.pack(enc["i1"], enc["ihi"], w, d_pad).ravel(), enc, D, tabs, d_pad


@pytest.mark.parametrize("d,w", [(128, 1), (128, 2), (128, 3), (200, 2)])
def test_dequantize(d, w):
    x = wl.head_vectors(500, d, seed=6) if d == 128 else wl.search_set(500, d, seed=6)
    buf, enc, D, tabs, d_pad = _oracle_records(x, d, w)
    p = tq.PolarParams(d, w, seed=42)
    out = torch.full((500, d), float("nan"), device="cuda")
    tq.tq_polar_dequantize(p, dev(buf), dev(enc["norm_f16"].view(np.int16)), 500, out)
    ref = polar.dequantize(enc["i1"], enc["ihi"], enc["norm_f16"], D, d, w, tabs)
    got = out.cpu().numpy().astype(np.float64)
    n = enc["norm_f16"].astype(np.float64)
    assert np.all(np.abs(got - ref) <= 1e-5 * n[:, None] + 1e-12)


@pytest.mark.parametrize("w,group,heads,n_keys", [
    (2, 4, 3, 1000), (3, 1, 2, 300), (1, 8, 2, 257), (3, 2, 1, 128), (2, 3, 4, 33),
])
def test_logits(w, group, heads, n_keys):
    x = np.concatenate([wl.head_vectors(n_keys, 128, seed=7, head=h) for h in range(heads)])
    buf, enc, D, tabs, d_pad = _oracle_records(x, 128, w)
    q = wl.queries(heads * group, 128, seed=8)
    p = tq.PolarParams(128, w, seed=42)
    out = torch.full((heads * group, n_keys), float("nan"), device="cuda")
    tq.tq_polar_logits(p, dev(q.astype(np.float32)), group, dev(buf), dev(enc["norm_f16"].view(np.int16)),
                       n_keys, heads, out)
    got = out.cpu().numpy().astype(np.float64)
    for h in range(heads * group):
        g = h // group
        sl = slice(g * n_keys, (g + 1) * n_keys)
        ref = polar.logits(q[h:h + 1], D, enc["i1"][sl], [a[sl] for a in enc["ihi"]], enc["norm_f16"][sl], w, tabs)
        tol = logit_tolerance(ref, enc["norm_f16"][sl], q[h:h + 1])
        assert np.all(np.abs(got[h] - ref[0]) <= tol[0]), h


def test_logits_d200():
    x = wl.search_set(400, 200, seed=9)
    buf, enc, D, tabs, d_pad = _oracle_records(x, 200, 2)
    q = wl.search_set(2, 200, seed=10)
    p = tq.PolarParams(200, 2, seed=42)
    out = torch.empty((2, 400), device="cuda")
    tq.tq_polar_logits(p, dev(q.astype(np.float32)), 2, dev(buf), dev(enc["norm_f16"].view(np.int16)), 400, 1, out)
    ref = polar.logits(q, D, enc["i1"], enc["ihi"], enc["norm_f16"], 2, tabs)
    tol = logit_tolerance(ref, enc["norm_f16"], q)
    assert np.all(np.abs(out.cpu().numpy() - ref) <= tol)


@pytest.mark.parametrize("w", [2, 3])
def test_layer_full_size_sampled(w):
    """The bench's polar launch (8 KV heads x 32768 bf16 keys, 32 query heads,
    GQA 4): indices and norms of 3000 sampled keys and of the last 64 against
    the oracle, and every query head's logits of those keys against the
    oracle's logits from its own encoding wherever the two encodings agree."""
    H, T, d, G = 8, 32768, 128, 4
    n = H * T
    x = wl.kv_block(1, H, T, d, seed=wl.SEED_KEYS).reshape(n, d)
    p = tq.PolarParams(d, w, seed=42)
    D, tabs, d_pad = _oracle(d, w)
    codes = torch.empty(p.code_bytes(n), dtype=torch.uint8, device="cuda")
    norms = torch.empty(n, dtype=torch.int16, device="cuda")
    tq.tq_polar_quantize(p, torch.from_numpy(x).to(torch.bfloat16).cuda(), codes, norms)
    q = wl.queries(H * G, d, seed=wl.SEED_QUERIES)
    lg = torch.empty((H * G, T), dtype=torch.float32, device="cuda")
    tq.tq_polar_logits(p, dev(q.astype(np.float32)), G, codes, norms, T, H, lg)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.random.default_rng(w).integers(0, n, 3000), np.arange(n - 64, n)]))
    rb = polar.record_bytes(d_pad, w)
    recs = codes.cpu().numpy().reshape(n, rb)[rows]
    i1, ihi = polar.unpack(recs.ravel(), rows.size, w, d_pad)
    nn = norms.cpu().numpy().view(np.float16)[rows]
    xin = torch.from_numpy(x[rows]).to(torch.bfloat16).float().numpy().astype(np.float64)
    enc = polar.encode(xin, D, w, tabs)
    f1, fl = polar.boundary_flags(enc, w, d_pad, tabs)
    same = np.all(i1 == enc["i1"], axis=1)
    assert not np.any((i1 != enc["i1"]) & ~f1)
    for a, b, f in zip(ihi, enc["ihi"], fl):
        assert not np.any((a != b) & ~f)
        same &= np.all(a == b, axis=1)
    tie = codec.f16_tie_flags(enc["norm"])
    assert np.all((nn == enc["norm_f16"]) | (tie & f16_neighbours(nn, enc["norm_f16"])))
    same &= nn == enc["norm_f16"]
    got = lg.cpu().numpy().astype(np.float64)
    for h in range(H * G):
        sel = np.flatnonzero((rows // T == h // G) & same)
        ref = polar.logits(q[h:h + 1], D, enc["i1"][sel], [a[sel] for a in enc["ihi"]], enc["norm_f16"][sel], w,
                           tabs)[0]
        tol = logit_tolerance(ref[None, :], enc["norm_f16"][sel], q[h:h + 1])[0]
        assert np.all(np.abs(got[h, rows[sel] % T] - ref) <= tol), h


# ---- QJL stage on the polar residual (product code of the polar stage) -----------------
def _qjl_S(d_pad, m):
    from oracle.params import qjl_matrix
    kp = tq.Params(d_pad, 4, tq.TQ_MODE_PROD, m, 42, d_pad)   # the library's S for this seed (device fp16)
    return kp.S, qjl_matrix(42, m, d_pad)


@pytest.mark.parametrize("w,d,dtype", [(1, 128, torch.bfloat16), (2, 128, torch.bfloat16), (3, 128, torch.float16),
                                       (2, 200, torch.float32)])
def test_qjl_encode(w, d, dtype):
    """tq_polar_qjl after tq_polar_quantize against polar.encode_prod: sign bits exact except
    projections within 1e-6 ||S_i|| gamma of zero (codec.boundary_flags' rule), gamma exact
    except fp16 ties, on every vector whose angle indices equal the oracle's."""
    n = 777
    x = wl.to_bf16(wl.head_vectors(n, 128, seed=11)) if d == 128 else wl.search_set(n, d, seed=11).astype(np.float32)
    p = tq.PolarParams(d, w, seed=42)
    D, tabs, d_pad = _oracle(d, w)
    m = d_pad
    S_dev, S_or = _qjl_S(d_pad, m)
    xt = torch.from_numpy(x).to(dtype)
    xin = xt.float().numpy().astype(np.float64)
    codes = torch.zeros(p.code_bytes(n), dtype=torch.uint8, device="cuda")
    norms = torch.zeros(n, dtype=torch.int16, device="cuda")
    signs = torch.full((n * m // 8,), 0xAB, dtype=torch.uint8, device="cuda")
    rn = torch.zeros(n, dtype=torch.int16, device="cuda")
    tq.tq_polar_quantize(p, xt.cuda(), codes, norms)
    tq.tq_polar_qjl(p, S_dev, m, xt.cuda(), codes, signs, rn)
    torch.cuda.synchronize()
    enc = polar.encode_prod(xin, D, w, S_or, tabs)
    i1, ihi = polar.unpack(codes.cpu().numpy(), n, w, d_pad)
    same = np.all(i1 == enc["i1"], axis=1)
    for a, b in zip(ihi, enc["ihi"]):
        same &= np.all(a == b, axis=1)
    assert same.mean() > 0.99
    got = np.unpackbits(signs.cpu().numpy().reshape(n, m // 8), axis=1, bitorder="little")
    fl = codec.boundary_flags(dict(y=enc["y"], norm=enc["norm"], gamma=enc["gamma"], z=enc["z"]),
                              np.zeros(0, np.float32), S_or)["signs"]
    bad = (got != enc["signs"]) & ~fl & same[:, None]
    assert not np.any(bad), np.argwhere(bad)[:5]
    g = rn.cpu().numpy().view(np.float16)
    tie = codec.f16_tie_flags(enc["gamma"])
    ok = (g == enc["rnorm_f16"]) | (tie & f16_neighbours(g, enc["rnorm_f16"])) | ~same
    assert np.all(ok)


@pytest.mark.parametrize("w,group,heads,n_keys", [(2, 4, 3, 1000), (3, 1, 2, 300), (1, 8, 1, 129)])
def test_qjl_logits(w, group, heads, n_keys):
    """tq_polar_logits_prod on oracle-made records, signs and gamma against polar.logits_prod."""
    x = np.concatenate([wl.head_vectors(n_keys, 128, seed=12, head=h) for h in range(heads)])
    D, tabs, d_pad = _oracle(128, w)
    m = 128
    S_dev, S_or = _qjl_S(d_pad, m)
    enc = polar.encode_prod(x, D, w, S_or, tabs)
    buf = polar.pack(enc["i1"], enc["ihi"], w, d_pad).ravel()
    sbytes = np.packbits(enc["signs"], axis=1, bitorder="little").ravel()
    q = wl.queries(heads * group, 128, seed=13)
    p = tq.PolarParams(128, w, seed=42)
    out = torch.full((heads * group, n_keys), float("nan"), device="cuda")
    tq.tq_polar_logits_prod(p, S_dev, m, dev(q.astype(np.float32)), group, dev(buf),
                            dev(enc["norm_f16"].view(np.int16)), dev(sbytes), dev(enc["rnorm_f16"].view(np.int16)),
                            n_keys, heads, out)
    got = out.cpu().numpy().astype(np.float64)
    for h in range(heads * group):
        gk = h // group
        sl = slice(gk * n_keys, (gk + 1) * n_keys)
        ref = polar.logits_prod(q[h:h + 1], D, S_or, enc["yhat"][sl], enc["signs"][sl], enc["norm_f16"][sl],
                                enc["rnorm_f16"][sl], m)
        tol = logit_tolerance(ref, enc["norm_f16"][sl], q[h:h + 1])
        assert np.all(np.abs(got[h] - ref[0]) <= tol[0]), h
