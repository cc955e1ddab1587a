"""Parity at the full workload sizes, in the launch configurations bench.py
times, on outputs the oracle can compute (sampled rows, sequences, queries):

* layer: 8 KV heads x 32768 tokens, 32 query heads (GQA 4), b = 3 and 4 -
  tq_quantize on sampled vectors, tq_logits on every (query, key) from
  oracle-made codes;
* batched decode: 64 sequences x 8 KV heads x 16384 tokens, K product b = 3,
  V MSE b = 3 - the full launch; three sampled sequences carry oracle-made
  codes (the others zero codes, whose rows are not compared);
* quantize 2^20 bf16 vectors at b = 2, 3, 4 - sampled vectors incl. the last tile;
* search: 10^6 database vectors (d = 200 -> 256), 10^4 queries, b = 2 and 4 -
  top-10 of 40 sampled queries against the oracle; quantize on sampled rows.
"""
import numpy as np
import pytest
import torch

import vector_quantization_randomized_b200 as tq
import workloads as wl
from oracle import codec, estimate
from gpu_util import make_pair, oracle_codes, compare_codes, logit_tolerance

pytestmark = pytest.mark.gpu
dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _gpu_codes(p, x_t):
    n = x_t.shape[0]
    c = torch.empty(p.code_bytes(n), dtype=torch.uint8, device="cuda")
    nn = torch.empty(n, dtype=torch.int16, device="cuda")
    rn = torch.empty(n, dtype=torch.int16, device="cuda") if p.mode == tq.TQ_MODE_PROD else None
    tq.tq_quantize(p, x_t, c, nn, rn)
    return c, nn, rn


def _sampled_compare(op, x_host, rows, c, nn, rn):
    """Compare the GPU codes of `rows` with the oracle encoding of those rows."""
    codes = c.cpu().numpy()
    norms = nn.cpu().numpy().view(np.float16)
    rnorms = rn.cpu().numpy().view(np.float16) if rn is not None else None
    idx_all, sg_all = codec.unpack(codes, x_host.shape[0], op.d_pad, op.kb, op.m)
    enc = codec.encode(x_host[rows], op.D, op.c, op.t, op.S)
    fl = codec.boundary_flags(enc, op.t, op.S)
    dif = idx_all[rows] != enc["idx"]
    assert not np.any(dif & ~fl["idx"])
    changed = np.any(dif, axis=1)
    assert np.all((norms[rows] == enc["norm_f16"]) | fl["norm"])
    if op.m:
        sd = (sg_all[rows] != enc["signs"]) & ~changed[:, None]
        assert not np.any(sd & ~fl["signs"])
        assert np.all((rnorms[rows] == enc["rnorm_f16"]) | fl["rnorm"] | changed)
    return int(fl["idx"].sum())


@pytest.mark.parametrize("bits", [3, 4])
def test_layer_quantize_and_logits(bits):
    H, T, d, G = 8, 32768, 128, 4
    n = H * T
    K = wl.kv_block(1, H, T, d, seed=wl.SEED_KEYS).reshape(n, d)
    V = wl.kv_block(1, H, T, d, seed=wl.SEED_VALUES).reshape(n, d)
    q = wl.queries(H * G, d, seed=wl.SEED_QUERIES)
    kp, kop = make_pair(d, bits, tq.TQ_MODE_PROD, 128, wl.SEED_PARAMS)
    vp, vop = make_pair(d, bits, tq.TQ_MODE_MSE, 0, wl.SEED_PARAMS + 1)
    rows = np.unique(np.concatenate([np.random.default_rng(bits).integers(0, n, 3000), [0, n - 1]]))
    c, nn, rn = _gpu_codes(kp, torch.from_numpy(K).to(torch.bfloat16).cuda())
    _sampled_compare(kop, K, rows, c, nn, rn)
    c, nn, rn = _gpu_codes(vp, torch.from_numpy(V).to(torch.bfloat16).cuda())
    _sampled_compare(vop, V, rows, c, nn, rn)
    # logits from oracle-made codes, every (query, key)
    codes, norms, rnorms, enc = oracle_codes(kop, K)
    ref = estimate.logits_gqa(q, kop.D, kop.S, enc["idx"], enc["signs"], norms, rnorms, kop.c, kop.m, H, G, T)
    out = torch.empty((H * G, T), dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.tq_logits_workspace(kp, H * G), dtype=torch.uint8, device="cuda")
    tq.tq_logits(kp, dev(q), G, dev(codes), dev(norms.view(np.int16)), dev(rnorms.view(np.int16)), T, H, out, ws)
    got = out.cpu().numpy().astype(np.float64)
    for h in range(H * G):
        g = h // G
        tol = logit_tolerance(ref[h:h + 1], norms[g * T:(g + 1) * T], q[h:h + 1])[0]
        assert np.all(np.abs(got[h] - ref[h]) <= tol), h


def test_batched_decode_full_launch():
    B, Hkv, T, d, Hq = 64, 8, 16384, 128, 32
    kp, kop = make_pair(d, 3, tq.TQ_MODE_PROD, 128, wl.SEED_PARAMS)
    vp, vop = make_pair(d, 3, tq.TQ_MODE_MSE, 0, wl.SEED_PARAMS + 1)
    sample = [0, 37, 63]
    n = B * Hkv * T
    kc = np.zeros(kp.code_bytes(n), np.uint8)
    vc = np.zeros(vp.code_bytes(n), np.uint8)
    kn = np.zeros(n, np.float16)
    krn = np.zeros(n, np.float16)
    vn = np.zeros(n, np.float16)
    Ks = wl.kv_block(B, Hkv, T, d, seed=wl.SEED_KEYS, seqs=sample)
    Vs = wl.kv_block(B, Hkv, T, d, seed=wl.SEED_VALUES, seqs=sample)
    ktb = codec.code_bytes(d_pad=128, kb=2, m=128, n_vec=32)
    vtb = codec.code_bytes(d_pad=128, kb=3, m=0, n_vec=32)
    per_seq = Hkv * T  # vectors per sequence (a multiple of 32: whole tiles)
    enc_k, enc_v = {}, {}
    for i, b in enumerate(sample):
        c1, n1, r1, ek = oracle_codes(kop, Ks[i].reshape(-1, d))
        c2, n2, _, ev = oracle_codes(vop, Vs[i].reshape(-1, d))
        t0 = b * per_seq // 32
        kc[t0 * ktb:t0 * ktb + c1.size] = c1
        vc[t0 * vtb:t0 * vtb + c2.size] = c2
        kn[b * per_seq:(b + 1) * per_seq] = n1
        krn[b * per_seq:(b + 1) * per_seq] = r1
        vn[b * per_seq:(b + 1) * per_seq] = n2
        enc_k[b], enc_v[b] = ek, ev
    q = wl.queries(B * Hq, d, seed=wl.SEED_QUERIES).reshape(B, Hq, d)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.tq_decode_attn_workspace(kp, B, Hq, Hkv, T), dtype=torch.uint8, device="cuda")
    sl = torch.full((B,), T, dtype=torch.int32, device="cuda")
    tq.tq_decode_attn(kp, vp, dev(q), Hkv, dev(kc), dev(kn.view(np.int16)), dev(krn.view(np.int16)), dev(vc),
                      dev(vn.view(np.int16)), sl, T, out, ws)
    got = out.cpu().numpy().astype(np.float64)
    for b in sample:
        ek, ev = enc_k[b], enc_v[b]
        kn_b, krn_b, vn_b = (a[b * per_seq:(b + 1) * per_seq] for a in (kn, krn, vn))
        ref = estimate.decode_attention(q[b:b + 1], kop.D, kop.S, ek["idx"], ek["signs"], kn_b, krn_b, kop.c, kop.m,
                                        vop.D, ev["idx"], vn_b, vop.c, d, [T], Hq, Hkv, T)[0]
        for h in range(Hq):
            assert np.linalg.norm(got[b, h] - ref[h]) <= 2e-3 * np.linalg.norm(ref[h]), (b, h)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quantize_2pow20(bits):
    n, d = 1 << 20, 128
    x = np.concatenate([wl.to_bf16(wl.head_vectors(n // 8, d, seed=wl.SEED_KEYS, head=h)) for h in range(8)])
    p, op = make_pair(d, bits, tq.TQ_MODE_PROD, 128, wl.SEED_PARAMS)
    c, nn, rn = _gpu_codes(p, torch.from_numpy(x).to(torch.bfloat16).cuda())
    rows = np.unique(np.concatenate([np.random.default_rng(bits).integers(0, n, 4000), np.arange(n - 300, n)]))
    _sampled_compare(op, x, rows, c, nn, rn)


@pytest.mark.parametrize("bits", [2, 4])
def test_search_full_size(bits):
    n_db, n_q, d, k = 1000000, 10000, 200, 10
    db = wl.to_bf16(wl.search_set(n_db, d, seed=wl.SEED_KEYS))
    qs = wl.search_set(n_q, d, seed=wl.SEED_QUERIES)
    p, op = make_pair(d, bits, tq.TQ_MODE_PROD, 256, wl.SEED_PARAMS)
    # quantize the database on the GPU, compare sampled rows
    c, nn, rn = _gpu_codes(p, torch.from_numpy(db).to(torch.bfloat16).cuda())
    rows = np.unique(np.random.default_rng(bits).integers(0, n_db, 2000))
    _sampled_compare(op, db, rows, c, nn, rn)
    del c, nn, rn
    # search on oracle-made codes, all queries; check 40 sampled queries
    codes, norms, rnorms, enc = oracle_codes(op, db)
    ids = torch.empty((n_q, k), dtype=torch.int32, device="cuda")
    sc = torch.empty((n_q, k), dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.tq_search_workspace(p, n_q, n_db, k), dtype=torch.uint8, device="cuda")
    tq.tq_search_topk(p, dev(qs), dev(codes), dev(norms.view(np.int16)), dev(rnorms.view(np.int16)), n_db, k, ids,
                      sc, ws)
    gi = ids.cpu().numpy().astype(np.int64)
    gs = sc.cpu().numpy().astype(np.float64)
    sample = np.random.default_rng(5).choice(n_q, 40, replace=False)
    q_rot, u = estimate.prep_queries(qs[sample], op.D, op.S)
    ref = estimate.logits_from_codes(q_rot, u, enc["idx"], enc["signs"], norms, rnorms, op.c, op.m)
    rid, rs = estimate.topk(ref, k)
    for r, qi in enumerate(sample):
        tol_all = 1e-4 * np.abs(ref[r]) + 1e-5 * np.linalg.norm(qs[qi].astype(np.float64)) * norms.astype(np.float64)
        assert np.all(np.abs(gs[qi] - ref[r, gi[qi]]) <= tol_all[gi[qi]])
        kth, tk = rs[r, -1], tol_all[rid[r, -1]]
        must = set(np.nonzero(ref[r] > kth + 2 * tk)[0])
        may = set(np.nonzero(ref[r] >= kth - 2 * tk)[0])
        assert must <= set(gi[qi]) <= may
