"""GPU parity of the sharded entry points (the multi-device search and decode),
with the shards emulated on one GPU:

* tq_decode_attn_partial on token shards of every sequence (each shard packed
  as a KV cache of its own, one sequence shorter than the first shard, one
  empty), then tq_decode_attn_merge, against the oracle's one-pass decode
  (||delta o|| <= 2e-3 ||o|| per row, empty rows zero); one shard's partial
  against the oracle's partial (m, l and the normalised o);
* tq_search_merge against the oracle's merge of the same lists (exact, ties
  across shards), and tq_search_topk per database shard + tq_search_merge
  against tq_search_topk over the whole database (identical ids and scores).
"""
import math

import numpy as np
import pytest
import torch

import vector_quantization_randomized_b200 as tq
import workloads as wl
from oracle import codec, estimate
from gpu_util import make_pair

pytestmark = pytest.mark.gpu
dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _decode_problem(B, Hkv, Hq, T, seed):
    kp, kop = make_pair(128, 3, tq.TQ_MODE_PROD)
    vp, vop = make_pair(128, 3, tq.TQ_MODE_MSE, seed=43)
    K = np.concatenate([wl.to_bf16(wl.head_vectors(T, 128, seed=seed, seq=b, head=g))
                        for b in range(B) for g in range(Hkv)])
    V = np.concatenate([wl.to_bf16(wl.head_vectors(T, 128, seed=seed + 1, seq=b, head=g))
                        for b in range(B) for g in range(Hkv)])
    ke = codec.encode(K, kop.D, kop.c, kop.t, kop.S)
    ve = codec.encode(V, vop.D, vop.c, vop.t)
    q = wl.queries(B * Hq, 128, seed=seed + 2).reshape(B, Hq, 128)
    return kp, kop, vp, vop, ke, ve, q


def _shard_rows(a, B, Hkv, T, t0, t1):
    a = np.asarray(a)
    return a.reshape((B * Hkv, T) + a.shape[1:])[:, t0:t1].reshape((-1,) + a.shape[1:])


@pytest.mark.parametrize("bounds", [[0, 320, 640], [0, 96, 352, 640]])
def test_decode_partials_merge(bounds):
    B, Hkv, Hq, T = 3, 2, 8, 640
    kp, kop, vp, vop, ke, ve, q = _decode_problem(B, Hkv, Hq, T, 30)
    seq_lens = [640, 200, 0]
    parts = []
    for t0, t1 in zip(bounds[:-1], bounds[1:]):
        Tl = t1 - t0
        sh = lambda a: _shard_rows(a, B, Hkv, T, t0, t1)
        kc = codec.pack(sh(ke["idx"]), sh(ke["signs"]), kop.kb, kop.m)
        vc = codec.pack(sh(ve["idx"]), None, vop.kb, 0)
        local = [max(0, min(L - t0, Tl)) for L in seq_lens]
        part = torch.empty((B, Hq, 130), dtype=torch.float32, device="cuda")
        ws = torch.empty(tq.tq_decode_attn_workspace(kp, B, Hq, Hkv, Tl), dtype=torch.uint8, device="cuda")
        tq.tq_decode_attn_partial(kp, vp, dev(q.astype(np.float32)), Hkv, dev(kc), dev(sh(ke["norm_f16"]).view(np.int16)),
                                  dev(sh(ke["rnorm_f16"]).view(np.int16)), dev(vc),
                                  dev(sh(ve["norm_f16"]).view(np.int16)), dev(np.array(local, np.int32)), Tl, part, ws)
        parts.append(part)
        # this shard's partial against the oracle's (natural-log units there)
        m, lsum, o = estimate.decode_partial(q, kop.D, kop.S, sh(ke["idx"]), sh(ke["signs"]), sh(ke["norm_f16"]),
                                             sh(ke["rnorm_f16"]), kop.c, kop.m, vop.D, sh(ve["idx"]),
                                             sh(ve["norm_f16"]), vop.c, 128, local, Hq, Hkv, Tl)
        g = part.cpu().numpy().astype(np.float64)
        for b in range(B):
            for h in range(Hq):
                if local[b] == 0:
                    assert np.isneginf(g[b, h, 128]) and g[b, h, 129] == 0 and not np.any(g[b, h, :128])
                    continue
                assert abs(g[b, h, 128] * math.log(2) - m[b, h]) <= 1e-3 * max(1.0, abs(m[b, h]))
                o_gpu = codec.unrotate(g[b, h, :128][None, :], vop.D)[0] / g[b, h, 129]
                o_ref = o[b, h] / lsum[b, h]
                assert np.linalg.norm(o_gpu - o_ref) <= 2e-3 * np.linalg.norm(o_ref), (b, h)
    out = torch.full((B, Hq, 128), float("nan"), device="cuda")
    tq.tq_decode_attn_merge(vp, torch.stack(parts), out)
    got = out.cpu().numpy()
    ref = estimate.decode_attention(q, kop.D, kop.S, ke["idx"], ke["signs"], ke["norm_f16"], ke["rnorm_f16"], kop.c,
                                    kop.m, vop.D, ve["idx"], ve["norm_f16"], vop.c, 128, seq_lens, Hq, Hkv, T)
    for b in range(B):
        for h in range(Hq):
            if seq_lens[b] == 0:
                assert np.all(got[b, h] == 0)
            else:
                assert np.linalg.norm(got[b, h] - ref[b, h]) <= 2e-3 * np.linalg.norm(ref[b, h]), (b, h)


def test_search_merge_lists_exact():
    rng = np.random.default_rng(8)
    n_parts, n_q, k = 5, 33, 10
    offs = [0, 100, 250, 251, 400]
    ids = np.stack([np.stack([rng.permutation(np.arange(100))[:k] for _ in range(n_q)]) for _ in range(n_parts)])
    sc = np.round(rng.standard_normal((n_parts, n_q, k)), 1).astype(np.float32)   # ties across parts
    ids[2, :, 7:] = 2147483647                                                     # empty slots
    sc[2, :, 7:] = -np.inf
    oi = torch.empty((n_q, k), dtype=torch.int32, device="cuda")
    os_ = torch.empty((n_q, k), dtype=torch.float32, device="cuda")
    tq.tq_search_merge(dev(ids.astype(np.int32)), dev(sc), offs, k, oi, os_)
    gi, gs = oi.cpu().numpy(), os_.cpu().numpy()
    ri, rs = estimate.merge_topk([np.where(i == 2147483647, -1, i) for i in ids], list(sc), offs, k)
    np.testing.assert_array_equal(gi, ri)
    np.testing.assert_array_equal(gs, rs.astype(np.float32))


def test_search_shards_equal_whole_database():
    n_db, n_q, k, d = 5000, 40, 10, 200
    p, op = make_pair(d, 4, tq.TQ_MODE_PROD)
    db = torch.from_numpy(wl.search_set(n_db, d, seed=3)).to(torch.bfloat16).cuda()
    qs = torch.from_numpy(wl.search_set(n_q, d, seed=4)).cuda()
    codes = torch.empty(p.code_bytes(n_db), dtype=torch.uint8, device="cuda")
    nn = torch.empty(n_db, dtype=torch.int16, device="cuda")
    rn = torch.empty(n_db, dtype=torch.int16, device="cuda")
    tq.tq_quantize(p, db, codes, nn, rn)

    def search(c, n, r, cnt):
        ids = torch.empty((n_q, k), dtype=torch.int32, device="cuda")
        sc = torch.empty((n_q, k), dtype=torch.float32, device="cuda")
        ws = torch.empty(tq.tq_search_workspace(p, n_q, cnt, k), dtype=torch.uint8, device="cuda")
        tq.tq_search_topk(p, qs, c, n, r, cnt, k, ids, sc, ws)
        return ids, sc

    whole_i, whole_s = search(codes, nn, rn, n_db)
    bounds = [0, 1600, 3200, n_db]                   # shard starts on whole 32-vector tiles
    tb = p.code_bytes(32)
    parts_i, parts_s = [], []
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        c = codes[lo // 32 * tb: lo // 32 * tb + p.code_bytes(hi - lo)]
        i, s = search(c, nn[lo:hi], rn[lo:hi], hi - lo)
        parts_i.append(i)
        parts_s.append(s)
    oi = torch.empty((n_q, k), dtype=torch.int32, device="cuda")
    os_ = torch.empty((n_q, k), dtype=torch.float32, device="cuda")
    tq.tq_search_merge(torch.stack(parts_i), torch.stack(parts_s), bounds[:-1], k, oi, os_)
    assert torch.equal(oi, whole_i)
    assert torch.equal(os_, whole_s)
