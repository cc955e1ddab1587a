"""Pins of the sharded forms of the oracle (the multi-device paths): the LSE merge of
decode partials over any token split equals one decode over all tokens, and the merge
of per-shard top-k lists equals the top-k of the whole score matrix (brute force,
with ties placed across shard boundaries)."""
import numpy as np

from oracle import codec, estimate
from oracle.codebook import stored_codebook
from oracle.params import sign_flips, qjl_matrix


def _kv(B, Hkv, T, d, seed):
    kc, kt = stored_codebook(128, 2)
    vc, vt = stored_codebook(128, 3)
    kD, vD = sign_flips(42, 128), sign_flips(43, 128)
    S = qjl_matrix(42, 128, 128)
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((B * Hkv * T, d)) * 3.0
    V = rng.standard_normal((B * Hkv * T, d))
    ke = codec.encode(K, kD, kc, kt, S)
    ve = codec.encode(V, vD, vc, vt)
    return dict(kc=kc, vc=vc, kD=kD, vD=vD, S=S, ke=ke, ve=ve)


def _shard(arr, B, Hkv, T, t0, t1):
    """Rows of tokens [t0, t1) of every (sequence, head), laid out as a cache of t1 - t0 tokens."""
    a = np.asarray(arr).reshape((B * Hkv, T) + np.asarray(arr).shape[1:])
    return a[:, t0:t1].reshape((-1,) + np.asarray(arr).shape[1:])


def test_decode_partials_merge_to_full_decode():
    B, Hkv, Hq, T, d = 2, 2, 4, 20, 128
    kv = _kv(B, Hkv, T, d, 3)
    ke, ve = kv["ke"], kv["ve"]
    q = np.random.default_rng(4).standard_normal((B, Hq, d))
    seq_lens = [20, 7]
    args = lambda idx, sg, kn, krn, vi, vn: (q, kv["kD"], kv["S"], idx, sg, kn, krn, kv["kc"], 128, kv["vD"], vi, vn,
                                             kv["vc"], d)
    full = estimate.decode_attention(*args(ke["idx"], ke["signs"], ke["norm_f16"], ke["rnorm_f16"], ve["idx"],
                                           ve["norm_f16"]), seq_lens, Hq, Hkv, T)
    for bounds in ([0, 10, 20], [0, 3, 9, 20], [0, 7, 20, 20]):   # the last split has an empty shard
        parts = []
        for t0, t1 in zip(bounds[:-1], bounds[1:]):
            sh = lambda a: _shard(a, B, Hkv, T, t0, t1)
            local = [max(0, min(L - t0, t1 - t0)) for L in seq_lens]
            parts.append(estimate.decode_partial(*args(sh(ke["idx"]), sh(ke["signs"]), sh(ke["norm_f16"]),
                                                       sh(ke["rnorm_f16"]), sh(ve["idx"]), sh(ve["norm_f16"])),
                                                 local, Hq, Hkv, t1 - t0))
        np.testing.assert_allclose(estimate.merge_partials(parts), full, rtol=1e-12, atol=1e-13)


def test_decode_partial_empty_and_single():
    B, Hkv, Hq, T, d = 1, 1, 2, 5, 128
    kv = _kv(B, Hkv, T, d, 5)
    ke, ve = kv["ke"], kv["ve"]
    q = np.random.default_rng(6).standard_normal((B, Hq, d))
    a = (q, kv["kD"], kv["S"], ke["idx"], ke["signs"], ke["norm_f16"], ke["rnorm_f16"], kv["kc"], 128, kv["vD"],
         ve["idx"], ve["norm_f16"], kv["vc"], d)
    m, lsum, o = estimate.decode_partial(*a, [0], Hq, Hkv, T)
    assert np.all(np.isneginf(m)) and np.all(lsum == 0) and np.all(o == 0)
    assert np.all(estimate.merge_partials([(m, lsum, o), (m, lsum, o)]) == 0)
    m1, l1, o1 = estimate.decode_partial(*a, [1], Hq, Hkv, T)   # one token: weight 1, o = v_hat_0
    np.testing.assert_allclose(l1, 1.0)
    vhat = estimate.dequant_mse(ve["idx"][:1], ve["norm_f16"][:1], kv["vc"], kv["vD"], d)
    np.testing.assert_allclose(o1[0], np.repeat(vhat, Hq, axis=0), rtol=1e-12)


def test_topk_merge_equals_global_topk():
    rng = np.random.default_rng(7)
    n_q, n_db, k = 6, 300, 10
    scores = np.round(rng.standard_normal((n_q, n_db)), 1)     # many exact ties, across shards too
    ref_i, ref_s = estimate.topk(scores, k)
    for bounds in ([0, 150, 300], [0, 1, 101, 299, 300], [0, 5, 300]):
        ids_p, sc_p, offs = [], [], []
        for t0, t1 in zip(bounds[:-1], bounds[1:]):
            li, ls = estimate.topk(scores[:, t0:t1], min(k, t1 - t0))
            if li.shape[1] < k:                                  # a shard smaller than k: empty slots
                pad = k - li.shape[1]
                li = np.concatenate([li, -np.ones((n_q, pad), np.int64)], axis=1)
                ls = np.concatenate([ls, np.full((n_q, pad), -np.inf)], axis=1)
            ids_p.append(li)
            sc_p.append(ls)
            offs.append(t0)
        gi, gs = estimate.merge_topk(ids_p, sc_p, offs, k)
        np.testing.assert_array_equal(gi, ref_i)
        np.testing.assert_array_equal(gs, ref_s)
