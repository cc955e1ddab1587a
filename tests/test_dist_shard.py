"""The sharded multi-device paths on CPU: world size 2 over gloo.

Each rank holds one shard of a small problem and runs the orchestration of
vector_quantization_randomized_b200.parallel with the oracle standing in for
the per-rank kernels and the merges (the GPU kernels themselves are checked
against the oracle in tests/test_gpu_shards.py):

* search over a database split by shard_bounds: per-rank top-k lists with
  shard-local ids, all-gathered, merged with the shard offsets - equal to the
  top-k of one search over the whole database (ties included);
* decode attention over a sequence split by token ranges (one sequence shorter
  than a shard, so a rank holds no token of it): per-rank partials (m, l, o)
  all-gathered and merged - equal to one decode over all tokens.
"""
import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem():
    from oracle import codec
    from oracle.codebook import stored_codebook
    from oracle.params import sign_flips, qjl_matrix
    B, Hkv, Hq, T, d = 2, 2, 4, 24, 128
    kc, kt = stored_codebook(128, 2)
    vc, vt = stored_codebook(128, 3)
    kD, vD = sign_flips(42, 128), sign_flips(43, 128)
    S = qjl_matrix(42, 128, 128)
    rng = np.random.default_rng(21)
    K = rng.standard_normal((B * Hkv * T, d)) * 3.0
    V = rng.standard_normal((B * Hkv * T, d))
    q = rng.standard_normal((B, Hq, d))
    return dict(B=B, Hkv=Hkv, Hq=Hq, T=T, d=d, kc=kc, vc=vc, kD=kD, vD=vD, S=S, q=q, seq_lens=[24, 9],
                ke=codec.encode(K, kD, kc, kt, S), ve=codec.encode(V, vD, vc, vt))


def _decode_args(P, sl):
    ke, ve = P["ke"], P["ve"]
    return (P["q"], P["kD"], P["S"], sl(ke["idx"]), sl(ke["signs"]), sl(ke["norm_f16"]), sl(ke["rnorm_f16"]),
            P["kc"], 128, P["vD"], sl(ve["idx"]), sl(ve["norm_f16"]), P["vc"], P["d"])


def _rank_main(rank, world, port, out_q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from vector_quantization_randomized_b200 import parallel
    from oracle import estimate
    errs = []

    # ---- search: database of 1000 rows split over the ranks
    rng = np.random.default_rng(5)
    n_db, n_q, k = 1001, 7, 10
    scores = np.round(rng.standard_normal((n_q, n_db)), 1)      # exact ties, some across the shard boundary
    lo, hi = parallel.shard_bounds(n_db, world, rank)

    def local_topk():
        i, s = estimate.topk(scores[:, lo:hi], k)
        return torch.from_numpy(i.astype(np.int32)), torch.from_numpy(s.astype(np.float64))

    def merge(ids, sc, offsets):
        gi, gs = estimate.merge_topk(list(ids.numpy()), list(sc.numpy()), offsets, k)
        return gi, gs

    gi, gs = parallel.sharded_search_topk(local_topk, merge, n_db)
    ri, rs = estimate.topk(scores, k)
    if not (np.array_equal(gi, ri) and np.array_equal(gs, rs)):
        errs.append("search merge differs from the one-rank top-k")

    # ---- decode: every sequence split by token ranges
    P = _problem()
    B, Hkv, Hq, T = P["B"], P["Hkv"], P["Hq"], P["T"]
    t0, t1 = parallel.shard_bounds(T, world, rank)
    sl_local = parallel.local_seq_lens(torch.tensor(P["seq_lens"], dtype=torch.int32), t0, t1).tolist()

    def shard(a):
        a = np.asarray(a)
        return a.reshape((B * Hkv, T) + a.shape[1:])[:, t0:t1].reshape((-1,) + a.shape[1:])

    def local_partial():
        m, lsum, o = estimate.decode_partial(*_decode_args(P, shard), sl_local, Hq, Hkv, t1 - t0)
        return torch.from_numpy(np.concatenate([o, m[..., None], lsum[..., None]], axis=-1))

    def merge_parts(parts):
        parts = parts.numpy()
        return estimate.merge_partials([(p[..., -2], p[..., -1], p[..., :-2]) for p in parts])

    out = parallel.sequence_split_decode(local_partial, merge_parts)
    full = estimate.decode_attention(*_decode_args(P, lambda a: a), P["seq_lens"], Hq, Hkv, T)
    if not np.allclose(out, full, rtol=1e-12, atol=1e-13):
        errs.append(f"decode merge differs from the one-rank decode: {np.abs(out - full).max()}")
    if rank == 1 and sl_local[1] != 0:
        errs.append("the short sequence should have no token on rank 1")
    dist.barrier()
    dist.destroy_process_group()
    out_q.put((rank, errs))


def test_sharded_search_and_sequence_split_decode_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, errs in res:
        assert not errs, (r, errs)


def test_shard_bounds_cover_exactly():
    sys.path.insert(0, ROOT)
    from vector_quantization_randomized_b200.parallel import shard_bounds
    for n in (0, 1, 7, 1000, 1001):
        for world in (1, 2, 3, 8):
            b = [shard_bounds(n, world, r) for r in range(world)]
            assert b[0][0] == 0 and b[-1][1] == n
            assert all(b[r][1] == b[r + 1][0] for r in range(world - 1))
            sizes = [hi - lo for lo, hi in b]
            assert max(sizes) - min(sizes) <= 1
