"""GPU parity of tq_search_topk against the oracle: top-k by the logit
estimate (group 1), descending, ties to the lower id.  The returned set equals
the oracle's except among candidates whose oracle scores lie within the logit
tolerance of the k-th score; returned scores match the oracle's scores of the
same ids within the logit tolerance (1e-4 |l| + 1e-5 n ||q||)."""
import numpy as np
import pytest
import torch

import vector_quantization_randomized_b200 as tq
import workloads as wl
from oracle import estimate
from gpu_util import make_pair, oracle_codes

pytestmark = pytest.mark.gpu


def _check(d, bits, n_db, n_q, k, seed=0, mode=tq.TQ_MODE_PROD):
    p, op = make_pair(d, bits, mode, seed=42)
    db = wl.to_bf16(wl.search_set(n_db, d, seed=seed))
    q = wl.search_set(n_q, d, seed=seed + 1)
    codes, norms, rnorms, enc = oracle_codes(op, db)
    q_rot, u = estimate.prep_queries(q, op.D, op.S)
    ref = estimate.logits_from_codes(q_rot, u, enc["idx"], enc.get("signs"), norms, rnorms, op.c, op.m)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    ids = torch.full((n_q, k), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((n_q, k), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.tq_search_workspace(p, n_q, n_db, k), dtype=torch.uint8, device="cuda")
    tq.tq_search_topk(p, dev(q), dev(codes), dev(norms.view(np.int16)),
                      dev(rnorms.view(np.int16)) if rnorms is not None else None, n_db, k, ids, sc, ws)
    gi = ids.cpu().numpy().astype(np.int64)
    gs = sc.cpu().numpy().astype(np.float64)
    qn = np.linalg.norm(q.astype(np.float64), axis=1)
    rid, rs = estimate.topk(ref, k)
    for r in range(n_q):
        assert np.all((gi[r] >= 0) & (gi[r] < n_db)) and len(set(gi[r])) == k
        tol_all = 1e-4 * np.abs(ref[r]) + 1e-5 * qn[r] * norms.astype(np.float64)
        # scores of the returned ids
        assert np.all(np.abs(gs[r] - ref[r, gi[r]]) <= tol_all[gi[r]]), r
        # descending order by returned score
        assert np.all(np.diff(gs[r]) <= 0)
        kth = rs[r, -1]
        tk = tol_all[rid[r, -1]]
        must = set(np.nonzero(ref[r] > kth + 2 * tk)[0])
        may = set(np.nonzero(ref[r] >= kth - 2 * tk)[0])
        got = set(gi[r])
        assert must <= got <= may, (r, sorted(must - got), sorted(got - may))


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_search_d200(bits):
    _check(200, bits, n_db=20000, n_q=37, k=10)


def test_search_d200_mse_codes_many_splits():
    """MSE-only codes (no sign plane); 40000 vectors make three database splits whose last
    item is ragged, and 33 queries three chunks of 16 (the last one with one query)."""
    _check(200, 3, n_db=40003, n_q=33, k=16, seed=3, mode=tq.TQ_MODE_MSE)


def test_search_d128_b4():
    _check(128, 4, n_db=9001, n_q=8, k=16)


def test_search_small_db_and_k1():
    _check(200, 2, n_db=45, n_q=5, k=10)
    _check(200, 4, n_db=1000, n_q=3, k=1)
