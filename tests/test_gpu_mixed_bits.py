"""Logits over a sequence with mixed bit widths (temporal decay, zhidx
turboquant_plus article: older tokens kept at fewer bits): per KV head the
first n_old keys are b = 2 product codes, the next n_new keys b = 4, each
segment scanned by its own tq_logits_ld call into one [n_q][n_old + n_new]
matrix.  Compared with the oracle's estimate of each segment; the
tensor-memory scan (key counts multiples of 32) and the general scan (ragged
counts) both appear."""
import numpy as np
import pytest
import torch

import vector_quantization_randomized_b200 as tq
import workloads as wl
from oracle import estimate
from gpu_util import make_pair, oracle_codes, logit_tolerance

pytestmark = pytest.mark.gpu
dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("n_old,n_new,group", [(2048, 1024, 4), (1000, 333, 4), (512, 96, 2)])
def test_two_width_segments_into_one_matrix(n_old, n_new, group):
    H, d = 2, 128
    total = n_old + n_new
    q = wl.queries(H * group, d, seed=11)
    out = torch.full((H * group, total + 5), float("nan"), device="cuda")
    refs = []
    for (bits, n, off, seed) in ((2, n_old, 0, 21), (4, n_new, n_old, 22)):
        p, op = make_pair(d, bits, tq.TQ_MODE_PROD)
        keys = np.concatenate([wl.to_bf16(wl.head_vectors(n, d, seed=seed, head=h)) for h in range(H)])
        codes, norms, rnorms, enc = oracle_codes(op, keys)
        ref = estimate.logits_gqa(q, op.D, op.S, enc["idx"], enc["signs"], norms, rnorms, op.c, op.m, H, group, n)
        ws = torch.empty(tq.tq_logits_workspace(p, H * group), dtype=torch.uint8, device="cuda")
        tq.tq_logits_ld(p, dev(q), group, dev(codes), dev(norms.view(np.int16)), dev(rnorms.view(np.int16)), n, H,
                        out[:, off:], total + 5, ws)
        refs.append((ref, norms, off, n))
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.isnan(got[:, total:]))              # columns past the sequence untouched
    for ref, norms, off, n in refs:
        for h in range(H * group):
            g = h // group
            tol = logit_tolerance(ref[h:h + 1], norms[g * n:(g + 1) * n], q[h:h + 1])[0]
            assert np.all(np.abs(got[h, off:off + n] - ref[h]) <= tol), (off, h)
