"""tq_logits_noalloc: the entry point for callers that cannot allocate device
memory when they call (graph capture, host frameworks that own all device
buffers).  It must give the same logits as tq_logits with a caller workspace,
on two calls in a row (the static scratch keeps the previous call's
contents), and reject requests larger than its static scratch.

Collected last on purpose (file name), so a stop-at-first-failure run has
already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import vector_quantization_randomized_b200 as tq
import workloads as wl
from gpu_util import make_pair, oracle_codes, logit_tolerance

pytestmark = pytest.mark.gpu


def _case(n_heads, group, n_keys, bits, seed):
    p, op = make_pair(128, bits, tq.TQ_MODE_PROD)
    keys = np.concatenate([wl.to_bf16(wl.head_vectors(n_keys, 128, seed=seed, head=h)) for h in range(n_heads)])
    q = wl.queries(n_heads * group, 128, seed=seed + 7)
    codes, norms, rnorms, _ = oracle_codes(op, keys)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return p, dev(q), dev(codes), dev(norms.view(np.int16)), dev(rnorms.view(np.int16)), norms, q


def _call_noalloc(p, q, group, codes, norms, rnorms, n_keys, n_heads, out):
    # straight through the C ABI
    rc = tq._lib.tq_logits_noalloc(p.ref, q.data_ptr(), q.shape[0], group, codes.data_ptr(), norms.data_ptr(),
                                   rnorms.data_ptr(), n_keys, n_heads, out.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
    assert rc == tq.TQ_OK, tq.tq_last_error()


def test_noalloc_matches_workspace_entry_point_twice():
    torch.cuda.init()
    cases = [(8, 4, 3000, 4, 1), (2, 5, 777, 3, 2)]   # different shapes so the second call rewrites the scratch
    for (n_heads, group, n_keys, bits, seed) in cases:
        p, q, codes, norms, rnorms, norms_h, q_h = _case(n_heads, group, n_keys, bits, seed)
        ref = torch.empty((q.shape[0], n_keys), dtype=torch.float32, device="cuda")
        ws = torch.empty(tq.tq_logits_workspace(p, q.shape[0]), dtype=torch.uint8, device="cuda")
        tq.tq_logits(p, q, group, codes, norms, rnorms, n_keys, n_heads, ref, ws)
        for _ in range(2):
            out = torch.full((q.shape[0], n_keys), float("nan"), dtype=torch.float32, device="cuda")
            _call_noalloc(p, q, group, codes, norms, rnorms, n_keys, n_heads, out)
            torch.cuda.synchronize()
            r = ref.cpu().numpy().astype(np.float64)
            o = out.cpu().numpy().astype(np.float64)
            for h in range(q.shape[0]):
                g = h // group
                tol = logit_tolerance(r[h:h + 1], norms_h[g * n_keys:(g + 1) * n_keys], q_h[h:h + 1])[0]
                assert np.all(np.abs(o[h] - r[h]) <= tol)


def test_noalloc_rejects_oversized_request():
    p, q, codes, norms, rnorms, _, _ = _case(1, 4, 64, 4, 3)
    limit = tq.tq_logits_noalloc_max_scratch()
    assert limit == 1 << 20
    n_heads = 1000   # 1000 chunks of query prep far exceed 1 MiB
    big_q = torch.zeros((n_heads * 4, 128), dtype=torch.float32, device="cuda")
    out = torch.zeros(1, device="cuda")
    rc = tq._lib.tq_logits_noalloc(p.ref, big_q.data_ptr(), n_heads * 4, 4, codes.data_ptr(), norms.data_ptr(),
                                   rnorms.data_ptr(), 64, n_heads, out.data_ptr(), None)
    assert rc == tq.TQ_EINVAL
    assert "static" in tq.tq_last_error()
