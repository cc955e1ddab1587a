"""tq_logits_noalloc: the entry point for callers that cannot allocate device
memory when they call (graph capture, host frameworks that own all device
buffers).  It runs the same kernels as tq_logits with a caller workspace, so
its logits must be bit-identical to tq_logits's, on two calls in a row (the
static scratch keeps the previous call's contents), on both the tensor-core
path (no scratch) and the other shapes (query preparation in the scratch).
The largest request that fits the static scratch is accepted and matches;
one more KV head is rejected.

Collected last on purpose (file name), so a stop-at-first-failure run has
already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import vector_quantization_randomized_b200 as tq
import workloads as wl
from gpu_util import make_pair, oracle_codes

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


def _reference(p, q, group, codes, norms, rnorms, n_keys, n_heads):
    ref = torch.empty((q.shape[0], n_keys), dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.tq_logits_workspace(p, q.shape[0]), dtype=torch.uint8, device="cuda")
    tq.tq_logits(p, q, group, codes, norms, rnorms, n_keys, n_heads, ref, ws)
    return ref


def test_noalloc_matches_workspace_entry_point_twice():
    torch.cuda.init()
    # tensor-core path, then two shapes that keep their query preparation in the scratch
    # (group 5; n_keys not a multiple of 32), so the later calls rewrite the scratch
    cases = [(8, 4, 3008, 4, 1), (2, 5, 777, 3, 2), (3, 4, 1000, 4, 4)]
    for (n_heads, group, n_keys, bits, seed) in cases:
        p, q, codes, norms, rnorms, norms_h, q_h = _case(n_heads, group, n_keys, bits, seed)
        ref = _reference(p, q, group, codes, norms, rnorms, n_keys, n_heads)
        for _ in range(2):
            out = torch.full((q.shape[0], n_keys), float("nan"), dtype=torch.float32, device="cuda")
            _call_noalloc(p, q, group, codes, norms, rnorms, n_keys, n_heads, out)
            torch.cuda.synchronize()
            assert torch.equal(out, ref)


def test_noalloc_scratch_boundary():
    """At b = 4 a chunk of 4 queries takes 12352 bytes of scratch; with group 8 (two chunks
    per KV head) 42 KV heads need 1037568 bytes (accepted, identical logits) and 43 need
    1062272 (rejected, nothing launched)."""
    limit = tq.tq_logits_noalloc_max_scratch()
    assert limit == 1 << 20
    group, n_keys = 8, 64
    p, q, codes, norms, rnorms, _, _ = _case(42, group, n_keys, 4, 5)
    ref = _reference(p, q, group, codes, norms, rnorms, n_keys, 42)
    out = torch.full((42 * group, n_keys), float("nan"), dtype=torch.float32, device="cuda")
    _call_noalloc(p, q, group, codes, norms, rnorms, n_keys, 42, out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    p43, q43, codes43, norms43, rnorms43, _, _ = _case(43, group, n_keys, 4, 6)
    out43 = torch.zeros((43 * group, n_keys), dtype=torch.float32, device="cuda")
    rc = tq._lib.tq_logits_noalloc(p43.ref, q43.data_ptr(), 43 * group, group, codes43.data_ptr(),
                                   norms43.data_ptr(), rnorms43.data_ptr(), n_keys, 43, out43.data_ptr(), None)
    assert rc == tq.TQ_EINVAL
    assert "static" in tq.tq_last_error()
    torch.cuda.synchronize()
    assert not torch.any(out43)   # nothing was written


def test_noalloc_tensor_core_path_needs_no_scratch():
    """600 KV heads x 4 queries would need far more than the static scratch on the other
    path; on the tensor-core path they need none and are accepted."""
    p, q, codes, norms, rnorms, _, _ = _case(600, 4, 32, 3, 7)
    ref = _reference(p, q, 4, codes, norms, rnorms, 32, 600)
    out = torch.full((2400, 32), float("nan"), dtype=torch.float32, device="cuda")
    _call_noalloc(p, q, 4, codes, norms, rnorms, 32, 600, out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
