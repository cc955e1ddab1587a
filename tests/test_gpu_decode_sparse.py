"""GPU parity of tq_decode_attn_sparse (Sparse V, zhidx turboquant_plus
article, "Sparse V") against the oracle: with v_eps = 0 it is exactly
tq_decode_attn; with v_eps > 0 the output lies within the Sparse V bound
v_eps * sum_{p_t < v_eps} |v_hat_t| of both the oracle's full output and its
Sparse V output (the kernel drops a subset of the oracle's tokens), plus the
decode tolerance 2e-3 |o|.  Shapes cover the staged kernel (max_tokens a
multiple of 32) and the plain one, several 256-token splits, ragged lengths
and GQA groups; a large softmax scale makes the attention peaked so that
many tokens fall below v_eps."""
import numpy as np
import pytest
import torch

import vector_quantization_randomized_b200 as tq
import workloads as wl
from oracle import estimate
from gpu_util import make_pair, oracle_codes

pytestmark = pytest.mark.gpu
dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _setup(B, Hkv, Hq, T, d=128):
    kp, kop = make_pair(d, 3, tq.TQ_MODE_PROD, seed=42)
    vp, vop = make_pair(d, 3, tq.TQ_MODE_MSE, seed=43)
    K = wl.kv_block(B, Hkv, T, d, seed=wl.SEED_KEYS).reshape(-1, d)
    V = wl.kv_block(B, Hkv, T, d, seed=wl.SEED_VALUES).reshape(-1, d)
    q = wl.queries(B * Hq, d, seed=wl.SEED_QUERIES).reshape(B, Hq, d)
    kc, kn, krn, ke = oracle_codes(kop, K)
    vc, vn, _, ve = oracle_codes(vop, V)
    return kp, kop, vp, vop, q, kc, kn, krn, ke, vc, vn, ve


def _run(fn, kp, vp, q, Hkv, kc, kn, krn, vc, vn, seq_lens, T, scale, **kw):
    B, Hq, d = q.shape
    out = torch.full((B, Hq, d), float("nan"), device="cuda")
    ws = torch.empty(tq.tq_decode_attn_workspace(kp, B, Hq, Hkv, T), dtype=torch.uint8, device="cuda")
    sl = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    fn(kp, vp, dev(q), Hkv, dev(kc), dev(kn.view(np.int16)), dev(krn.view(np.int16)), dev(vc),
       dev(vn.view(np.int16)), sl, T, out, ws, scale=scale, **kw)
    return out


@pytest.mark.parametrize("T,seq_lens", [(1024, [1024, 700]), (1100, [1100, 517])])
def test_zero_threshold_is_exactly_the_full_kernel(T, seq_lens):
    kp, kop, vp, vop, q, kc, kn, krn, ke, vc, vn, ve = _setup(2, 2, 8, T)
    full = _run(tq.tq_decode_attn, kp, vp, q, 2, kc, kn, krn, vc, vn, seq_lens, T, 0.0)
    sp = _run(tq.tq_decode_attn_sparse, kp, vp, q, 2, kc, kn, krn, vc, vn, seq_lens, T, 0.0, v_eps=0.0)
    assert torch.equal(full, sp)


@pytest.mark.parametrize("T,seq_lens,Hq,eps", [
    (1024, [1024, 1000], 8, 1e-3),   # staged kernel, two splits
    (2048, [2048, 33], 4, 1e-4),     # staged, four splits, a 33-token sequence
    (1100, [1100, 517], 8, 1e-3),    # plain kernel
    (1024, [900], 5, 1e-2),          # group of 5 (a chunk with one query head)
])
def test_within_sparse_v_bound(T, seq_lens, Hq, eps):
    B, Hkv, d, scale = len(seq_lens), 1, 128, 1.0
    kp, kop, vp, vop, q, kc, kn, krn, ke, vc, vn, ve = _setup(B, Hkv, Hq, T)
    args = (q, kop.D, kop.S, ke["idx"], ke["signs"], kn, krn, kop.c, kop.m, vop.D, ve["idx"], vn, vop.c, d,
            seq_lens, Hq, Hkv, T)
    bound = np.zeros((B, Hq))
    ref_full = estimate.decode_attention(*args, scale=scale)
    ref_sp = estimate.decode_attention(*args, scale=scale, v_eps=eps, bound=bound)
    got = _run(tq.tq_decode_attn_sparse, kp, vp, q, Hkv, kc, kn, krn, vc, vn, seq_lens, T, scale,
               v_eps=eps).cpu().numpy().astype(np.float64)
    assert np.mean(bound > 0) > 0.5  # the threshold actually drops tokens in most rows
    for b in range(B):
        for h in range(Hq):
            tol = bound[b, h] + 2e-3 * np.linalg.norm(ref_full[b, h])
            assert np.linalg.norm(got[b, h] - ref_full[b, h]) <= tol, (b, h)
            assert np.linalg.norm(got[b, h] - ref_sp[b, h]) <= tol, (b, h)


def test_rejects_negative_threshold():
    kp, kop, vp, vop, q, kc, kn, krn, ke, vc, vn, ve = _setup(1, 1, 4, 64)
    with pytest.raises(tq.TQError):
        _run(tq.tq_decode_attn_sparse, kp, vp, q, 1, kc, kn, krn, vc, vn, [64], 64, 0.0, v_eps=-1.0)
